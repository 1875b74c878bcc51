"""The decode entry point for callers that cannot allocate device memory.

pkv_paged_attention_decode_static_ws takes no workspace: its split-K
scratch is a fixed area the library keeps on each device.  It serves
callers that must not call cudaMalloc (code under a framework's caching
allocator that has reserved the GPU's memory, or on a latency-critical path
where an allocation may synchronise the device).  These tests call it
through the C ABI and check it bit for bit against pkv_paged_attention_decode
with a caller-owned workspace (and once against the oracle), on two calls in
a row with different inputs, so a value left in the shared scratch area by
the first call would show up in the second; the Python wrapper is checked
the same way.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2, "f32": 1e-5}


def _prepare(wl, values):
    import paged_kv_cache_365_b200 as pkv
    from paged_kv_cache_365_b200.replay import build_step
    st = build_step(wl, values, "cuda")
    c = st["cache"]
    pkv.copy_blocks(c.k, c.v, st["cow_pairs"])
    pkv.kv_append(st["k_new"], st["v_new"], c.k, c.v, st["slot_mapping"])
    return st


def _call_static(st, wl, out):
    from paged_kv_cache_365_b200 import _lib
    c = st["cache"]
    dt = {"f32": 0, "f16": 1, "bf16": 2}[wl.dtype]
    stream = torch.cuda.current_stream().cuda_stream
    return _lib.lib.pkv_paged_attention_decode_static_ws(
        out.data_ptr(), st["q"].data_ptr(), c.k.data_ptr(), c.v.data_ptr(), st["block_tables"].data_ptr(),
        st["block_tables"].shape[1], st["context_lens"].data_ptr(), st["max_context_len"], wl.B, wl.Hq,
        wl.Hkv, wl.D, wl.num_blocks, ctypes.c_float(wl.scale), 0, dt, ctypes.c_void_p(stream))


def test_static_scratch_decode_matches_workspace_decode_twice():
    """Two C-ABI calls in a row on the shared scratch area: each output is
    bit-identical to the caller-workspace decode (the same kernels on the
    same partitions, with the same fixed summation order), and the first is
    also within tolerance of the fp64 oracle."""
    import numpy as np
    import oracle
    import paged_kv_cache_365_b200 as pkv
    cases = [
        workloads.custom([1, 600, 1100, 2000, 33, 1537], Hq=32, Hkv=8, D=128, dtype="bf16", seed=21,
                         name="no_alloc_a"),
        workloads.custom([2047, 5, 900, 513, 1024], Hq=16, Hkv=16, D=128, dtype="f16", seed=22,
                         name="no_alloc_b"),
    ]
    prepared, wants, gots, vals = [], [], [], []
    for wl in cases:
        v = workloads.draw_values(wl)
        st = _prepare(wl, v)
        need = pkv.decode_workspace_bytes(wl.B, wl.Hq, wl.D, st["max_context_len"])
        assert 0 < need <= pkv._lib.STATIC_WORKSPACE_BYTES  # the split-K path really uses the scratch
        c = st["cache"]
        wants.append(pkv.paged_attention_decode(st["q"], c.k, c.v, st["block_tables"], st["context_lens"],
                                                st["max_context_len"], wl.scale))
        gots.append(torch.full_like(wants[-1], float("nan")))
        prepared.append(st)
        vals.append(v)
    torch.cuda.synchronize()
    # two calls in a row on the shared scratch area
    for wl, st, got in zip(cases, prepared, gots):
        assert _call_static(st, wl, got) == 0
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    for wl, want, got in zip(cases, wants, gots):
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), wl.name
    # the first call's output against the oracle itself
    wl, v = cases[0], vals[0]
    ref = oracle.replay(wl, v)
    exact = oracle.paged_decode(v["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"], ref["context_lens"],
                                wl.scale, wl.dtype)
    err = float(np.abs(gots[0].float().cpu().numpy().astype(np.float64) - exact).max())
    assert err <= TOL[wl.dtype], err


def test_static_scratch_python_wrapper():
    """The binding's wrapper (argument order, the out= path) gives the same
    bits as the C-ABI call, and raises PkvError when the call needs more
    scratch than the fixed area holds."""
    import paged_kv_cache_365_b200 as pkv
    wl = workloads.custom([700, 1500, 64], Hq=16, Hkv=4, D=64, dtype="f16", seed=23, name="no_alloc_py")
    st = _prepare(wl, workloads.draw_values(wl))
    c = st["cache"]
    ref = torch.full_like(st["q"], float("nan"))
    assert _call_static(st, wl, ref) == 0
    out = torch.full_like(st["q"], float("nan"))
    got = pkv.paged_attention_decode_static_ws(st["q"], c.k, c.v, st["block_tables"], st["context_lens"],
                                               st["max_context_len"], wl.scale, out=out)
    torch.cuda.synchronize()
    assert got is out
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    B, Hq, Hkv, D, nb, max_blocks = 2000, 64, 8, 128, 32, 4096
    q = torch.zeros(B, Hq, D, dtype=torch.float16, device="cuda")
    kc = torch.zeros(nb, Hkv, 16, D, dtype=torch.float16, device="cuda")
    bt = torch.zeros(B, max_blocks, dtype=torch.int32, device="cuda")
    cl = torch.zeros(B, dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PkvError):
        pkv.paged_attention_decode_static_ws(q, kc, kc, bt, cl, 16 * max_blocks, 0.1, out=torch.empty_like(q))


def test_static_scratch_rejects_oversized_requests():
    from paged_kv_cache_365_b200 import _lib
    import paged_kv_cache_365_b200 as pkv
    B, Hq, Hkv, D, nb, max_blocks = 2000, 64, 8, 128, 32, 4096
    big_ctx = 16 * max_blocks
    assert pkv.decode_workspace_bytes(B, Hq, D, big_ctx) > _lib.STATIC_WORKSPACE_BYTES
    # every buffer is sized for the claimed batch and every length is 0, so
    # even a launch would stay in bounds (and would only write zeros)
    q = torch.zeros(B, Hq, D, dtype=torch.float16, device="cuda")
    out = torch.full_like(q, float("nan"))
    kc = torch.zeros(nb, Hkv, 16, D, dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    bt = torch.zeros(B, max_blocks, dtype=torch.int32, device="cuda")
    cl = torch.zeros(B, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = _lib.lib.pkv_paged_attention_decode_static_ws(
        out.data_ptr(), q.data_ptr(), kc.data_ptr(), vc.data_ptr(), bt.data_ptr(), max_blocks, cl.data_ptr(),
        big_ctx, B, Hq, Hkv, D, nb, ctypes.c_float(0.1), 0, 1, ctypes.c_void_p(stream))
    assert rc == _lib.PKV_EINVAL
    torch.cuda.synchronize()
    assert torch.isnan(out).all().item()  # nothing was launched
