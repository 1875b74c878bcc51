"""Full-size GPU parity of the next rows on the BASELINE-sized workloads
(the same shapes the bench measures): the FP8 cache on the 7B batch (codes
bit-exact on every token of the sampled sequences, decode within 2e-3 of
the oracle on the stored values) and the multi-token kernel on the 7B batch
with 5 new tokens per sequence and on the long-context batch with 4, on
sampled sequences."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from oracle import fp8

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}
SCALE = 6.0 / 448.0


def pkv():
    import paged_kv_cache_365_b200 as m
    return m


def to_dev(a, dt):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dt == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.cuda()


def test_fp8_cache_full_size_7b():
    m = pkv()
    from paged_kv_cache_365_b200.replay import build_step
    wl = workloads.named("llama7b", 0)
    vals = workloads.draw_values(wl)
    ref = oracle.replay(wl, vals)
    st = build_step(wl, vals, "cuda")
    c = st["cache"]
    m.copy_blocks(c.k, c.v, st["cow_pairs"])
    m.kv_append(st["k_new"], st["v_new"], c.k, c.v, st["slot_mapping"])
    # the whole pool quantised on the device, token rows through the FP8 append
    NB, Hkv, _, D = c.k.shape
    k8 = torch.empty(c.k.shape, dtype=torch.uint8, device="cuda")
    v8 = torch.empty(c.v.shape, dtype=torch.uint8, device="cuda")
    slots = torch.arange(NB * 16, dtype=torch.int64, device="cuda")
    for src, dst in ((c.k, k8), (c.v, v8)):
        rows = src.permute(0, 2, 1, 3).reshape(NB * 16, Hkv, D).contiguous()
        m.kv_append_fp8(rows, rows, dst, dst, slots, SCALE, SCALE)
        del rows
    torch.cuda.synchronize()
    assert m.get_error() == 0
    rng = np.random.default_rng(5)
    seqs = sorted(set(rng.choice(wl.B, size=8, replace=False).tolist()) | {int(np.argmax(wl.context_lens))})
    tables, lens = ref["block_tables"], ref["context_lens"]
    # the oracle's codes of the sampled sequences' blocks
    blocks = np.unique(np.concatenate([tables[b, :-(-int(lens[b]) // 16)] for b in seqs]))
    ok = np.full(c.k.shape, fp8.NAN_CODE, dtype=np.uint8)
    ov = np.full(c.v.shape, fp8.NAN_CODE, dtype=np.uint8)
    ok[blocks] = fp8.quantize(oracle.widen(ref["cache"].k[blocks], wl.dtype).astype(np.float32), SCALE)
    ov[blocks] = fp8.quantize(oracle.widen(ref["cache"].v[blocks], wl.dtype).astype(np.float32), SCALE)
    gk, gv = k8.cpu().numpy(), v8.cpu().numpy()
    for b in seqs:  # every written token of the sampled sequences, bit for bit
        n = int(lens[b])
        tok = np.arange(n)
        blk, off = tables[b, tok // 16], tok % 16
        assert np.array_equal(gk[blk, :, off], ok[blk, :, off])
        assert np.array_equal(gv[blk, :, off], ov[blk, :, off])
    out = m.paged_attention_decode_fp8(st["q"], k8, v8, st["block_tables"], st["context_lens"], st["max_context_len"],
                                       wl.scale, SCALE, SCALE)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    want = oracle.paged_decode(vals["q"], ok, ov, tables, lens, wl.scale, wl.dtype, seqs=seqs, kv_dtype="e4m3",
                               k_scale=SCALE, v_scale=SCALE)
    got = out.float().cpu().numpy().astype(np.float64)
    assert np.abs(got[seqs] - want[seqs]).max() <= TOL[wl.dtype]


@pytest.mark.parametrize("name,n_new", [("llama7b", 5), ("long", 4)])
def test_multi_token_full_size(name, n_new):
    """The bench's multi-token step: n_new new tokens appended to every
    sequence of the workload (values drawn on the host here), then all of
    them attend causally; sampled sequences against the oracle."""
    m = pkv()
    wl = workloads.named(name, 0)
    vals = workloads.draw_values(wl)
    # the op log without the step (its last append is the step's), then
    # n_new new tokens per sequence through the library's allocator and the
    # oracle's, checked equal
    ref_alloc = oracle.RefAllocator(wl.num_blocks, wl.free_order)
    ref_cache = oracle.RefCache(wl.num_blocks, wl.Hkv, wl.D, wl.dtype)
    from paged_kv_cache_365_b200.replay import replay_ops, to_torch
    cache = m.PagedKVCache(wl.num_blocks, wl.Hkv, wl.D, {"f16": torch.float16, "bf16": torch.bfloat16}[wl.dtype],
                           "cuda", wl.free_order)
    replay_ops(cache, wl.ops, to_torch(vals["k_tokens"], wl.dtype, "cuda"), to_torch(vals["v_tokens"], wl.dtype,
                                                                                     "cuda"))
    cursor = 0
    for op in wl.ops:
        if op[0] == "add":
            ref_alloc.add_seq(op[1])
        elif op[0] == "fork":
            ref_alloc.fork(op[1], op[2])
        elif op[0] == "free":
            ref_alloc.free_seq(op[1])
        else:
            s_, c_ = ref_alloc.append_tokens(op[1], op[2])
            ref_cache.copy_blocks(c_)
            ref_cache.append_many(vals["k_tokens"][cursor:cursor + op[2]], vals["v_tokens"][cursor:cursor + op[2]],
                                  np.array(s_))
            cursor += op[2]
    ids = [int(s) for s in wl.step_seqs]
    slots, pairs, qs, tables, lens = cache.plan_multi_step(ids, [n_new] * len(ids))
    r_slots, r_pairs = [], []
    for sid in ids:
        s_, c_ = ref_alloc.append_tokens(sid, n_new)
        r_slots += s_
        r_pairs += c_
    assert list(slots) == r_slots and [tuple(p) for p in pairs] == r_pairs
    T = int(qs[-1])
    rng = np.random.default_rng(11)
    draw = lambda *shape: workloads._to_storage(rng.standard_normal(shape).astype(np.float32), wl.dtype)  # noqa
    q, kn, vn = draw(T, wl.Hq, wl.D), draw(T, wl.Hkv, wl.D), draw(T, wl.Hkv, wl.D)
    ref_cache.copy_blocks(r_pairs)
    ref_cache.append_many(kn, vn, np.array(r_slots))
    out = cache.run_multi_step(torch.from_numpy(slots), torch.from_numpy(pairs), torch.from_numpy(tables),
                               torch.from_numpy(lens), int(lens.max()), torch.from_numpy(qs), n_new,
                               to_dev(q, wl.dtype), to_dev(kn, wl.dtype), to_dev(vn, wl.dtype), scale=wl.scale)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    seqs = sorted(set(rng.choice(wl.B, size=min(wl.B, 4), replace=False).tolist()))
    want = oracle.paged_multi(q, ref_cache.k, ref_cache.v, tables, lens, qs, wl.scale, wl.dtype, seqs=seqs)
    rows = np.concatenate([np.arange(qs[b], qs[b + 1]) for b in seqs])
    got = out.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(got[rows]).all()
    assert np.abs(got[rows] - want[rows]).max() <= TOL[wl.dtype]
