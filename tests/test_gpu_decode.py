"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.

Bit-exact: the step's plan (slots, copy pairs, tables, lengths) and the
cache contents after the copy-on-write copy and the append.  Attention:
max-abs error against the fp64 oracle within 2e-3 (fp16), 1e-2 (bf16),
1e-5 (fp32).  The unwritten slots of every pool hold NaN and every table
is padded with out-of-range ids, so a read outside a sequence's tokens
shows up as a NaN or an error flag.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2, "f32": 1e-5}


def pkv():
    import paged_kv_cache_365_b200 as m
    return m


def run_gpu_step(wl, vals, partition=0):
    """Replay, then one step on the device: copy, append, decode."""
    from paged_kv_cache_365_b200.replay import build_step
    m = pkv()
    st = build_step(wl, vals, "cuda")
    c = st["cache"]
    m.copy_blocks(c.k, c.v, st["cow_pairs"])
    m.kv_append(st["k_new"], st["v_new"], c.k, c.v, st["slot_mapping"])
    out = m.paged_attention_decode(st["q"], c.k, c.v, st["block_tables"], st["context_lens"],
                                   st["max_context_len"], wl.scale, partition=partition)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    return out, st


def to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def storage_bits(t):
    """Device tensor -> numpy array of its raw storage (for bitwise checks)."""
    if t.dtype == torch.float32:
        return t.cpu().view(torch.int32).numpy()
    return t.cpu().view(torch.int16).numpy()


def oracle_bits(a):
    return a.view(np.int32) if a.dtype == np.float32 else a.view(np.int16)


_CACHE = {}


def oracle_state(wl):
    key = (wl.name, wl.seed, wl.B, wl.Hq, wl.D, wl.dtype)
    if key not in _CACHE:
        vals = workloads.draw_values(wl)
        _CACHE.clear()
        _CACHE[key] = (vals, oracle.replay(wl, vals))
    return _CACHE[key]


def check_plan(st, ref):
    h = st["host"]
    assert np.array_equal(h["step_slots"], ref["step_slots"])
    assert np.array_equal(np.asarray(h["cow_pairs"]).reshape(-1, 2), ref["cow_pairs"])
    assert np.array_equal(h["context_lens"], ref["context_lens"])
    for b, n in enumerate(ref["context_lens"]):
        pages = -(-int(n) // 16)
        assert np.array_equal(h["block_tables"][b, :pages], ref["block_tables"][b, :pages])


SMALL = [
    workloads.tiny(0),
    workloads.custom([1, 15, 16, 17, 200, 511, 512, 513, 1300], Hq=32, Hkv=8, D=128, dtype="bf16", seed=1,
                     name="gqa4_bf16_d128"),
    workloads.custom([3, 40, 700, 1025], Hq=8, Hkv=8, D=128, dtype="f16", seed=2, name="mha_f16_d128"),
    workloads.custom([5, 33, 600], Hq=16, Hkv=2, D=64, dtype="f16", seed=3, name="gqa8_f16_d64"),
    workloads.custom([2, 100, 520], Hq=4, Hkv=2, D=64, dtype="bf16", seed=4, name="gqa2_bf16_d64"),
    workloads.custom([7, 129, 1100], Hq=16, Hkv=2, D=128, dtype="f32", seed=5, name="gqa8_f32_d128"),
    workloads.custom([9, 530], Hq=4, Hkv=1, D=64, dtype="f32", seed=6, name="gqa4_f32_d64"),
    workloads.custom([0, 1, 17, 0, 64], Hq=8, Hkv=4, D=128, dtype="f16", seed=7, name="with_empty"),
    workloads.prefix13b(seed=8, B=12, prefix_tokens=256, suffix_range=(1, 100), Hq=8, Hkv=8, D=128,
                        dtype="f16", name="prefix_small"),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_step_parity(wl):
    vals, ref = oracle_state(wl)
    out, st = run_gpu_step(wl, vals)
    check_plan(st, ref)
    # the whole pool after copy + append, bit for bit (NaN where unwritten)
    c = st["cache"]
    assert np.array_equal(storage_bits(c.k), oracle_bits(ref["cache"].k))
    assert np.array_equal(storage_bits(c.v), oracle_bits(ref["cache"].v))
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"],
                               ref["context_lens"], wl.scale, wl.dtype)
    got = to_f64(out)
    assert np.isfinite(got).all()
    err = np.abs(got - want).max()
    assert err <= TOL[wl.dtype], err


@pytest.mark.parametrize("partition", [16, 32, 48, 256, 2048])
def test_partition_sizes_agree_with_oracle(partition):
    wl = SMALL[1]
    vals, ref = oracle_state(wl)
    out, _ = run_gpu_step(wl, vals, partition=partition)
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"],
                               ref["context_lens"], wl.scale, wl.dtype)
    assert np.abs(to_f64(out) - want).max() <= TOL[wl.dtype]


@pytest.mark.parametrize("wl", [SMALL[1], SMALL[3], SMALL[5]], ids=lambda w: w.name)
def test_block_relabelling_is_bit_identical_on_gpu(wl):
    m = pkv()
    vals, _ = oracle_state(wl)
    out, st = run_gpu_step(wl, vals)
    c = st["cache"]
    perm = torch.from_numpy(np.random.default_rng(5).permutation(wl.num_blocks)).cuda()
    k2 = torch.empty_like(c.k)
    v2 = torch.empty_like(c.v)
    k2[perm] = c.k
    v2[perm] = c.v
    bt = st["block_tables"].clone().long()
    valid = bt < wl.num_blocks
    bt[valid] = perm[bt[valid]]
    out2 = m.paged_attention_decode(st["q"], k2, v2, bt.int().contiguous(), st["context_lens"],
                                    st["max_context_len"], wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_shared_prefix_equals_private_copy_on_gpu():
    m = pkv()
    wl = SMALL[8]
    vals, _ = oracle_state(wl)
    out, st = run_gpu_step(wl, vals)
    c = st["cache"]
    bt = st["host"]["block_tables"]
    lens = st["host"]["context_lens"]
    pages = [-(-int(n) // 16) for n in lens]
    total = wl.num_blocks + sum(pages)
    k2 = torch.full((total,) + tuple(c.k.shape[1:]), float("nan"), dtype=c.k.dtype, device="cuda")
    v2 = torch.full_like(k2, float("nan"))
    k2[:wl.num_blocks] = c.k
    v2[:wl.num_blocks] = c.v
    bt2 = bt.copy()
    nxt = wl.num_blocks
    src, dst = [], []
    for b, p in enumerate(pages):
        for j in range(p):
            src.append(int(bt[b, j]))
            dst.append(nxt)
            bt2[b, j] = nxt
            nxt += 1
    # the private copies are made with the library's own block copy
    pairs = torch.tensor(np.stack([src, dst], axis=1), dtype=torch.int32, device="cuda")
    m.copy_blocks(k2, v2, pairs)
    out2 = m.paged_attention_decode(st["q"], k2, v2, torch.from_numpy(bt2).cuda(), st["context_lens"],
                                    st["max_context_len"], wl.scale)
    torch.cuda.synchronize()
    assert len(set(bt[:, 0].tolist())) == 1  # really shared before
    assert torch.equal(out, out2)


FULL = ["llama7b", "gqa8b", "prefix13b", "long"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_parity_on_sampled_sequences(name):
    """Named workloads at full size, default launch configuration: the plan,
    the slots the step wrote and the blocks it copied, bit for bit; the
    decode output of a sample of sequences against the oracle."""
    wl = workloads.named(name, 0)
    vals, ref = oracle_state(wl)
    out, st = run_gpu_step(wl, vals)
    check_plan(st, ref)
    c = st["cache"]
    slots = ref["step_slots"][ref["step_slots"] >= 0]
    blk = torch.from_numpy(slots // 16).cuda()
    off = torch.from_numpy(slots % 16).cuda()
    assert np.array_equal(storage_bits(c.k[blk, :, off]), oracle_bits(ref["cache"].k[slots // 16, :, slots % 16]))
    assert np.array_equal(storage_bits(c.v[blk, :, off]), oracle_bits(ref["cache"].v[slots // 16, :, slots % 16]))
    if len(ref["cow_pairs"]):
        dst = ref["cow_pairs"][:, 1]
        d = torch.from_numpy(dst.astype(np.int64)).cuda()
        assert np.array_equal(storage_bits(c.k[d]), oracle_bits(ref["cache"].k[dst]))
        assert np.array_equal(storage_bits(c.v[d]), oracle_bits(ref["cache"].v[dst]))
    rng = np.random.default_rng(17)
    n_sample = min(wl.B, 6 if name == "long" else 12)
    seqs = sorted(set(rng.choice(wl.B, size=n_sample, replace=False).tolist())
                  | {int(np.argmax(wl.context_lens)), int(np.argmin(wl.context_lens))})
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"],
                               ref["context_lens"], wl.scale, wl.dtype, seqs=seqs)
    got = to_f64(out)
    assert np.isfinite(got).all()
    err = np.abs(got[seqs] - want[seqs]).max()
    assert err <= TOL[wl.dtype], err


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 8])
def test_edge_lengths(dtype, D, G):
    wl = workloads.custom([0, 1, 15, 16, 17, 511, 512, 513, 1024, 1025], Hq=2 * G, Hkv=2, D=D, dtype=dtype,
                          seed=10 + D + G, name=f"edges_{dtype}_{D}_{G}")
    vals, ref = oracle_state(wl)
    out, _ = run_gpu_step(wl, vals)
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"],
                               ref["context_lens"], wl.scale, wl.dtype)
    got = to_f64(out)
    assert np.array_equal(got[0], np.zeros_like(got[0]))            # ctx 0 -> zeros
    assert np.array_equal(got[1], oracle.widen(vals["v_new"][1], dtype)[np.arange(2 * G) // G])  # ctx 1 -> v
    assert np.abs(got - want).max() <= TOL[dtype]


def test_append_bit_exact_and_negative_slots_skip():
    m = pkv()
    nb, hkv, D = 8, 3, 64
    for dt, tdt in (("f16", torch.float16), ("bf16", torch.bfloat16), ("f32", torch.float32)):
        k = torch.full((nb, hkv, 16, D), float("nan"), dtype=tdt, device="cuda")
        v = torch.full_like(k, float("nan"))
        rng = np.random.default_rng(0)
        slots = np.array([5, -1, 127, 16, -7, 64], dtype=np.int64)
        kn = torch.randn(len(slots), hkv, D, generator=torch.Generator().manual_seed(1)).to(tdt)
        vn = torch.randn(len(slots), hkv, D, generator=torch.Generator().manual_seed(2)).to(tdt)
        m.kv_append(kn.cuda(), vn.cuda(), k, v, torch.from_numpy(slots).cuda())
        ref = oracle.RefCache(nb, hkv, D, dt)
        kn_np = kn.view(torch.int16).numpy().view(np.uint16) if dt == "bf16" else kn.numpy()
        vn_np = vn.view(torch.int16).numpy().view(np.uint16) if dt == "bf16" else vn.numpy()
        ref.append(kn_np, vn_np, slots)
        assert np.array_equal(storage_bits(k), oracle_bits(ref.k))
        assert np.array_equal(storage_bits(v), oracle_bits(ref.v))
        del rng
    assert m.get_error() == 0


def test_device_range_checks_raise_flags_without_faulting():
    m = pkv()
    m.get_error()  # clear
    wl = SMALL[2]
    vals, _ = oracle_state(wl)
    out, st = run_gpu_step(wl, vals)
    c = st["cache"]
    # a table entry inside a sequence's pages out of range
    bt = st["block_tables"].clone()
    bt[2, 3] = wl.num_blocks + 5
    m.paged_attention_decode(st["q"], c.k, c.v, bt, st["context_lens"], st["max_context_len"], wl.scale)
    assert m.get_error() & m.ERR_BLOCK_RANGE
    bt[2, 3] = -3
    m.paged_attention_decode(st["q"], c.k, c.v, bt, st["context_lens"], st["max_context_len"], wl.scale)
    assert m.get_error() & m.ERR_BLOCK_RANGE
    # a context length above the bound the host passed
    cl = st["context_lens"].clone()
    cl[1] = st["max_context_len"] + 100
    m.paged_attention_decode(st["q"], c.k, c.v, st["block_tables"], cl, st["max_context_len"], wl.scale)
    assert m.get_error() & m.ERR_CONTEXT_RANGE
    # an append slot beyond the pool, and a copy pair beyond the pool
    bad_slot = torch.tensor([wl.num_blocks * 16 + 3], dtype=torch.int64, device="cuda")
    m.kv_append(st["k_new"][:1].contiguous(), st["v_new"][:1].contiguous(), c.k, c.v, bad_slot)
    assert m.get_error() & m.ERR_SLOT_RANGE
    m.copy_blocks(c.k, c.v, torch.tensor([[0, wl.num_blocks]], dtype=torch.int32, device="cuda"))
    assert m.get_error() & m.ERR_COPY_RANGE
    assert m.get_error() == 0


def test_workspace_contents_and_graph_replays_do_not_matter():
    """A split-K decode with a workspace full of garbage, or one reused by a
    replayed CUDA graph, gives the same bits as with a fresh zeroed one, with
    no error flag."""
    m = pkv()
    wl = workloads.custom([3000, 1700, 40, 2049], Hq=8, Hkv=2, D=128, dtype="f16", seed=77, name="fold")
    vals = workloads.draw_values(wl)
    from paged_kv_cache_365_b200.replay import build_step
    st = build_step(wl, vals, "cuda")
    c = st["cache"]
    m.copy_blocks(c.k, c.v, st["cow_pairs"])
    m.kv_append(st["k_new"], st["v_new"], c.k, c.v, st["slot_mapping"])
    args = (st["q"], c.k, c.v, st["block_tables"], st["context_lens"], st["max_context_len"], wl.scale)
    need = m.decode_workspace_bytes(wl.B, wl.Hq, wl.D, st["max_context_len"])
    assert need > 0
    clean = m.paged_attention_decode(*args, workspace=torch.zeros(need, dtype=torch.uint8, device="cuda"))
    garbage = torch.randint(0, 256, (need,), dtype=torch.uint8, device="cuda")
    dirty = m.paged_attention_decode(*args, workspace=garbage)
    again = m.paged_attention_decode(*args, workspace=garbage)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    assert torch.equal(clean.view(torch.int16), dirty.view(torch.int16))
    assert torch.equal(clean.view(torch.int16), again.view(torch.int16))
    # a captured call replayed: the same epoch every replay
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(st["q"])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        m.paged_attention_decode(*args, out=out, workspace=ws)  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        m.paged_attention_decode(*args, out=out, workspace=ws)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(clean.view(torch.int16), out.view(torch.int16))
    assert m.get_error() == 0
    ref = oracle.replay(wl, vals)
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"], ref["context_lens"],
                               wl.scale, wl.dtype)
    assert np.abs(clean.float().cpu().numpy() - want).max() <= TOL["f16"]


def _ramp_values(wl, step):
    """Values whose scores climb along every sequence: q[..., 0] = 4 and
    k[token t, :, 0] = step * t / 16, the other entries N(0, 1), so that a
    later page's scores pass the first pages' maximum by many units and the
    kernels' reference max has to move (and O and l be rescaled) mid-sequence,
    in every partition."""
    vals = workloads.draw_values(wl)
    f = {k: oracle.widen(v, wl.dtype).astype(np.float32) for k, v in vals.items()}
    f["q"][:, :, 0] = 4.0
    r = 0
    for b, c in enumerate(wl.context_lens):
        n = max(int(c) - 1, 0)
        f["k_tokens"][r:r + n, :, 0] = (step * np.arange(n) / 16.0)[:, None]
        f["k_new"][b, :, 0] = step * max(int(c) - 1, 0) / 16.0
        r += n
    return {k: workloads._to_storage(v, wl.dtype) for k, v in f.items()}


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("partition", [0, 256])
def test_reference_max_moves_mid_sequence(dtype, G, partition):
    """Scores that climb page after page (and one sequence whose scores fall
    instead): the decode's reference max moves only when a page passes it by
    more than 2^8, rescaling what was accumulated; the result must still be
    the oracle's softmax within the stated tolerance."""
    wl = workloads.custom([700, 1500, 37, 2100], Hq=2 * G, Hkv=2, D=128, dtype=dtype, seed=31 + G,
                          name=f"ramp_{dtype}_{G}")
    vals = _ramp_values(wl, 3.0)
    # sequence 2 falls instead of climbing
    f = oracle.widen(vals["k_tokens"], dtype).astype(np.float32)
    r0 = sum(max(int(c) - 1, 0) for c in wl.context_lens[:2])
    n2 = int(wl.context_lens[2]) - 1
    f[r0:r0 + n2, :, 0] = f[r0:r0 + n2, :, 0][::-1]
    vals["k_tokens"] = workloads._to_storage(f, dtype)
    ref = oracle.replay(wl, vals)
    out, _ = run_gpu_step(wl, vals, partition=partition)
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"],
                               ref["context_lens"], wl.scale, wl.dtype)
    got = to_f64(out)
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL[dtype]
