"""GPU parity of multi-token paged attention (several query tokens per
sequence, causal over the paged context) against the fp64 oracle on the
same seeded inputs: max-abs error within 2e-3 (fp16) / 1e-2 (bf16).
Unwritten slots hold NaN and tables are padded with out-of-range ids, so a
read outside a row's visible tokens shows up."""
import numpy as np
import pytest
import torch

import oracle
from helpers import make_multi_case, ulp_aware_bound

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}
TORCH = {"f16": torch.float16, "bf16": torch.bfloat16}


def pkv():
    import paged_kv_cache_365_b200 as m
    return m


def to_dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.cuda()


def run_gpu(c, scale, partition=0, max_q=None):
    m = pkv()
    dt = c["dtype"]
    q, k, v = to_dev(c["q"], dt), to_dev(c["k"], dt), to_dev(c["v"], dt)
    nq = np.diff(c["qs"])
    out = m.paged_attention_multi(q, k, v, torch.from_numpy(c["tables"]).cuda(), torch.from_numpy(c["ctx"]).cuda(),
                                  torch.from_numpy(c["qs"]).cuda(), int(c["ctx"].max()),
                                  int(nq.max()) if max_q is None else max_q, scale, partition=partition)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), m.get_error()


CASES = [
    # ctx, nq, Hq, Hkv, D, dtype
    ([5, 16, 17, 40, 1], [1, 4, 17, 8, 1], 4, 4, 128, "f16"),
    ([33, 20, 3, 64], [5, 20, 3, 16], 8, 2, 64, "bf16"),
    ([48, 7, 300], [16, 2, 9], 8, 1, 128, "f16"),
    ([100, 130, 520, 1100], [2, 3, 4, 5], 16, 4, 128, "bf16"),
    ([1030, 600], [40, 33], 2, 2, 64, "f16"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[5]}_G{c[2] // c[3]}_D{c[4]}")
@pytest.mark.parametrize("partition", [0, 16, 64])
def test_multi_matches_oracle(case, partition):
    ctx, nq, Hq, Hkv, D, dt = case
    c = make_multi_case(ctx, nq, Hq, Hkv, D, dt, seed=sum(ctx) + partition)
    scale = D ** -0.5
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], scale, dt)
    got, err = run_gpu(c, scale, partition)
    assert err == 0
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL[dt]


@pytest.mark.parametrize("case", [
    ([700, 1500, 90], [5, 5, 3], 32, 8, 128, "bf16"),   # 20 rows: 3 row warps
    ([1300, 260], [4, 6], 32, 4, 128, "f16"),           # 32 rows: 4 row warps
    ([2100, 40], [3, 2], 16, 2, 64, "f16"),             # 24 rows, D = 64
], ids=lambda c: f"{c[5]}_G{c[2] // c[3]}_D{c[4]}")
@pytest.mark.parametrize("scale", [0.5, 3.0])
def test_row_split_kernel_wide_logits(case, scale):
    """Logits spread over tens of log2 units (the running max jumps by
    large and small steps, the attention is sharply peaked) through the
    kernel whose warps split the rows; the auto partition and 64 tokens.
    Peaked attention returns single V rows, so V is drawn N(0, 1/4): its
    values stay below 4, where the output dtype's own rounding (half an
    ulp: 2^-8 in bf16 on [2, 4), 2^-6 on [4, 8)) fits the bound."""
    ctx, nq, Hq, Hkv, D, dt = case
    c = make_multi_case(ctx, nq, Hq, Hkv, D, dt, seed=sum(ctx) + int(10 * scale), v_scale=0.5)
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], scale, dt)
    for partition in (0, 64):
        got, err = run_gpu(c, scale, partition)
        assert err == 0
        assert np.isfinite(got).all()
        assert np.abs(got - want).max() <= TOL[dt]


def test_one_token_per_sequence_agrees_with_decode():
    m = pkv()
    c = make_multi_case([9, 16, 50, 700, 2100], [1] * 5, 8, 2, 128, "bf16", seed=3)
    scale = 128 ** -0.5
    got, err = run_gpu(c, scale)
    dec = m.paged_attention_decode(to_dev(c["q"], "bf16"), to_dev(c["k"], "bf16"), to_dev(c["v"], "bf16"),
                                   torch.from_numpy(c["tables"]).cuda(), torch.from_numpy(c["ctx"]).cuda(),
                                   int(c["ctx"].max()), scale)
    assert err == 0
    assert np.abs(got - dec.float().cpu().numpy()).max() <= TOL["bf16"]


def test_speculative_verify_shape_sampled():
    """64 sequences of a 7B shape (32 heads, D 128, fp16), contexts up to
    2048, 4 draft tokens + 1 verified each; every 8th sequence checked."""
    rng = np.random.default_rng(21)
    ctx = [int(x) for x in rng.integers(128, 2049, 64)]
    c = make_multi_case(ctx, [5] * 64, 32, 32, 128, "f16", seed=22)
    scale = 128 ** -0.5
    got, err = run_gpu(c, scale)
    assert err == 0
    seqs = list(range(0, 64, 8))
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], scale, "f16", seqs=seqs)
    rows = np.concatenate([np.arange(c["qs"][b], c["qs"][b + 1]) for b in seqs])
    assert np.abs(got[rows] - want[rows]).max() <= TOL["f16"]


def test_prefill_chunk_sampled():
    """A 512-token prefill chunk at the end of a 2000-token context (GQA 4,
    bf16): every row against the oracle."""
    c = make_multi_case([2000, 700], [512, 300], 8, 2, 128, "bf16", seed=31)
    scale = 128 ** -0.5
    got, err = run_gpu(c, scale)
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], scale, "bf16")
    assert err == 0
    assert np.abs(got - want).max() <= TOL["bf16"]


def test_edge_rows_and_flags():
    m = pkv()
    # more new tokens than context: the first rows are zeros, flagged
    c = make_multi_case([3, 20], [5, 4], 4, 2, 64, "f16", seed=5)
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], 0.125, "f16")
    got, err = run_gpu(c, 0.125)
    assert err == m.ERR_CONTEXT_RANGE
    assert np.abs(got - want).max() <= TOL["f16"]
    # a sequence with no new token, and max_query_len smaller than a
    # sequence's tokens: that sequence is skipped and flagged
    c = make_multi_case([40, 30, 50], [3, 0, 6], 4, 4, 64, "f16", seed=6)
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], 0.125, "f16")
    got, err = run_gpu(c, 0.125)
    assert err == 0 and np.abs(got - want).max() <= TOL["f16"]
    got, err = run_gpu(c, 0.125, max_q=4)
    assert err == m.ERR_CONTEXT_RANGE
    assert np.abs(got[:3] - want[:3]).max() <= TOL["f16"]


@pytest.mark.parametrize("case", [
    ([70, 600, 37], [37, 20, 37], 4, 4, 128, "f16"),    # 37 rows: one 64-row tile, 27 padded
    ([900, 300], [20, 11], 16, 2, 64, "bf16"),          # 160 rows: three tiles, the last partial
    ([2500, 130, 16], [100, 64, 16], 8, 8, 128, "bf16"),  # long chunks, whole contexts of new tokens
], ids=lambda c: f"{c[5]}_G{c[2] // c[3]}_D{c[4]}_rows{max(c[1]) * c[2] // c[3]}")
@pytest.mark.parametrize("partition", [0, 64, 2048])
def test_rows_as_m_kernel(case, partition):
    """More than 32 rows per kv-head go to the kernel with the rows as the
    MMA's M dimension (16 per warp, 64 per tile): tiles that start mid-
    sequence, padded rows, chunks whose causal diagonal crosses pages and
    partitions, sequences made only of new tokens."""
    ctx, nq, Hq, Hkv, D, dt = case
    c = make_multi_case(ctx, nq, Hq, Hkv, D, dt, seed=sum(ctx) + partition)
    scale = D ** -0.5
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], scale, dt)
    got, err = run_gpu(c, scale, partition)
    assert err == 0
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL[dt]


def test_rows_as_m_kernel_flags_rows_before_the_context():
    m = pkv()
    # 40 new tokens against a 30-token context: the first 10 rows of each
    # head are zeros and flagged
    c = make_multi_case([30, 200], [40, 40], 4, 4, 64, "f16", seed=9)
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], 0.125, "f16")
    got, err = run_gpu(c, 0.125)
    assert err == m.ERR_CONTEXT_RANGE
    assert np.abs(got - want).max() <= TOL["f16"]


def test_multi_step_through_the_cache_api():
    """PagedKVCache.plan_multi_step + run_multi_step (host inputs, one of
    them forcing a copy-on-write) against the oracle allocator, cache and
    attention: slots, pairs and the pool bit-exact, output within 2e-3."""
    m = pkv()
    rng = np.random.default_rng(41)
    Hq, Hkv, D, nb = 8, 4, 128, 48
    order = rng.permutation(nb).astype(np.int32)
    cache = m.PagedKVCache(nb, Hkv, D, torch.float16, free_order=order)
    ref = oracle.RefAllocator(nb, order)
    dev = oracle.RefCache(nb, Hkv, D, "f16")

    def write(sid, n):
        vals = rng.standard_normal((2, n, Hkv, D)).astype(np.float16)
        slots, cows = ref.append_tokens(sid, n)
        dev.copy_blocks(cows)
        dev.append(vals[0], vals[1], np.array(slots))
        cache.prefill(sid, torch.from_numpy(vals[0]), torch.from_numpy(vals[1]))

    for sid, n in ((0, 70), (1, 16), (2, 200)):
        ref.add_seq(sid)
        cache.add_seq(sid)
        write(sid, n)
    ref.fork(0, 3)
    cache.fork(0, 3)  # shares a partial last block: the step copies it
    ids, n_new = [0, 1, 2, 3], [5, 3, 8, 4]
    slots, pairs, qs, tables, lens = cache.plan_multi_step(ids, n_new)
    r_slots, r_pairs = [], []
    for sid, n in zip(ids, n_new):
        s_, p_ = ref.append_tokens(sid, n)
        r_slots += s_
        r_pairs += p_
    assert list(slots) == r_slots and [tuple(p) for p in pairs] == r_pairs
    T = int(qs[-1])
    q = rng.standard_normal((T, Hq, D)).astype(np.float16)
    kn = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    vn = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    dev.copy_blocks(r_pairs)
    dev.append(kn, vn, np.array(r_slots))
    out = torch.empty((T, Hq, D), dtype=torch.float16, pin_memory=True)
    cache.run_multi_step(torch.from_numpy(slots).pin_memory(), torch.from_numpy(pairs).pin_memory(),
                         torch.from_numpy(tables).pin_memory(), torch.from_numpy(lens).pin_memory(),
                         int(lens.max()), torch.from_numpy(qs).pin_memory(), max(n_new),
                         torch.from_numpy(q).pin_memory(), torch.from_numpy(kn).pin_memory(),
                         torch.from_numpy(vn).pin_memory(), out=out)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    held = sorted({b for t in ref.tables.values() for b in t})
    assert np.array_equal(cache.k.cpu().view(torch.int16).numpy()[held], dev.k.view(np.int16)[held])
    assert np.array_equal(cache.v.cpu().view(torch.int16).numpy()[held], dev.v.view(np.int16)[held])
    want = oracle.paged_multi(q, dev.k, dev.v, tables, lens, qs, D ** -0.5, "f16")
    assert np.abs(out.float().numpy() - want).max() <= TOL["f16"]


@pytest.mark.parametrize("case", [
    ([700, 1500, 90], [5, 5, 3], 32, 8, 128, "bf16"),     # 20 rows: row-split kernel
    ([1300, 260], [4, 6], 32, 4, 128, "f16"),             # 24 rows
    ([900, 300], [20, 11], 16, 2, 64, "bf16"),            # 160 rows: 128-row tiles
    ([2500, 130], [100, 64], 8, 8, 128, "f16"),           # 100 rows
], ids=lambda c: f"{c[5]}_G{c[2] // c[3]}_D{c[4]}_rows{max(c[1]) * c[2] // c[3]}")
@pytest.mark.parametrize("scale", [None, 3.0])
def test_multi_wide_values(case, scale):
    """V drawn N(0, 4): peaked attention returns values up to ~8, where the
    16-bit formats' own half-ulp passes the stated tolerance.  The bound is
    the stated tolerance, or that half-ulp of the oracle's value plus a
    2^-14 relative slack where it is larger."""
    ctx, nq, Hq, Hkv, D, dt = case
    c = make_multi_case(ctx, nq, Hq, Hkv, D, dt, seed=sum(ctx) + 13, v_scale=2.0)
    sc = D ** -0.5 if scale is None else scale
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], sc, dt)
    for partition in (0, 64):
        got, err = run_gpu(c, sc, partition)
        assert err == 0
        assert np.isfinite(got).all()
        assert (np.abs(got - want) <= ulp_aware_bound(want, dt, TOL[dt])).all()
    if scale is not None:
        assert np.abs(want).max() > 4.0


def test_tcgen05_kernel_huge_logits():
    """Scores far past 2^20 in log2 units (q scaled by 1e4, logit scale
    1e3) on the tcgen05 kernel (160 rows per kv-head): the attention is
    one-hot on each row's best key, and the output must be that V row,
    finite, within the stated tolerance."""
    ctx, nq, Hq, Hkv, D, dt = [900, 300], [40, 11], 8, 2, 128, "bf16"
    c = make_multi_case(ctx, nq, Hq, Hkv, D, dt, seed=12)
    import workloads
    q = oracle.widen(c["q"], dt) * 1e4
    c["q"] = workloads._to_storage(q.astype(np.float32), dt)
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], 1e3, dt)
    got, err = run_gpu(c, 1e3)
    assert err == 0
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL[dt]


@pytest.mark.parametrize("partition", [0, 32])
def test_tcgen05_scheduler_many_items(partition):
    """Far more work items than CTAs for the persistent tcgen05 kernel: 200
    sequences with random lengths (some empty, some shorter than their new
    tokens, whose first rows are zeros and flagged) and 0..70 new tokens each
    (G = 2: up to 140 rows, two 128-row tiles), with the auto partition and
    with 32-token partitions (thousands of items, most sequences split and
    merged). Every row against the oracle."""
    m = pkv()
    rng = np.random.default_rng(31 + partition)
    B = 200
    nq = rng.integers(0, 71, size=B)
    nq[:3] = 70  # at least one sequence with more than 32 rows per kv-head
    ctx = np.maximum(nq + rng.integers(-5, 180, size=B), 0)
    ctx[5] = 0
    c = make_multi_case(list(ctx), list(nq), 4, 2, 64, "bf16", seed=77 + partition)
    want = oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], 0.125, "bf16")
    got, err = run_gpu(c, 0.125, partition)
    assert err in (0, m.ERR_CONTEXT_RANGE)
    assert (err != 0) == bool(np.any(nq > ctx))
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL["bf16"]
