"""GPU parity of the FP8 (E4M3) KV cache against the oracle: the quantising
append bit-exact (codes, every block of the pool), decode over the FP8
cache within the query dtype's tolerance (2e-3 fp16, 1e-2 bf16) of the fp64
oracle evaluated on the stored values (code value x scale).  Unwritten
slots hold the NaN code and tables are padded with out-of-range ids."""
import numpy as np
import pytest
import torch

import oracle
from helpers import ulp_aware_bound
from oracle import fp8

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}
TORCH = {"f16": torch.float16, "bf16": torch.bfloat16}


def pkv():
    import paged_kv_cache_365_b200 as m
    return m


def storage(x32, dt):
    """float32 draws -> storage array of dt (bf16 as uint16 bits, RNE)."""
    if dt == "f16":
        return x32.astype(np.float16)
    import workloads
    return workloads._to_storage(x32, "bf16")


def to_dev(a, dt):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dt == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.cuda()


def build(ctx, Hkv, D, dt, ks, vs, seed, sigma=1.0, ramp=0.0):
    """An FP8 pool written through the GPU append and the oracle append from
    the same 16-bit values (N(0, sigma^2); with ``ramp``, K's first entry of
    token j of every sequence is ramp * j / 16 instead); returns both plus
    tables."""
    m = pkv()
    rng = np.random.default_rng(seed)
    pages = [-(-c // 16) for c in ctx]
    nb = sum(pages) + 4
    perm = rng.permutation(nb)
    W = max(pages) + 2
    tables = np.full((len(ctx), W), nb + 50, dtype=np.int32)
    slots = []
    used = 0
    for b, c in enumerate(ctx):
        tables[b, :pages[b]] = perm[used:used + pages[b]]
        used += pages[b]
        slots += [int(tables[b, j // 16]) * 16 + j % 16 for j in range(c)]
    slots = np.array(slots, dtype=np.int64)
    n = len(slots)
    k32 = rng.standard_normal((n, Hkv, D)).astype(np.float32) * sigma
    if ramp:
        k32[:, :, 0] = (ramp * np.concatenate([np.arange(c) for c in ctx]) / 16.0)[:, None]
    kx = storage(k32, dt)
    vx = storage(rng.standard_normal((n, Hkv, D)).astype(np.float32) * sigma, dt)
    ref = oracle.RefCache(nb, Hkv, D, "e4m3")
    ref.append_fp8(kx, vx, slots, dt, ks, vs)
    kc = torch.full((nb, Hkv, 16, D), 0x7F, dtype=torch.uint8, device="cuda")
    vc = torch.full((nb, Hkv, 16, D), 0x7F, dtype=torch.uint8, device="cuda")
    m.kv_append_fp8(to_dev(kx, dt), to_dev(vx, dt), kc, vc, torch.from_numpy(slots).cuda(), ks, vs)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    return ref, kc, vc, tables, np.array(ctx, dtype=np.int32)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
def test_append_codes_bit_exact(dt, D):
    ref, kc, vc, _, _ = build([37, 16, 100, 1], 4, D, dt, 0.013, 0.021, seed=D)
    assert np.array_equal(kc.cpu().numpy(), ref.k)
    assert np.array_equal(vc.cpu().numpy(), ref.v)


def test_append_saturates_and_keeps_signs():
    m = pkv()
    vals = np.array([500.0, -500.0, 448.0, 1e-4, -0.0, 3.0 * 2 ** -10, 1.0625], dtype=np.float32)
    x = np.zeros((1, 1, 64), dtype=np.float16)
    x[0, 0, :len(vals)] = vals.astype(np.float16)
    kc = torch.zeros((2, 1, 16, 64), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    xt = torch.from_numpy(x).cuda()
    m.kv_append_fp8(xt, xt, kc, vc, torch.tensor([17], dtype=torch.int64, device="cuda"), 1.0, 1.0)
    torch.cuda.synchronize()
    got = kc[1, 0, 1, :len(vals)].cpu().numpy()
    want = fp8.quantize(x[0, 0, :len(vals)].astype(np.float32), 1.0)
    assert np.array_equal(got, want)
    assert list(got[:3]) == [0x7E, 0xFE, 0x7E] and got[4] == 0x80


CASES = [
    # ctx, Hq, Hkv, D, q dtype
    ([1, 15, 16, 17, 100], 4, 4, 128, "f16"),
    ([33, 700, 1100], 8, 2, 128, "bf16"),
    ([5, 48, 300, 2049], 8, 1, 64, "f16"),
    ([64, 129, 513], 16, 4, 64, "bf16"),
    ([17000, 300, 2100], 8, 1, 128, "bf16"),  # auto partition: 2048 tokens past 16384
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[4]}_G{c[1] // c[2]}_D{c[3]}")
@pytest.mark.parametrize("partition", [0, 16, 96])
def test_decode_fp8_matches_oracle(case, partition):
    m = pkv()
    ctx, Hq, Hkv, D, dt = case
    ks, vs = 0.011, 0.017
    ref, kc, vc, tables, lens = build(ctx, Hkv, D, dt, ks, vs, seed=len(ctx) + D)
    rng = np.random.default_rng(partition + D)
    q = storage(rng.standard_normal((len(ctx), Hq, D)).astype(np.float32), dt)
    scale = D ** -0.5
    want = oracle.paged_decode(q, ref.k, ref.v, tables, lens, scale, dt, kv_dtype="e4m3", k_scale=ks, v_scale=vs)
    out = m.paged_attention_decode_fp8(to_dev(q, dt), kc, vc, torch.from_numpy(tables).cuda(),
                                       torch.from_numpy(lens).cuda(), int(lens.max()), scale, ks, vs,
                                       partition=partition)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL[dt]


def test_decode_fp8_float8_dtype_and_zero_context():
    m = pkv()
    ref, kc, vc, tables, lens = build([20, 0, 3], 2, 64, "f16", 0.05, 0.05, seed=3)
    q = np.random.default_rng(1).standard_normal((3, 4, 64)).astype(np.float16)
    want = oracle.paged_decode(q, ref.k, ref.v, tables, lens, 0.125, "f16", kv_dtype="e4m3", k_scale=0.05,
                               v_scale=0.05)
    out = m.paged_attention_decode_fp8(torch.from_numpy(q).cuda(), kc.view(torch.float8_e4m3fn),
                                       vc.view(torch.float8_e4m3fn), torch.from_numpy(tables).cuda(),
                                       torch.from_numpy(lens).cuda(), 20, 0.125, 0.05, 0.05)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    got = out.float().cpu().numpy()
    assert np.array_equal(got[1], np.zeros_like(got[1]))
    assert np.abs(got - want).max() <= TOL["f16"]


def test_cache_with_fp8_pool_steps_like_the_oracle():
    """PagedKVCache with an FP8 pool: prefill and two decode steps (one with
    a copy-on-write) through the quantising append, host inputs staged; the
    pool's codes and the outputs against the oracle."""
    m = pkv()
    rng = np.random.default_rng(2)
    Hq, Hkv, D, nb, ks, vs = 8, 2, 128, 40, 0.013, 0.019
    order = rng.permutation(nb).astype(np.int32)
    cache = m.PagedKVCache(nb, Hkv, D, torch.bfloat16, free_order=order, fp8_scales=(ks, vs))
    ref = oracle.RefAllocator(nb, order)
    dev = oracle.RefCache(nb, Hkv, D, "e4m3")

    def vals(n):
        return (storage(rng.standard_normal((n, Hkv, D)).astype(np.float32), "bf16"),
                storage(rng.standard_normal((n, Hkv, D)).astype(np.float32), "bf16"))

    for sid, n in ((0, 50), (1, 7), (2, 130)):
        ref.add_seq(sid)
        cache.add_seq(sid)
        k, v = vals(n)
        slots, cows = ref.append_tokens(sid, n)
        dev.copy_blocks(cows)
        dev.append_fp8(k, v, np.array(slots), "bf16", ks, vs)
        cache.prefill(sid, to_dev(k, "bf16"), to_dev(v, "bf16"))
    ref.fork(0, 3)
    cache.fork(0, 3)
    ids = [0, 1, 2, 3]
    for _ in range(2):
        q = storage(rng.standard_normal((4, Hq, D)).astype(np.float32), "bf16")
        k, v = vals(4)
        slots, cows = ref.step(ids)
        dev.copy_blocks(cows)
        dev.append_fp8(k, v, np.array(slots), "bf16", ks, vs)
        out = cache.step(ids, to_dev(q, "bf16").cpu(), to_dev(k, "bf16").cpu(), to_dev(v, "bf16").cpu())
        torch.cuda.synchronize()
        assert m.get_error() == 0
        tables = np.array([ref.block_table(s)[0] + [nb + 3] * (20 - len(ref.block_table(s)[0])) for s in ids],
                          dtype=np.int32)
        lens = np.array([ref.block_table(s)[1] for s in ids], dtype=np.int32)
        want = oracle.paged_decode(q, dev.k, dev.v, tables, lens, D ** -0.5, "bf16", kv_dtype="e4m3", k_scale=ks,
                                   v_scale=vs)
        assert np.abs(out.float().numpy() - want).max() <= TOL["bf16"]
    held = sorted({b for t in ref.tables.values() for b in t})
    assert np.array_equal(cache.k.cpu().numpy()[held], dev.k[held])
    assert np.array_equal(cache.v.cpu().numpy()[held], dev.v[held])


@pytest.mark.parametrize("case", CASES[:4], ids=lambda c: f"{c[4]}_G{c[1] // c[2]}_D{c[3]}")
@pytest.mark.parametrize("scale", [None, 0.5])
def test_decode_fp8_wide_values(case, scale):
    """K, V and q drawn N(0, 4) (scales covering 6 standard deviations),
    with the default logit scale and a sharper one (peaked attention, whose
    outputs approach single V values of magnitude up to ~8).  Where the
    output's magnitude makes the 16-bit format's own half-ulp larger than
    the stated tolerance (bf16 past 4, fp16 past 8), the bound is that
    half-ulp of the oracle's value plus a 2^-14 relative slack; elsewhere
    the stated tolerance."""
    m = pkv()
    ctx, Hq, Hkv, D, dt = case
    ks = vs = 2.0 * 6.0 / 448.0
    ref, kc, vc, tables, lens = build(ctx, Hkv, D, dt, ks, vs, seed=7 * len(ctx) + D, sigma=2.0)
    rng = np.random.default_rng(D + len(ctx))
    q = storage(rng.standard_normal((len(ctx), Hq, D)).astype(np.float32) * 2.0, dt)
    sc = D ** -0.5 if scale is None else scale
    want = oracle.paged_decode(q, ref.k, ref.v, tables, lens, sc, dt, kv_dtype="e4m3", k_scale=ks, v_scale=vs)
    out = m.paged_attention_decode_fp8(to_dev(q, dt), kc, vc, torch.from_numpy(tables).cuda(),
                                       torch.from_numpy(lens).cuda(), int(lens.max()), sc, ks, vs)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert (np.abs(got - want) <= ulp_aware_bound(want, dt, TOL[dt])).all()
    if scale is not None:
        assert np.abs(want).max() > 4.0  # the wide range is really exercised


@pytest.mark.parametrize("case", [
    ("f16", 12, 256, (1, 100), 8, 8, 128, 0),
    ("bf16", 20, 512, (0, 700), 16, 2, 128, 0),
    ("bf16", 9, 160, (3, 40), 8, 2, 64, 0),
    ("f16", 12, 256, (1, 300), 8, 4, 128, 64),
], ids=lambda c: f"{c[0]}_B{c[1]}_G{c[4] // c[5]}_D{c[6]}_p{c[7]}")
def test_cascade_over_fp8_cache_matches_oracle(case):
    """The shared-prefix decode over an FP8 pool (prefix pass on the exact
    16-bit code values, suffix pass over the codes, merge) against the
    oracle on the stored values, and against the plain FP8 decode; a
    relabelled table (a sequence that does not start with the prefix) is
    decoded over its whole context."""
    import workloads
    from paged_kv_cache_365_b200.replay import build_step
    m = pkv()
    dt, B, pre, suf, Hq, Hkv, D, partition = case
    wl = workloads.prefix13b(seed=B + pre, B=B, prefix_tokens=pre, suffix_range=suf, Hq=Hq, Hkv=Hkv, D=D, dtype=dt,
                             name="fp8_cascade")
    vals = workloads.draw_values(wl)
    st = build_step(wl, vals, "cuda")
    c = st["cache"]
    m.copy_blocks(c.k, c.v, st["cow_pairs"])
    m.kv_append(st["k_new"], st["v_new"], c.k, c.v, st["slot_mapping"])
    ks, vs = 6.0 / 448.0, 5.0 / 448.0
    NB = c.k.shape[0]
    k8 = torch.empty(c.k.shape, dtype=torch.uint8, device="cuda")
    v8 = torch.empty(c.v.shape, dtype=torch.uint8, device="cuda")
    all_slots = torch.arange(NB * 16, dtype=torch.int64, device="cuda")
    rows_k = c.k.permute(0, 2, 1, 3).reshape(NB * 16, Hkv, D).contiguous()
    rows_v = c.v.permute(0, 2, 1, 3).reshape(NB * 16, Hkv, D).contiguous()
    m.kv_append_fp8(rows_k, rows_v, k8, v8, all_slots, ks, vs)
    tables, lens = st["host"]["block_tables"], st["host"]["context_lens"]
    tables = tables.copy()
    pp = m.common_prefix_pages(tables, lens)
    assert pp >= 8
    # sequence 1 keeps its blocks but its table names a different block for
    # page 0: give it a private copy of that block (codes copied bit for bit)
    spare = int(min(set(range(NB)) - set(tables.ravel().tolist())))  # a block no table of the batch names
    k8[spare] = k8[int(tables[1, 0])]
    v8[spare] = v8[int(tables[1, 0])]
    tables[1, 0] = spare
    prefix = torch.from_numpy(np.ascontiguousarray(tables[0, :pp])).cuda()
    dt_t = torch.from_numpy(np.ascontiguousarray(tables)).cuda()
    out = m.paged_attention_decode_prefix_fp8(st["q"], k8, v8, dt_t, st["context_lens"], st["max_context_len"], prefix,
                                              wl.scale, ks, vs, partition=partition)
    plain = m.paged_attention_decode_fp8(st["q"], k8, v8, dt_t, st["context_lens"], st["max_context_len"], wl.scale,
                                         ks, vs)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    codes_k, codes_v = k8.cpu().numpy(), v8.cpu().numpy()
    want = oracle.paged_decode(vals["q"], codes_k, codes_v, tables, lens, wl.scale, dt, kv_dtype="e4m3",
                               k_scale=ks, v_scale=vs)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL[dt]
    assert np.abs(got - plain.float().cpu().numpy()).max() <= TOL[dt]


# ---- several query tokens per sequence over an FP8 cache ---------------------

MULTI_CASES = [
    # ctx, new tokens, Hq, Hkv, D, q dtype
    ([5, 16, 17, 40, 1], [1, 4, 17, 8, 1], 4, 4, 128, "f16"),   # a few rows (one padded tile)
    ([33, 20, 3, 64], [5, 20, 3, 16], 8, 2, 64, "bf16"),        # 64 rows per kv-head
    ([300, 140, 2100], [150, 40, 33], 2, 1, 128, "bf16"),       # 300 rows: three tiles; two partitions
    ([1030, 600], [40, 33], 2, 2, 64, "f16"),
    ([700, 1500, 90], [5, 5, 3], 32, 8, 128, "bf16"),           # G = 4, 20 rows
]


def run_multi_fp8(q, kc, vc, tables, lens, qs, scale, ks, vs, dt, partition=0):
    m = pkv()
    out = m.paged_attention_multi_fp8(to_dev(q, dt), kc, vc, torch.from_numpy(tables).cuda(),
                                      torch.from_numpy(lens).cuda(), torch.from_numpy(qs).cuda(), int(lens.max()),
                                      int(np.diff(qs).max()), scale, ks, vs, partition=partition)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), m.get_error()


@pytest.mark.parametrize("case", MULTI_CASES, ids=lambda c: f"{c[5]}_G{c[2] // c[3]}_D{c[4]}_rows{max(c[1]) * c[2] // c[3]}")
@pytest.mark.parametrize("partition", [0, 16, 96])
def test_multi_fp8_matches_oracle(case, partition):
    """The tcgen05 kernel over E4M3 codes (widened in shared memory) against
    the oracle's multi-token attention on the stored values; unwritten slots
    hold the NaN code, tables are padded with out-of-range ids."""
    ctx, nq, Hq, Hkv, D, dt = case
    ks, vs = 0.011, 0.017
    ref, kc, vc, tables, lens = build(ctx, Hkv, D, dt, ks, vs, seed=sum(ctx) + D)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    rng = np.random.default_rng(partition + D + len(ctx))
    q = storage(rng.standard_normal((int(qs[-1]), Hq, D)).astype(np.float32), dt)
    scale = D ** -0.5
    want = oracle.paged_multi(q, ref.k, ref.v, tables, lens, qs, scale, dt, kv_dtype="e4m3", k_scale=ks, v_scale=vs)
    got, err = run_multi_fp8(q, kc, vc, tables, lens, qs, scale, ks, vs, dt, partition)
    assert err == 0
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL[dt]


@pytest.mark.parametrize("case", [MULTI_CASES[1], MULTI_CASES[2]],
                         ids=lambda c: f"{c[5]}_G{c[2] // c[3]}_D{c[4]}")
@pytest.mark.parametrize("scale", [None, 0.5])
def test_multi_fp8_wide_values(case, scale):
    """K, V and q drawn N(0, 4), bf16 queries with magnitudes that the
    per-row power-of-two rescale must carry into fp16; bound as in
    test_decode_fp8_wide_values (ulp-aware where the output is large)."""
    ctx, nq, Hq, Hkv, D, dt = case
    ks = vs = 2.0 * 6.0 / 448.0
    ref, kc, vc, tables, lens = build(ctx, Hkv, D, dt, ks, vs, seed=3 * sum(ctx) + D, sigma=2.0)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    rng = np.random.default_rng(D + 5)
    q = storage(rng.standard_normal((int(qs[-1]), Hq, D)).astype(np.float32) * 2.0, dt)
    sc = D ** -0.5 if scale is None else scale
    want = oracle.paged_multi(q, ref.k, ref.v, tables, lens, qs, sc, dt, kv_dtype="e4m3", k_scale=ks, v_scale=vs)
    got, err = run_multi_fp8(q, kc, vc, tables, lens, qs, sc, ks, vs, dt)
    assert err == 0
    assert np.isfinite(got).all()
    assert (np.abs(got - want) <= ulp_aware_bound(want, dt, TOL[dt])).all()
    if scale is not None:
        assert np.abs(want).max() > 4.0


def test_multi_fp8_large_and_small_query_rows():
    """bf16 query rows far outside fp16's range (1e6) and far below its
    normal range (1e-6): the per-row rescale keeps both; the logit scale is
    chosen so the attention stays well-conditioned."""
    ctx, nq, Hq, Hkv, D, dt = [90, 40], [20, 9], 4, 2, 128, "bf16"
    ks, vs = 0.011, 0.017
    ref, kc, vc, tables, lens = build(ctx, Hkv, D, dt, ks, vs, seed=77)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    rng = np.random.default_rng(8)
    q32 = rng.standard_normal((int(qs[-1]), Hq, D)).astype(np.float32)
    q32[::2] *= 1e6
    q32[1::2] *= 1e-6
    q = storage(q32, dt)
    for scale in (1e-7, 1e5):
        want = oracle.paged_multi(q, ref.k, ref.v, tables, lens, qs, scale, dt, kv_dtype="e4m3", k_scale=ks,
                                  v_scale=vs)
        got, err = run_multi_fp8(q, kc, vc, tables, lens, qs, scale, ks, vs, dt)
        assert err == 0 and np.isfinite(got).all()
        rows = slice(0, None, 2) if scale < 1 else slice(1, None, 2)
        assert np.abs(got[rows] - want[rows]).max() <= TOL[dt]


def test_multi_fp8_rejects_bad_scales_and_16_bit_pools():
    m = pkv()
    ref, kc, vc, tables, lens = build([20], 1, 64, "f16", 0.05, 0.05, seed=1)
    qs = np.array([0, 4], dtype=np.int32)
    q = torch.zeros((4, 1, 64), dtype=torch.float16, device="cuda")
    args = (q, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(), torch.from_numpy(qs).cuda(),
            20, 4, 0.125)
    for ks, vs in ((0.0, 0.05), (0.05, -1.0), (float("inf"), 0.05)):
        with pytest.raises(m.PkvError):
            m.paged_attention_multi_fp8(*args, ks, vs)
    with pytest.raises(ValueError):
        m.paged_attention_multi_fp8(q, kc.half(), vc.half(), *args[3:], 0.05, 0.05)


def test_multi_step_over_an_fp8_pool_through_the_cache_api():
    """PagedKVCache with an FP8 pool: prefill, a fork that forces a
    copy-on-write, then plan_multi_step + run_multi_step (host inputs); the
    pool's codes bit-exact and the output against the oracle."""
    m = pkv()
    rng = np.random.default_rng(43)
    Hq, Hkv, D, nb, ks, vs = 8, 2, 128, 48, 0.013, 0.019
    order = rng.permutation(nb).astype(np.int32)
    cache = m.PagedKVCache(nb, Hkv, D, torch.bfloat16, free_order=order, fp8_scales=(ks, vs))
    ref = oracle.RefAllocator(nb, order)
    dev = oracle.RefCache(nb, Hkv, D, "e4m3")

    def vals(n):
        return (storage(rng.standard_normal((n, Hkv, D)).astype(np.float32), "bf16"),
                storage(rng.standard_normal((n, Hkv, D)).astype(np.float32), "bf16"))

    for sid, n in ((0, 70), (1, 16), (2, 200)):
        ref.add_seq(sid)
        cache.add_seq(sid)
        k, v = vals(n)
        slots, cows = ref.append_tokens(sid, n)
        dev.copy_blocks(cows)
        dev.append_fp8(k, v, np.array(slots), "bf16", ks, vs)
        cache.prefill(sid, to_dev(k, "bf16"), to_dev(v, "bf16"))
    ref.fork(0, 3)
    cache.fork(0, 3)
    ids, n_new = [0, 1, 2, 3], [5, 3, 40, 4]
    slots, pairs, qs, tables, lens = cache.plan_multi_step(ids, n_new)
    r_slots, r_pairs = [], []
    for sid, n in zip(ids, n_new):
        s_, p_ = ref.append_tokens(sid, n)
        r_slots += s_
        r_pairs += p_
    assert list(slots) == r_slots and [tuple(p) for p in pairs] == r_pairs
    T = int(qs[-1])
    q = storage(rng.standard_normal((T, Hq, D)).astype(np.float32), "bf16")
    kn, vn = vals(T)
    dev.copy_blocks(r_pairs)
    dev.append_fp8(kn, vn, np.array(r_slots), "bf16", ks, vs)
    out = torch.empty((T, Hq, D), dtype=torch.bfloat16, pin_memory=True)
    cache.run_multi_step(torch.from_numpy(slots).pin_memory(), torch.from_numpy(pairs).pin_memory(),
                         torch.from_numpy(tables).pin_memory(), torch.from_numpy(lens).pin_memory(),
                         int(lens.max()), torch.from_numpy(qs).pin_memory(), max(n_new),
                         to_dev(q, "bf16").cpu().pin_memory(), to_dev(kn, "bf16").cpu().pin_memory(),
                         to_dev(vn, "bf16").cpu().pin_memory(), out=out)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    held = sorted({b for t in ref.tables.values() for b in t})
    assert np.array_equal(cache.k.cpu().numpy()[held], dev.k[held])
    assert np.array_equal(cache.v.cpu().numpy()[held], dev.v[held])
    want = oracle.paged_multi(q, dev.k, dev.v, tables, lens, qs, D ** -0.5, "bf16", kv_dtype="e4m3", k_scale=ks,
                              v_scale=vs)
    assert np.abs(out.float().numpy() - want).max() <= TOL["bf16"]


STEP_CASES = [  # (name, dtype, Hq, Hkv, D, partition, cascade)
    ("fp8_step_f16_G4", "f16", 8, 2, 128, 0, False),
    ("fp8_step_bf16_G2_split", "bf16", 8, 4, 64, 64, False),
    ("fp8_step_bf16_G8", "bf16", 8, 1, 128, 0, False),
    ("fp8_step_f16_G1_split", "f16", 4, 4, 128, 32, False),
    ("fp8_step_cascade_f16_G4", "f16", 8, 2, 128, 0, True),
    ("fp8_step_cascade_bf16_G1_split", "bf16", 4, 4, 64, 64, True),
]


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: c[0])
def test_fused_fp8_step_matches_separate_calls(case):
    """pkv_decode_step_fp8 (the copy-on-write copies and the quantising
    append made by the decode's CTAs; in the cascade by its suffix pass,
    which runs beside the prefix pass) against copy_blocks, kv_append_fp8
    and paged_attention_decode_fp8 / _prefix_fp8 on the same FP8 pool:
    every token row of the pool and the output bit-identical; the output
    within tolerance of the oracle, whose FP8 pool is its own replay of the
    workload with every token row quantised by oracle.fp8.quantize."""
    import workloads
    from paged_kv_cache_365_b200.replay import build_step
    m = pkv()
    name, dt, Hq, Hkv, D, partition, cascade = case
    wl = workloads.prefix13b(seed=71, B=10, prefix_tokens=256, suffix_range=(1, 300), Hq=Hq, Hkv=Hkv, D=D,
                             dtype=dt, name=name)
    ks, vs = 0.011, 0.017
    vals = workloads.draw_values(wl)
    st = build_step(wl, vals, "cuda")
    c = st["cache"]
    copies = m.cow_copy_rows(st["host"]["cow_pairs"], st["host"]["step_slots"])
    assert len(copies) > 0
    dcopies = torch.from_numpy(copies).cuda()
    tables, lens = st["host"]["block_tables"], st["host"]["context_lens"]
    nb = c.k.shape[0]
    # the 16-bit pool before the step, quantised row by row
    rows_k = c.k.permute(0, 2, 1, 3).reshape(nb * 16, wl.Hkv, D).contiguous()
    rows_v = c.v.permute(0, 2, 1, 3).reshape(nb * 16, wl.Hkv, D).contiguous()
    slots_all = torch.arange(nb * 16, dtype=torch.int64, device="cuda")
    kf = torch.full((nb, wl.Hkv, 16, D), 0x7F, dtype=torch.uint8, device="cuda")
    vf = torch.full_like(kf, 0x7F)
    m.kv_append_fp8(rows_k, rows_v, kf, vf, slots_all, ks, vs)
    kf2, vf2 = kf.clone(), vf.clone()
    prefix = None
    if cascade:
        pp = m.cascade_prefix_pages(tables, lens, torch.uint8)
        assert pp > 0
        prefix = torch.from_numpy(np.ascontiguousarray(tables[0, :pp])).cuda()
    m.copy_blocks(kf2, vf2, st["cow_pairs"])
    m.kv_append_fp8(st["k_new"], st["v_new"], kf2, vf2, st["slot_mapping"], ks, vs)
    if cascade:
        sep = m.paged_attention_decode_prefix_fp8(st["q"], kf2, vf2, st["block_tables"], st["context_lens"],
                                                  st["max_context_len"], prefix, wl.scale, ks, vs,
                                                  partition=partition)
    else:
        sep = m.paged_attention_decode_fp8(st["q"], kf2, vf2, st["block_tables"], st["context_lens"],
                                           st["max_context_len"], wl.scale, ks, vs, partition=partition)
    fused = m.decode_step_fp8(st["q"], kf, vf, st["k_new"], st["v_new"], st["slot_mapping"], dcopies,
                              st["block_tables"], st["context_lens"], st["max_context_len"], wl.scale, ks, vs,
                              prefix_blocks=prefix, partition=partition)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    assert torch.equal(fused.view(torch.int16), sep.view(torch.int16))
    gk, gv, sk, sv = (t.cpu().numpy() for t in (kf, vf, kf2, vf2))
    ref = oracle.replay(wl, vals)
    rk = oracle.RefCache(nb, wl.Hkv, D, "e4m3")
    for b in range(wl.B):
        tok = np.arange(int(lens[b]))
        blk, off = tables[b, tok // 16], tok % 16
        assert np.array_equal(gk[blk, :, off], sk[blk, :, off])
        assert np.array_equal(gv[blk, :, off], sv[blk, :, off])
        rk.append_fp8(ref["cache"].k[blk, :, off], ref["cache"].v[blk, :, off],
                      blk.astype(np.int64) * 16 + off, wl.dtype, ks, vs)
    for b in range(wl.B):
        tok = np.arange(int(lens[b]))
        blk, off = tables[b, tok // 16], tok % 16
        assert np.array_equal(gk[blk, :, off], rk.k[blk, :, off])
        assert np.array_equal(gv[blk, :, off], rk.v[blk, :, off])
    want = oracle.paged_decode(vals["q"], rk.k, rk.v, ref["block_tables"], ref["context_lens"], wl.scale, wl.dtype,
                               kv_dtype="e4m3", k_scale=ks, v_scale=vs)
    assert np.abs(fused.float().cpu().numpy() - want).max() <= TOL[dt]


@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("partition", [0, 256])
def test_fp8_reference_max_moves_mid_sequence(G, partition):
    """Scores that climb page after page over an FP8 pool (K's first entry
    grows along each sequence, the queries' first entry is 4): the FP8
    decode's reference max moves only past 2^8, rescaling what it has
    accumulated, and the result must stay the oracle's within tolerance."""
    m = pkv()
    dt, Hkv, D = "f16", 2, 128
    ctx = [700, 1500, 37, 2100]
    ks, vs = 1.0, 0.017
    ref, kc, vc, tables, lens = build(ctx, Hkv, D, dt, ks, vs, seed=41 + G, ramp=3.0)
    rng = np.random.default_rng(7 + G)
    q32 = rng.standard_normal((len(ctx), Hkv * G, D)).astype(np.float32)
    q32[:, :, 0] = 4.0
    q = storage(q32, dt)
    scale = D ** -0.5
    want = oracle.paged_decode(q, ref.k, ref.v, tables, lens, scale, dt, kv_dtype="e4m3", k_scale=ks, v_scale=vs)
    out = m.paged_attention_decode_fp8(to_dev(q, dt), kc, vc, torch.from_numpy(tables).cuda(),
                                       torch.from_numpy(lens).cuda(), int(lens.max()), scale, ks, vs,
                                       partition=partition)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL[dt]
