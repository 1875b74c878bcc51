"""GPU parity of the FP8 (E4M3) KV cache against the oracle: the quantising
append bit-exact (codes, every block of the pool), decode over the FP8
cache within the query dtype's tolerance (2e-3 fp16, 1e-2 bf16) of the fp64
oracle evaluated on the stored values (code value x scale).  Unwritten
slots hold the NaN code and tables are padded with out-of-range ids."""
import numpy as np
import pytest
import torch

import oracle
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


def build(ctx, Hkv, D, dt, ks, vs, seed):
    """An FP8 pool written through the GPU append and the oracle append from
    the same 16-bit values; returns both plus tables."""
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
    kx = storage(rng.standard_normal((n, Hkv, D)).astype(np.float32), dt)
    vx = storage(rng.standard_normal((n, Hkv, D)).astype(np.float32), dt)
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
