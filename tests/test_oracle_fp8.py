"""Pins of the oracle's FP8 E4M3 codec against the format's published
definition (OCP FP8: bias 7, subnormals m * 2^-9, max 448, one NaN pattern
per sign) and against torch's float8_e4m3fn cast (a library implementation
of the same format) where the two are defined alike (|x| < 464: torch
turns larger values into NaN, the cache saturates them)."""
import math

import numpy as np
import pytest
import torch

from oracle import fp8


def test_spec_values():
    assert fp8.e4m3_value(0x7E) == 448.0
    assert fp8.e4m3_value(0xFE) == -448.0
    assert fp8.e4m3_value(0x01) == 2.0 ** -9
    assert fp8.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert fp8.e4m3_value(0x08) == 2.0 ** -6
    assert fp8.e4m3_value(0x38) == 1.0
    assert fp8.e4m3_value(0x3F) == 1.875
    assert fp8.e4m3_value(0xC0) == -2.0
    assert math.isnan(fp8.e4m3_value(0x7F)) and math.isnan(fp8.e4m3_value(0xFF))
    assert np.isfinite(fp8.TABLE).sum() == 254


@pytest.mark.parametrize("x,code", [
    (1.0625, 0x38),          # halfway 1 / 1.125 -> even (1.0)
    (1.1875, 0x3A),          # halfway 1.125 / 1.25 -> even (1.25)
    (1.07, 0x39),            # nearer 1.125
    (2.0 ** -10, 0x00),      # halfway 0 / 2^-9 -> even (0)
    (3 * 2.0 ** -10, 0x02),  # halfway 2^-9 / 2^-8 -> even
    (448.0, 0x7E), (460.0, 0x7E), (470.0, 0x7E), (1e6, 0x7E),  # saturation
    (-470.0, 0xFE), (-0.0, 0x80), (0.0, 0x00),
    (240.0, 0x77), (1.875 * 2.0 ** -6, 0x0F),  # 0x0F: exponent field 1, mantissa 7
])
def test_rounding_cases(x, code):
    assert int(fp8.e4m3_encode(np.array([x]))[0]) == code


def test_nan_and_round_trip():
    assert int(fp8.e4m3_encode(np.array([np.nan]))[0]) & 0x7F == 0x7F
    finite = [c for c in range(256) if np.isfinite(fp8.TABLE[c])]
    vals = fp8.e4m3_decode(np.array(finite, dtype=np.uint8))
    back = fp8.e4m3_encode(vals)
    assert list(back) == finite


def test_against_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(50000) * 3, rng.uniform(-463, 463, 20000),
                        rng.standard_normal(20000) * 2.0 ** -8]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.e4m3_encode(x.astype(np.float64)), want)


def test_quantize_divides_in_float32():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(20000).astype(np.float32)
    for scale in (1.0, 0.0123, 3.0, 1.0 / 7.0):
        want = (torch.from_numpy(x) / torch.tensor(scale, dtype=torch.float32)).to(torch.float8_e4m3fn)
        assert np.array_equal(fp8.quantize(x, scale), want.view(torch.uint8).numpy())


def test_fp8_cache_attention_matches_brute_force():
    """An FP8 cache written by append_fp8 through a permuted pool: the paged
    oracle (codes widened through the table, times the scales) against pure
    Python attention over the codes in logical order (no table, no slots)."""
    import oracle
    rng = np.random.default_rng(3)
    Hkv, Hq, D, n = 2, 4, 16, 37
    ks, vs = 0.02, 0.05
    kx = rng.standard_normal((n, Hkv, D)).astype(np.float16)
    vx = rng.standard_normal((n, Hkv, D)).astype(np.float16)
    pages = -(-n // 16)
    nb = pages + 3
    perm = rng.permutation(nb)
    slots = np.array([perm[j // 16] * 16 + j % 16 for j in range(n)], dtype=np.int64)
    cache = oracle.RefCache(nb, Hkv, D, "e4m3")
    cache.append_fp8(kx, vx, slots, "f16", ks, vs)
    kc, vc = fp8.quantize(kx.astype(np.float32), ks), fp8.quantize(vx.astype(np.float32), vs)
    q = rng.standard_normal((1, Hq, D)).astype(np.float16)
    table = np.array([list(perm[:pages]) + [nb + 9]], dtype=np.int32)
    out = oracle.paged_decode(q, cache.k, cache.v, table, np.array([n]), 0.25, "f16", kv_dtype="e4m3",
                              k_scale=ks, v_scale=vs)
    G = Hq // Hkv
    for h in range(Hq):
        keys = [[fp8.e4m3_value(int(c)) * ks for c in kc[j, h // G]] for j in range(n)]
        vals = [[fp8.e4m3_value(int(c)) * vs for c in vc[j, h // G]] for j in range(n)]
        want = oracle.contiguous_decode([float(x) for x in q[0, h]], keys, vals, 0.25)
        np.testing.assert_allclose(out[0, h], want, rtol=0, atol=1e-12)


def test_quantisation_error_within_half_an_fp8_step():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal(100000) * 4).astype(np.float32)
    scale = 0.01
    dq = fp8.e4m3_decode(fp8.quantize(x, scale)) * scale
    y = x.astype(np.float64) / scale
    normal = np.abs(y) >= 2.0 ** -6
    # 3 mantissa bits: half a step is at most 2^-4 of the magnitude (normals),
    # 2^-10 in absolute terms below 2^-6 (subnormals); values past 448 clip
    inside = np.abs(y) <= 448
    assert np.all(np.abs(dq - x)[normal & inside] <= 2.0 ** -4 * np.abs(x)[normal & inside] * (1 + 1e-6))
    assert np.all(np.abs(dq - x)[~normal] <= 2.0 ** -10 * scale * (1 + 1e-6))
    assert np.all(np.abs(dq[~inside]) == 448 * scale)


def _fp8_multi_case(rng, ctx, nq, Hkv, Hq, D, ks, vs):
    """Sequences' K/V drawn in logical order, quantised into a permuted FP8
    pool by append_fp8; their new tokens' queries in fp16."""
    import oracle
    pages = [-(-n // 16) for n in ctx]
    nb = sum(pages) + 3
    perm = rng.permutation(nb)
    cache = oracle.RefCache(nb, Hkv, D, "e4m3")
    tables = np.full((len(ctx), max(pages) + 1), nb + 5, dtype=np.int32)
    codes, at = [], 0
    for b, n in enumerate(ctx):
        kx = rng.standard_normal((n, Hkv, D)).astype(np.float16)
        vx = rng.standard_normal((n, Hkv, D)).astype(np.float16)
        blocks = perm[at:at + pages[b]]
        at += pages[b]
        tables[b, :pages[b]] = blocks
        slots = np.array([blocks[j // 16] * 16 + j % 16 for j in range(n)], dtype=np.int64)
        cache.append_fp8(kx, vx, slots, "f16", ks, vs)
        codes.append((fp8.quantize(kx.astype(np.float32), ks), fp8.quantize(vx.astype(np.float32), vs)))
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    q = rng.standard_normal((int(qs[-1]), Hq, D)).astype(np.float16)
    return cache, tables, qs, q, codes


def test_fp8_multi_matches_causal_brute_force():
    """Several new tokens per sequence over an FP8 cache: the paged oracle
    against pure Python causal attention over the codes in logical order
    (no table, no slots), each code's value times its scale."""
    import oracle
    rng = np.random.default_rng(5)
    Hkv, Hq, D, ks, vs = 2, 4, 16, 0.03, 0.07
    ctx, nq = [37, 16, 9], [5, 16, 2]
    cache, tables, qs, q, codes = _fp8_multi_case(rng, ctx, nq, Hkv, Hq, D, ks, vs)
    out = oracle.paged_multi(q, cache.k, cache.v, tables, np.array(ctx), qs, 0.25, "f16", kv_dtype="e4m3",
                             k_scale=ks, v_scale=vs)
    G = Hq // Hkv
    for b, n in enumerate(ctx):
        kc, vc = codes[b]
        for i in range(nq[b]):
            pos = n - nq[b] + i
            for h in range(Hq):
                keys = [[fp8.e4m3_value(int(c)) * ks for c in kc[j, h // G]] for j in range(pos + 1)]
                vals = [[fp8.e4m3_value(int(c)) * vs for c in vc[j, h // G]] for j in range(pos + 1)]
                want = oracle.contiguous_decode([float(x) for x in q[qs[b] + i, h]], keys, vals, 0.25)
                np.testing.assert_allclose(out[qs[b] + i, h], want, rtol=0, atol=1e-12)


def test_fp8_multi_brute_force_catches_a_swapped_scale():
    """A planted slip -- V's scale applied to K -- is caught."""
    import oracle
    rng = np.random.default_rng(6)
    Hkv, Hq, D = 1, 2, 16
    cache, tables, qs, q, _ = _fp8_multi_case(rng, [20], [4], Hkv, Hq, D, 0.03, 0.07)
    good = oracle.paged_multi(q, cache.k, cache.v, tables, np.array([20]), qs, 0.25, "f16", kv_dtype="e4m3",
                              k_scale=0.03, v_scale=0.07)
    bad = oracle.paged_multi(q, cache.k, cache.v, tables, np.array([20]), qs, 0.25, "f16", kv_dtype="e4m3",
                             k_scale=0.07, v_scale=0.07)
    assert np.abs(good - bad).max() > 1e-4
