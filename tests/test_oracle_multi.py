"""Pins of the oracle's multi-token paged attention (several query tokens
per sequence, each attending causally over its sequence's tokens up to its
own position) against things other than itself:

* brute force in pure Python over each sequence's tokens in logical order,
  the keys cut at the row's position, read from the drawn values (no table);
* causality: changing K/V after a row's position leaves the row
  bit-identical, changing one at or before it does not;
* one query token per sequence is plain decode (the last row sees the whole
  context);
* closed form: equal keys give the running mean of V.
"""
import numpy as np
import pytest

import oracle
from helpers import make_multi_case as make_case


def run(c, scale=0.3):
    return oracle.paged_multi(c["q"], c["k"], c["v"], c["tables"], c["ctx"], c["qs"], scale, c["dtype"])


CASES = [
    dict(ctx=[5, 16, 17, 40], nq=[1, 4, 17, 8], Hq=2, Hkv=2, D=8, dtype="f32"),
    dict(ctx=[33, 20, 3], nq=[5, 20, 3], Hq=4, Hkv=2, D=8, dtype="bf16"),
    dict(ctx=[48, 7], nq=[16, 2], Hq=8, Hkv=1, D=16, dtype="f16"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c['dtype']}_G{c['Hq'] // c['Hkv']}")
def test_multi_matches_causal_brute_force(case):
    c = make_case(case["ctx"], case["nq"], case["Hq"], case["Hkv"], case["D"], case["dtype"], seed=9)
    out = run(c)
    assert np.isfinite(out).all()
    dt = c["dtype"]
    for b, n in enumerate(c["ctx"]):
        r0, r1 = c["qs"][b], c["qs"][b + 1]
        for i in range(r1 - r0):
            pos = n - (r1 - r0) + i
            for h in range(case["Hq"]):
                g = h // c["G"]
                keys = [list(oracle.widen(c["rows_k"][b][j, g], dt)) for j in range(pos + 1)]
                vals = [list(oracle.widen(c["rows_v"][b][j, g], dt)) for j in range(pos + 1)]
                qrow = list(oracle.widen(c["q"][r0 + i, h], dt))
                want = oracle.contiguous_decode(qrow, keys, vals, 0.3)
                np.testing.assert_allclose(out[r0 + i, h], want, rtol=0, atol=1e-12)


def test_brute_force_catches_an_off_by_one_mask():
    """A planted slip -- the row's own token left out -- is caught."""
    c = make_case([20], [6], 2, 2, 8, "f32", seed=2)
    out = run(c)
    b, n, nq = 0, 20, 6
    i = 3
    pos = n - nq + i
    keys = [list(oracle.widen(c["rows_k"][b][j, 0], "f32")) for j in range(pos)]
    vals = [list(oracle.widen(c["rows_v"][b][j, 0], "f32")) for j in range(pos)]
    wrong = oracle.contiguous_decode(list(oracle.widen(c["q"][i, 0], "f32")), keys, vals, 0.3)
    assert np.abs(out[i, 0] - np.array(wrong)).max() > 1e-6


def test_later_tokens_do_not_change_earlier_rows():
    c = make_case([40], [12], 4, 2, 8, "f32", seed=4)
    base = run(c)
    n, nq = 40, 12
    # overwrite the K/V of position 35 (rows of positions 28..34 must not move)
    t = c["tables"][0]
    c["k"][t[35 // 16], :, 35 % 16] += 1.0
    c["v"][t[35 // 16], :, 35 % 16] -= 2.0
    after = run(c)
    first_seeing = 35 - (n - nq)
    assert np.array_equal(after[:first_seeing], base[:first_seeing])
    assert not np.allclose(after[first_seeing:], base[first_seeing:])


def test_single_query_token_is_decode():
    c = make_case([9, 16, 50], [1, 1, 1], 4, 4, 16, "f16", seed=6)
    multi = run(c)
    dec = oracle.paged_decode(c["q"], c["k"], c["v"], c["tables"], c["ctx"], 0.3, "f16")
    assert np.array_equal(multi, dec)


def test_equal_keys_give_running_mean():
    rng = np.random.default_rng(8)
    c = make_case([30], [30], 1, 1, 8, "f32", seed=8)
    key = rng.standard_normal(8).astype(np.float32)
    t = c["tables"][0]
    for j in range(30):
        c["k"][t[j // 16], 0, j % 16] = key
    out = run(c)
    vals = np.stack([c["v"][t[j // 16], 0, j % 16].astype(np.float64) for j in range(30)])
    for i in range(30):
        np.testing.assert_allclose(out[i, 0], vals[:i + 1].mean(0), rtol=0, atol=1e-12)


def test_more_queries_than_context_gives_zero_rows():
    c = make_case([3], [5], 2, 2, 8, "f32", seed=1)
    out = run(c)
    assert np.array_equal(out[:2], np.zeros_like(out[:2]))
    assert np.isfinite(out[2:]).all()
