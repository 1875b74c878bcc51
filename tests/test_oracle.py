"""Pins of the fp64 oracle against things other than itself.

* brute force: pure-Python attention over each sequence's tokens in logical
  order, read straight from the drawn values (no allocator, slot or table),
  must agree with the paged oracle to 1e-12;
* relabelling every physical block leaves the output bit-identical;
* a shared prefix and a private copy of it give bit-identical output;
* closed forms: one token gives that token's V exactly; a zero query, a zero
  scale or identical keys give the mean of V; one dominant logit gives that
  token's V;
* exact widening of the stored formats (bf16 bit patterns with known values);
* unwritten slots hold NaN, so a finite output proves they were never read.
"""
import math

import numpy as np
import pytest

import oracle
import workloads
from helpers import logical_rows, privatise, relabel_blocks


def _run(wl):
    vals = workloads.draw_values(wl)
    st = oracle.replay(wl, vals)
    out = oracle.paged_decode(vals["q"], st["cache"].k, st["cache"].v, st["block_tables"],
                              st["context_lens"], wl.scale, wl.dtype)
    return vals, st, out


def _brute(wl, vals, b, h):
    G = wl.Hq // wl.Hkv
    keys, values = logical_rows(wl, vals, b, h // G, oracle.widen)
    q = oracle.widen(vals["q"][b, h], wl.dtype)
    return np.array(oracle.contiguous_decode(list(q), [list(r) for r in keys],
                                             [list(r) for r in values], wl.scale))


TINY_CASES = [
    workloads.tiny(0),
    workloads.custom([1, 5, 16, 17, 40], Hq=4, Hkv=2, D=8, dtype="bf16", seed=3, name="gqa2_bf16"),
    workloads.custom([2, 31, 32, 33], Hq=8, Hkv=1, D=16, dtype="f16", seed=4, name="mqa_f16"),
    workloads.prefix13b(seed=5, B=5, prefix_tokens=48, suffix_range=(1, 40), Hq=4, Hkv=2, D=8,
                        dtype="f32", name="prefix_tiny"),
]


@pytest.mark.parametrize("wl", TINY_CASES, ids=lambda w: w.name)
def test_paged_oracle_matches_contiguous_brute_force(wl):
    vals, st, out = _run(wl)
    assert np.isfinite(out).all(), "an unwritten (NaN) slot was read"
    assert list(st["context_lens"]) == list(wl.context_lens)
    for b in range(wl.B):
        for h in range(wl.Hq):
            ref = _brute(wl, vals, b, h)
            np.testing.assert_allclose(out[b, h], ref, rtol=0, atol=1e-12)


def test_brute_force_catches_wrong_gqa_mapping():
    """Sanity of the pin itself: using kv-head h % Hkv instead of h // G
    must disagree with the brute force."""
    wl = TINY_CASES[1]
    vals, st, out = _run(wl)
    G = wl.Hq // wl.Hkv
    b, h = 2, 1  # h // G = 0 but h % Hkv = 1
    keys, values = logical_rows(wl, vals, b, h % wl.Hkv, oracle.widen)
    q = oracle.widen(vals["q"][b, h], wl.dtype)
    wrong = oracle.decode_head(q, keys, values, wl.scale)
    assert G == 2 and np.abs(wrong - out[b, h]).max() > 1e-3


@pytest.mark.parametrize("wl", TINY_CASES[:3], ids=lambda w: w.name)
def test_block_relabelling_is_bit_identical(wl):
    vals, st, out = _run(wl)
    perm = np.random.default_rng(11).permutation(wl.num_blocks)
    k2, v2, t2 = relabel_blocks(st["cache"].k, st["cache"].v, st["block_tables"],
                                st["context_lens"], perm)
    out2 = oracle.paged_decode(vals["q"], k2, v2, t2, st["context_lens"], wl.scale, wl.dtype)
    assert np.array_equal(out, out2)


def test_shared_prefix_equals_private_copy():
    wl = TINY_CASES[3]
    vals, st, out = _run(wl)
    # the prefix really is shared before privatising
    tables = st["block_tables"]
    assert len({int(tables[b, 0]) for b in range(wl.B)}) == 1
    k2, v2, t2 = privatise(st["cache"].k, st["cache"].v, tables, st["context_lens"])
    out2 = oracle.paged_decode(vals["q"], k2, v2, t2, st["context_lens"], wl.scale, wl.dtype)
    assert np.array_equal(out, out2)


def _single_seq_cache(keys, values, dtype="f32", order=None):
    n, D = keys.shape
    pages = -(-n // 16)
    nb = pages + 3
    k = oracle.nan_fill((nb, 1, 16, D), dtype)
    v = oracle.nan_fill((nb, 1, 16, D), dtype)
    order = list(range(nb))[::-1] if order is None else order
    table = np.array([order[:pages]], dtype=np.int32)
    for j in range(n):
        k[table[0, j // 16], 0, j % 16] = keys[j]
        v[table[0, j // 16], 0, j % 16] = values[j]
    return k, v, table


def test_one_token_gives_its_value_exactly():
    rng = np.random.default_rng(1)
    key = rng.standard_normal((1, 32)).astype(np.float32)
    val = rng.standard_normal((1, 32)).astype(np.float32)
    q = rng.standard_normal((1, 1, 32)).astype(np.float32)
    k, v, t = _single_seq_cache(key, val)
    out = oracle.paged_decode(q, k, v, t, np.array([1]), 0.3, "f32")
    assert np.array_equal(out[0, 0], val[0].astype(np.float64))


@pytest.mark.parametrize("case", ["zero_query", "zero_scale", "equal_keys"])
def test_uniform_weights_give_mean_of_values(case):
    rng = np.random.default_rng(2)
    n, D = 37, 16
    keys = rng.standard_normal((n, D)).astype(np.float32)
    vals = rng.standard_normal((n, D)).astype(np.float32)
    q = rng.standard_normal((1, 1, D)).astype(np.float32)
    scale = 0.25
    if case == "zero_query":
        q[:] = 0
    elif case == "zero_scale":
        scale = 0.0
    else:
        keys[:] = keys[0]
    k, v, t = _single_seq_cache(keys, vals)
    out = oracle.paged_decode(q, k, v, t, np.array([n]), scale, "f32")
    mean = vals.astype(np.float64).mean(axis=0)
    np.testing.assert_allclose(out[0, 0], mean, rtol=0, atol=1e-14)


def test_dominant_logit_selects_its_value():
    rng = np.random.default_rng(3)
    n, D = 50, 16
    keys = np.zeros((n, D), dtype=np.float32)
    vals = rng.standard_normal((n, D)).astype(np.float32)
    q = np.zeros((1, 1, D), dtype=np.float32)
    q[0, 0, 0] = 1.0
    keys[23, 0] = 1000.0  # logit 1000 against 0 elsewhere: e^-1000 underflows
    k, v, t = _single_seq_cache(keys, vals)
    out = oracle.paged_decode(q, k, v, t, np.array([n]), 1.0, "f32")
    assert np.array_equal(out[0, 0], vals[23].astype(np.float64))


def test_two_logits_give_logistic_weights():
    """Closed form: two tokens with logit gap a weigh 1/(1+e^-a), 1/(1+e^a)."""
    D = 8
    keys = np.zeros((2, D), dtype=np.float32)
    keys[0, 0] = 1.5
    keys[1, 0] = -0.5
    vals = np.zeros((2, D), dtype=np.float32)
    vals[0, :] = 1.0
    vals[1, :] = -1.0
    q = np.zeros((1, 1, D), dtype=np.float32)
    q[0, 0, 0] = 1.0
    k, v, t = _single_seq_cache(keys, vals)
    out = oracle.paged_decode(q, k, v, t, np.array([2]), 0.5, "f32")
    a = 0.5 * (1.5 - (-0.5))
    w0 = 1.0 / (1.0 + math.exp(-a))
    np.testing.assert_allclose(out[0, 0], np.full(D, w0 - (1 - w0)), rtol=0, atol=1e-15)


def test_zero_length_sequence_gives_zeros():
    wl = workloads.custom([0, 3], Hq=2, Hkv=2, D=8, dtype="f16", seed=9)
    vals, st, out = _run(wl)
    assert np.array_equal(out[0], np.zeros((2, 8)))
    assert st["step_slots"][0] == -1


def test_widen_known_bit_patterns():
    bits = np.array([0x3F80, 0xC000, 0x3E20, 0x7F7F, 0x0001, 0x8000], dtype=np.uint16)
    expect = [1.0, -2.0, 0.15625, 3.3895313892515355e38, 2.0 ** -133, -0.0]
    got = oracle.widen(bits, "bf16")
    assert list(got) == expect
    assert math.copysign(1.0, got[-1]) == -1.0
    h = np.array([1.0, -2.0, 65504.0, 2.0 ** -24], dtype=np.float16)
    assert list(oracle.widen(h, "f16")) == [1.0, -2.0, 65504.0, 2.0 ** -24]


def test_bf16_draws_round_to_nearest_even():
    """The generator's bf16 cast: ties go to the even pattern."""
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9], dtype=np.float32)
    got = workloads._to_storage(x, "bf16")
    assert list(oracle.widen(got, "bf16")) == [1.0, 1.0 + 2.0 ** -6, 1.0]


def test_unwritten_slots_stay_nan():
    wl = TINY_CASES[0]
    vals, st, out = _run(wl)
    k = st["cache"].k
    written = 0
    for b, n in enumerate(st["context_lens"]):
        written += int(n)
    finite_rows = np.isfinite(k[:, 0, :, 0]).sum()
    assert finite_rows == written


def test_partial_copy_then_append_matches_full_copy_on_every_token():
    """Cutting a copy-on-write copy to the rows below the first appended row
    changes no token any sequence holds: for the shared-prefix workload's
    step (a copy per sequence), every (sequence, token) row is identical to
    the full-copy step's, and the decode output is bit-identical."""
    wl = workloads.prefix13b(seed=3, B=10, prefix_tokens=48, suffix_range=(1, 40), Hq=4, Hkv=2, D=8, dtype="f16",
                             name="pfx_rows")
    vals = workloads.draw_values(wl)
    full = oracle.replay(wl, vals)
    alloc = oracle.RefAllocator(wl.num_blocks, wl.free_order)
    cache = oracle.RefCache(wl.num_blocks, wl.Hkv, wl.D, wl.dtype)
    cursor = 0
    for op in wl.ops:
        if op[0] == "add":
            alloc.add_seq(op[1])
        elif op[0] == "fork":
            alloc.fork(op[1], op[2])
        elif op[0] == "free":
            alloc.free_seq(op[1])
        else:
            s_, c_ = alloc.append_tokens(op[1], op[2])
            cache.copy_blocks(c_)
            cache.append_many(vals["k_tokens"][cursor:cursor + op[2]], vals["v_tokens"][cursor:cursor + op[2]],
                              np.array(s_))
            cursor += op[2]
    ids = [int(s) for s in wl.step_seqs]
    slots, pairs = alloc.step(ids)
    assert len(pairs) > 0
    copies = []
    for src, dst in pairs:
        rows = min(int(s) % 16 for s in slots if int(s) // 16 == dst)
        copies.append((src, dst, rows))
    assert any(r < 16 for _, _, r in copies)
    cache.copy_rows_then_append(copies, vals["k_new"], vals["v_new"], np.array(slots))
    for b, sid in enumerate(ids):
        table, n = alloc.block_table(sid)
        for j in range(n):
            blk, off = table[j // 16], j % 16
            assert np.array_equal(cache.k[blk, :, off].view(np.int16), full["cache"].k[blk, :, off].view(np.int16))
            assert np.array_equal(cache.v[blk, :, off].view(np.int16), full["cache"].v[blk, :, off].view(np.int16))
    a = oracle.paged_decode(vals["q"], cache.k, cache.v, full["block_tables"], full["context_lens"], wl.scale, wl.dtype)
    b = oracle.paged_decode(vals["q"], full["cache"].k, full["cache"].v, full["block_tables"], full["context_lens"],
                            wl.scale, wl.dtype)
    assert np.array_equal(a, b)
