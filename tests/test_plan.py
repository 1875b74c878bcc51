"""The library's host planning calls, through ctypes, against definitions
worked out here independently (no GPU):

* pkv_cow_copy_rows / pkv_alloc_step_copies: the copy-on-write row cut
  ("PagedAttention 与 vLLM 推理加速" §3.2(3)) -- rows = the first row of the
  new block that the step writes -- by brute force over the step's slots,
  and the property that defines it: copying only those rows and then
  appending (the oracle's RefCache.copy_rows_then_append) leaves every token
  row of every sequence equal to the whole-block copy followed by the
  append;
* pkv_common_prefix_pages: the longest run of leading pages that every
  table shares and every sequence fills, by brute force over the columns;
* pkv_cascade_prefix_pages: that prefix, gated by the thresholds and the
  dtype pkv.h states.
"""
import ctypes

import numpy as np
import pytest

import oracle
import workloads


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_365_b200 as m
    return m


def brute_rows(dst, slots):
    rows = 16
    for s in slots:
        s = int(s)
        if s >= 0 and s // 16 == dst:
            rows = min(rows, s % 16)
    return rows


def test_cow_copy_rows_brute_force(pkv):
    rng = np.random.default_rng(5)
    for _ in range(200):
        n = int(rng.integers(0, 12))
        dsts = rng.choice(200, size=n, replace=False)
        pairs = np.stack([rng.integers(200, 400, size=n), dsts], axis=1).astype(np.int32)
        m = int(rng.integers(0, 30))
        blocks = rng.choice(np.concatenate([dsts, rng.integers(0, 400, size=5)]), size=m) if m else np.zeros(0)
        slots = (blocks.astype(np.int64) * 16 + rng.integers(0, 16, size=m)) if m else np.zeros(0, np.int64)
        slots = np.where(rng.random(m) < 0.15, -1, slots).astype(np.int64)
        got = pkv.cow_copy_rows(pairs, slots)
        assert got.shape == (n, 3)
        for i in range(n):
            assert tuple(got[i]) == (pairs[i, 0], pairs[i, 1], brute_rows(int(pairs[i, 1]), slots))


def test_cow_copy_rows_rejects_bad_arguments(pkv):
    lib = pkv._lib.lib
    P32, P64 = ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)
    out = np.zeros((4, 3), np.int32)
    bad_pairs = np.array([[1, -2]], np.int32)
    slots = np.array([5], np.int64)
    assert lib.pkv_cow_copy_rows(bad_pairs.ctypes.data_as(P32), 1, slots.ctypes.data_as(P64), 1,
                                 out.ctypes.data_as(P32)) == pkv._lib.PKV_EINVAL
    assert lib.pkv_cow_copy_rows(None, 1, slots.ctypes.data_as(P64), 1, out.ctypes.data_as(P32)) == 1
    assert lib.pkv_cow_copy_rows(None, -1, None, 0, None) == 1
    assert lib.pkv_cow_copy_rows(None, 0, None, 0, None) == 0


@pytest.mark.parametrize("seed", range(3))
def test_step_copies_against_oracle_row_rule(pkv, seed):
    """A shared-prefix batch, forked once per sequence before the step (a
    copy per sequence whose suffix ends mid-block): the library's triples
    equal the oracle allocator's pairs with the brute-force row cut, and
    the cut copy + append leaves every token row as the whole-block copy."""
    wl = workloads.prefix13b(seed=10 + seed, B=12, prefix_tokens=48, suffix_range=(1, 40), Hq=4, Hkv=2, D=8,
                             dtype="f16", name="plan_rows")
    vals = workloads.draw_values(wl)
    full = oracle.replay(wl, vals)  # whole-block copies, then the append
    ref = oracle.RefAllocator(wl.num_blocks, wl.free_order)
    lib_a = pkv.BlockAllocator(wl.num_blocks, wl.free_order)
    cache = oracle.RefCache(wl.num_blocks, wl.Hkv, wl.D, wl.dtype)
    cursor = 0
    for op in wl.ops:
        if op[0] == "add":
            ref.add_seq(op[1]); lib_a.add_seq(op[1])
        elif op[0] == "fork":
            ref.fork(op[1], op[2]); lib_a.fork(op[1], op[2])
        elif op[0] == "free":
            ref.free_seq(op[1]); lib_a.free_seq(op[1])
        else:
            s_, c_ = ref.append_tokens(op[1], op[2])
            lib_a.append_tokens(op[1], op[2])
            cache.copy_blocks(c_)
            cache.append_many(vals["k_tokens"][cursor:cursor + op[2]], vals["v_tokens"][cursor:cursor + op[2]],
                              np.array(s_))
            cursor += op[2]
    ids = [int(s) for s in wl.step_seqs]
    ref_slots, ref_pairs = ref.step(ids)
    slots, copies = lib_a.step_copies(ids)
    assert slots.tolist() == list(ref_slots)
    assert [(int(a), int(b)) for a, b, _ in copies] == [tuple(p) for p in ref_pairs]
    assert len(copies) > 0
    for src, dst, rows in copies:
        assert rows == brute_rows(int(dst), slots)
    assert any(r < 16 for _, _, r in copies)
    cache.copy_rows_then_append([tuple(int(x) for x in c) for c in copies], vals["k_new"], vals["v_new"],
                                np.array(slots))
    for sid in ids:
        table, n = ref.block_table(sid)
        for j in range(n):
            blk, off = table[j // 16], j % 16
            assert np.array_equal(cache.k[blk, :, off].view(np.int16), full["cache"].k[blk, :, off].view(np.int16))
            assert np.array_equal(cache.v[blk, :, off].view(np.int16), full["cache"].v[blk, :, off].view(np.int16))


def brute_prefix(tables, lens):
    n, w = tables.shape
    if n < 2:
        return 0
    p = 0
    while p < w and all(int(lens[b]) >= 16 * (p + 1) for b in range(n)) and \
            all(tables[b, p] == tables[0, p] for b in range(n)):
        p += 1
    return p


def test_common_prefix_pages_brute_force(pkv):
    rng = np.random.default_rng(9)
    for _ in range(300):
        n = int(rng.integers(0, 7))
        w = int(rng.integers(1, 12))
        shared = int(rng.integers(0, w + 1))
        tables = rng.integers(0, 50, size=(n, w)).astype(np.int32)
        if n:
            tables[:, :shared] = tables[0, :shared]
            if rng.random() < 0.3 and shared:   # one sequence breaks the run
                tables[int(rng.integers(0, n)), int(rng.integers(0, shared))] = 99
        lens = rng.integers(0, 16 * w + 1, size=n).astype(np.int32)
        assert pkv.common_prefix_pages(tables, lens) == brute_prefix(tables, lens)


def test_cascade_prefix_pages_thresholds(pkv):
    import torch
    lib = pkv._lib
    w = 20
    base = np.arange(w, dtype=np.int32)
    for n, pages, dtype, want in [
            (4, 8, torch.float16, 8), (4, 7, torch.float16, 0), (3, 12, torch.bfloat16, 0),
            (6, 12, torch.bfloat16, 12), (6, 12, torch.float32, 0), (6, 12, torch.uint8, 12),
            (3, 12, torch.uint8, 0), (6, 7, torch.uint8, 0)]:
        tables = np.tile(base, (n, 1))
        tables[:, pages:] = 100 + np.arange(n)[:, None] * w + np.arange(w - pages)[None, :]
        lens = np.full(n, 16 * w, dtype=np.int32)
        assert pkv.common_prefix_pages(tables, lens) == pages
        assert pkv.cascade_prefix_pages(tables, lens, dtype) == want, (n, pages, dtype)
    assert lib.lib.pkv_cascade_prefix_pages(None, 2, 4, None, 1, None) == lib.PKV_EINVAL
    with pytest.raises(pkv.PkvError):
        pkv.common_prefix_pages(np.zeros((2, 3), np.int32), np.array([-1, 5], np.int32))
