"""The library's C++ allocator against the oracle's allocator, bit for bit:
free list in order, every refcount, every table, every slot and copy pair,
after each operation of seeded random op sequences (host only, no GPU).
Also the pages' worked examples at the library's fixed block size 16."""
import json
import os

import numpy as np
import pytest

import workloads
from oracle import RefAllocator, RefAllocError, replay as oracle_replay

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_365_b200 as m
    return m


def same_state(lib_a, ref):
    lf, lrc = lib_a.state()
    rf, rrc = ref.state()
    assert lf == rf
    assert lrc == rrc
    assert lib_a.num_seqs == len(ref.tables)
    for sid in ref.tables:
        assert lib_a.block_table(sid) == ref.block_table(sid)


def random_ops(rng, n_ops):
    ops, live, nxt = [], [], 0
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.12 or not live:
            ops.append(("add", nxt)); live.append(nxt); nxt += 1
        elif r < 0.22:
            ops.append(("fork", int(rng.choice(live)), nxt)); live.append(nxt); nxt += 1
        elif r < 0.30:
            s = int(rng.choice(live)); ops.append(("free", s)); live.remove(s)
        elif r < 0.55:
            k = int(rng.integers(1, min(len(live), 8) + 1))
            ops.append(("step", [int(x) for x in rng.choice(live, size=k, replace=False)]))
        elif r < 0.60:
            ops.append(("slot", int(rng.choice(live))))
        elif r < 0.63:  # invalid calls: unknown ids, duplicate ids, existing ids
            ops.append(("bad", int(rng.integers(0, 4))))
        else:
            ops.append(("append", int(rng.choice(live)), int(rng.integers(0, 60))))
    return ops


@pytest.mark.parametrize("seed", range(8))
def test_library_allocator_matches_oracle(pkv, seed):
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(20, 120))
    order = rng.permutation(nb).astype(np.int32)
    lib_a = pkv.BlockAllocator(nb, order)
    ref = RefAllocator(nb, order)
    for op in random_ops(rng, 400):
        kind = op[0]
        ref_err = lib_err = None
        if kind == "bad":
            which = op[1]
            calls = [
                (lambda: lib_a.free_seq(10 ** 9), lambda: ref.free_seq(10 ** 9)),
                (lambda: lib_a.step([0, 0]), lambda: ref.step([0, 0])),
                (lambda: lib_a.fork(10 ** 9, 10 ** 9 + 1), lambda: ref.fork(10 ** 9, 10 ** 9 + 1)),
                (lambda: lib_a.append_slot(10 ** 9), lambda: ref.append_slot(10 ** 9)),
            ][which]
            try:
                calls[0]()
            except pkv.PkvError as e:
                lib_err = e.status
            try:
                calls[1]()
            except RefAllocError as e:
                ref_err = e.kind
            assert lib_err == 1 and ref_err == "inval"
            same_state(lib_a, ref)
            continue
        try:
            if kind == "add":
                ref.add_seq(op[1])
            elif kind == "fork":
                ref.fork(op[1], op[2])
            elif kind == "free":
                ref.free_seq(op[1])
            elif kind == "append":
                r_out = ref.append_tokens(op[1], op[2])
            elif kind == "slot":
                r_out = ref.append_slot(op[1])
            else:
                r_out = ref.step(op[1])
        except RefAllocError as e:
            ref_err = e.kind
        try:
            if kind == "add":
                lib_a.add_seq(op[1])
            elif kind == "fork":
                lib_a.fork(op[1], op[2])
            elif kind == "free":
                lib_a.free_seq(op[1])
            elif kind == "append":
                l_out = lib_a.append_tokens(op[1], op[2])
            elif kind == "slot":
                l_out = lib_a.append_slot(op[1])
            else:
                l_out = lib_a.step(op[1])
        except pkv.PkvError as e:
            lib_err = e.status
        assert (ref_err is None) == (lib_err is None), (op, ref_err, lib_err)
        if ref_err is not None:
            assert {"inval": 1, "nomem": 2}[ref_err] == lib_err
        elif kind in ("append", "step"):
            assert list(l_out[0]) == list(r_out[0])
            assert [tuple(p) for p in l_out[1]] == [tuple(p) for p in r_out[1]]
        elif kind == "slot":
            assert l_out == r_out
        same_state(lib_a, ref)


def test_block_table_example_at_block_16(pkv):
    """Page 3 §2.3's 7 tokens at block 4 become 28 tokens at block 16: two
    pages in blocks 3 and 7, four slots left in the last one."""
    g = json.load(open(os.path.join(GOLDEN, "block_table_example.json")))
    a = pkv.BlockAllocator(g["num_blocks"], g["free_order"])
    a.add_seq(0)
    n = g["tokens"] * (16 // g["block_size"])
    slots, pairs = a.append_tokens(0, n)
    table, ln = a.block_table(0)
    assert table == g["expected_table"] and ln == n and len(pairs) == 0
    assert len(table) * 16 - ln == g["expected_free_slots_in_last_block"] * (16 // g["block_size"])


def test_os_paging_and_prefix_examples(pkv):
    g = json.load(open(os.path.join(GOLDEN, "os_paging_example.json")))
    a = pkv.BlockAllocator(g["num_blocks"])
    ids = {"A": 1, "B": 2, "C": 3}
    for op in g["ops"]:
        if op[0] == "add":
            a.add_seq(ids[op[1]])
        elif op[0] == "append":
            a.append_tokens(ids[op[1]], op[2])
        else:
            a.free_seq(ids[op[1]])
    for k, t in g["expected_tables"].items():
        assert a.block_table(ids[k])[0] == t
    assert a.state()[0] == g["expected_free_list"]

    g = json.load(open(os.path.join(GOLDEN, "prefix_sharing_example.json")))
    a = pkv.BlockAllocator(g["num_blocks"], g["free_order"])
    a.add_seq(99)
    a.append_tokens(99, g["prefix_blocks"] * 16)
    for r in range(3):
        a.fork(99, r)
    a.free_seq(99)
    for r, n in enumerate(g["private_tokens"]):
        a.append_tokens(r, n)
    assert [a.block_table(r)[0] for r in range(3)] == g["expected_tables"]
    free, rc = a.state()
    assert g["num_blocks"] - len(free) == g["expected_blocks_in_use"]
    assert all(rc[b] == g["expected_prefix_refcount"] for b in range(g["prefix_blocks"]))


def test_create_rejects_bad_free_order(pkv):
    with pytest.raises(pkv.PkvError):
        pkv.BlockAllocator(4, [0, 1, 1, 2])
    with pytest.raises(pkv.PkvError):
        pkv.BlockAllocator(0)


@pytest.mark.parametrize("name", ["tiny", "llama7b", "gqa8b", "prefix13b"])
def test_named_workload_plans_match_oracle(pkv, name):
    """Replaying a named workload's op log and step through both allocators
    gives identical tables, lengths, slots and copy pairs."""
    wl = workloads.named(name, seed=0)
    ref = RefAllocator(wl.num_blocks, wl.free_order)
    lib_a = pkv.BlockAllocator(wl.num_blocks, wl.free_order)
    for op in wl.ops:
        if op[0] == "add":
            ref.add_seq(op[1]); lib_a.add_seq(op[1])
        elif op[0] == "fork":
            ref.fork(op[1], op[2]); lib_a.fork(op[1], op[2])
        elif op[0] == "free":
            ref.free_seq(op[1]); lib_a.free_seq(op[1])
        else:
            rs, rc = ref.append_tokens(op[1], op[2])
            ls, lc = lib_a.append_tokens(op[1], op[2])
            assert list(ls) == rs and [tuple(p) for p in lc] == rc
    ids = [int(s) for s in wl.step_seqs]
    rs, rc = ref.step(ids)
    ls, lc = lib_a.step(ids)
    assert list(ls) == rs and [tuple(p) for p in lc] == rc
    same_state(lib_a, ref)
    tables, lens = lib_a.block_tables(ids, 1 + max(len(ref.block_table(s)[0]) for s in ids), -7)
    assert list(lens) == list(wl.context_lens)
    if name == "prefix13b":
        # every sequence whose cached suffix ends mid-block copied its block
        suffix = wl.context_lens - 1 - 1024
        assert len(rc) == int(np.sum(suffix % 16 != 0))
