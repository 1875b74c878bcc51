"""Pins of the oracle's allocator: the pages' worked examples (fixtures
under tests/golden/, each with its citation) and invariants that must hold
after any sequence of operations."""
import json
import os

import numpy as np
import pytest

from oracle import RefAllocator, RefAllocError

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_block_table_example():
    g = load("block_table_example.json")
    a = RefAllocator(g["num_blocks"], g["free_order"], block_size=g["block_size"])
    a.add_seq(0)
    slots, cows = a.append_tokens(0, g["tokens"])
    table, n = a.block_table(0)
    assert table == g["expected_table"] and n == g["tokens"] and cows == []
    assert slots == g["expected_slots"]
    assert len(table) * g["block_size"] - n == g["expected_free_slots_in_last_block"]


def test_os_paging_example():
    g = load("os_paging_example.json")
    a = RefAllocator(g["num_blocks"], block_size=g["block_size"])
    for op in g["ops"]:
        if op[0] == "add":
            a.add_seq(op[1])
        elif op[0] == "append":
            a.append_tokens(op[1], op[2])
        elif op[0] == "free":
            a.free_seq(op[1])
    for sid, table in g["expected_tables"].items():
        assert a.block_table(sid)[0] == table
    assert a.state()[0] == g["expected_free_list"]


def test_utilisation_example():
    g = load("utilisation_example.json")
    n_req = len(g["request_tokens"])
    contiguous = sum(g["request_tokens"]) / (n_req * g["contiguous_slots_per_request"])
    assert contiguous == g["expected_contiguous_utilisation"]
    a = RefAllocator(g["num_blocks"], block_size=g["block_size"])
    for r, n in enumerate(g["request_tokens"]):
        a.add_seq(r)
        a.append_tokens(r, n)
    assert [a.block_table(r)[0] for r in range(n_req)] == g["expected_tables"]
    assert a.state()[0] == g["expected_free_list"]
    assert a.used_slots() == g["expected_used_slots"]
    assert a.allocated_slots() == g["expected_allocated_slots"]


def test_prefix_sharing_example():
    g = load("prefix_sharing_example.json")
    bs = g["block_size"]
    a = RefAllocator(g["num_blocks"], g["free_order"], block_size=bs)
    a.add_seq("prompt")
    a.append_tokens("prompt", g["prefix_blocks"] * bs)
    for r in range(3):
        a.fork("prompt", r)
    a.free_seq("prompt")
    for r, n in enumerate(g["private_tokens"]):
        a.append_tokens(r, n)
    assert [a.block_table(r)[0] for r in range(3)] == g["expected_tables"]
    free, rc = a.state()
    assert all(rc[b] == g["expected_prefix_refcount"] for b in range(g["prefix_blocks"]))
    in_use = g["num_blocks"] - len(free)
    assert in_use == g["expected_blocks_in_use"]
    unshared = sum(len(t) for t in g["expected_tables"])
    assert unshared == g["expected_blocks_without_sharing"]
    assert (unshared - in_use) == g["expected_saving_in_prefix_sizes"] * g["prefix_blocks"]


def test_copy_on_write_only_on_append_to_shared_partial_block():
    a = RefAllocator(8, block_size=4)
    a.add_seq("p")
    a.append_tokens("p", 6)          # blocks 0 (full), 1 (2 of 4)
    a.fork("p", "c")
    before = (a.state(), a.block_table("p"), a.block_table("c"))
    # reading never changes anything
    assert (a.state(), a.block_table("p"), a.block_table("c")) == before
    slot, cow = a.append_slot("c")    # writes into shared block 1 -> copy
    assert cow == (1, 2)
    assert a.block_table("c") == ([0, 2], 7) and slot == 2 * 4 + 2
    assert a.block_table("p") == ([0, 1], 6)
    free, rc = a.state()
    assert rc[:3] == [2, 1, 1]
    slot, cow = a.append_slot("p")    # block 1 is now private to p: no copy
    assert cow is None and slot == 1 * 4 + 2


def test_full_shared_block_gets_fresh_block_without_copy():
    a = RefAllocator(8, block_size=4)
    a.add_seq("p")
    a.append_tokens("p", 4)
    a.fork("p", "c")
    slot, cow = a.append_slot("c")
    assert cow is None and a.block_table("c") == ([0, 1], 5) and slot == 4


def test_freed_blocks_return_to_the_tail_of_the_pool():
    a = RefAllocator(4, block_size=4)
    a.add_seq(0)
    a.append_tokens(0, 8)            # blocks 0, 1
    a.free_seq(0)
    assert a.state()[0] == [2, 3, 0, 1]
    a.add_seq(1)
    a.append_tokens(1, 12)
    assert a.block_table(1)[0] == [2, 3, 0]


def test_out_of_memory_leaves_state_unchanged():
    a = RefAllocator(3, block_size=4)
    a.add_seq(0)
    a.append_tokens(0, 10)           # 3 blocks
    snap = (a.state(), a.block_table(0))
    with pytest.raises(RefAllocError) as e:
        a.append_tokens(0, 3)
    assert e.value.kind == "nomem"
    assert (a.state(), a.block_table(0)) == snap
    a.add_seq(1)
    with pytest.raises(RefAllocError):
        a.step([1])
    assert a.state() == snap[0]


def test_step_counts_copy_drops_between_siblings():
    """Two siblings share a partial block: the first copies, the second then
    owns the block alone and writes into it.  One free block suffices."""
    a = RefAllocator(3, block_size=4)
    a.add_seq("x")
    a.append_tokens("x", 5)          # blocks 0, 1 (1 of 4)
    a.fork("x", "y")
    slots, cows = a.step(["x", "y"])
    assert cows == [(1, 2)]
    assert a.block_table("x")[0] == [0, 2] and a.block_table("y")[0] == [0, 1]
    assert slots == [2 * 4 + 1, 1 * 4 + 1]


def test_invalid_calls_raise_and_change_nothing():
    a = RefAllocator(4)
    a.add_seq(1)
    snap = a.state()
    for bad in (lambda: a.add_seq(1), lambda: a.fork(9, 2), lambda: a.fork(1, 1),
                lambda: a.free_seq(7), lambda: a.append_slot(7), lambda: a.step([1, 1])):
        with pytest.raises(RefAllocError) as e:
            bad()
        assert e.value.kind == "inval"
    assert a.state() == snap
    with pytest.raises(RefAllocError):
        RefAllocator(3, [0, 1, 1])


def random_ops(rng, n_ops, max_seqs=12, max_append=40):
    ops = []
    live = []
    nxt = 0
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.15 or not live:
            ops.append(("add", nxt))
            live.append(nxt)
            nxt += 1
        elif r < 0.25:
            ops.append(("fork", int(rng.choice(live)), nxt))
            live.append(nxt)
            nxt += 1
        elif r < 0.33:
            s = int(rng.choice(live))
            ops.append(("free", s))
            live.remove(s)
        elif r < 0.6:
            k = int(rng.integers(1, min(len(live), 6) + 1))
            ops.append(("step", [int(x) for x in rng.choice(live, size=k, replace=False)]))
        else:
            ops.append(("append", int(rng.choice(live)), int(rng.integers(1, max_append))))
    return ops


def check_invariants(a, block_size):
    free, rc = a.state()
    holders = np.zeros(a.num_blocks, dtype=np.int64)
    for sid, table in a.tables.items():
        n = a.lengths[sid]
        # only the last block may be partly empty: waste < one block
        assert len(table) == -(-n // block_size)
        for blk in table:
            holders[blk] += 1
    assert list(holders) == rc
    assert sorted(free + [b for b in range(a.num_blocks) if rc[b] > 0]) == list(range(a.num_blocks))
    assert all(rc[b] == 0 for b in free)


@pytest.mark.parametrize("seed", range(6))
def test_invariants_hold_under_random_operations(seed):
    rng = np.random.default_rng(seed)
    bs = 4 if seed % 2 else 16
    a = RefAllocator(40, rng.permutation(40), block_size=bs)
    for op in random_ops(rng, 300):
        try:
            if op[0] == "add":
                a.add_seq(op[1])
            elif op[0] == "fork":
                a.fork(op[1], op[2])
            elif op[0] == "free":
                a.free_seq(op[1])
            elif op[0] == "append":
                a.append_tokens(op[1], op[2])
            else:
                a.step(op[1])
        except RefAllocError as e:
            assert e.kind == "nomem"
        check_invariants(a, bs)
