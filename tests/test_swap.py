"""Preemption by swapping ("LLM Systems 24 ..." §3, conclusion: a request
preempted for lack of KV blocks is swapped out and later swapped back in).

Oracle pins: a hand-worked example of the policy, invariants of both pools
under random operation sequences, all-or-nothing failures, and the content
round trip (a swapped-out-and-in sequence attends to exactly the same K/V,
bit for bit, even after its old device blocks were overwritten).  Then the
library's C++ allocator against the oracle's, bit for bit, on random
sequences that include swaps (host only, no GPU)."""
import numpy as np
import pytest

from oracle import RefAllocError, RefAllocator, RefCache, paged_decode, swap_blocks


def holders(tables):
    cnt = {}
    for t in tables:
        for b in t:
            cnt[b] = cnt.get(b, 0) + 1
    return cnt


def check_invariants(a: RefAllocator):
    dev = holders(a.tables.values())
    host = holders(t for t, _ in a.swapped.values())
    free, rc = a.state()
    hfree, hrc = a.host_state()
    assert rc == [dev.get(b, 0) for b in range(a.num_blocks)]
    assert hrc == [host.get(b, 0) for b in range(a.num_host_blocks)]
    assert sorted(free + list(dev)) == list(range(a.num_blocks))
    assert sorted(hfree + list(host)) == list(range(a.num_host_blocks))
    for sid, (t, n) in a.swapped.items():
        assert len(t) == -(-n // 16)


def test_hand_worked_example():
    a = RefAllocator(8, num_host_blocks=4)
    a.add_seq(1)
    a.append_tokens(1, 20)          # blocks 0 (full), 1 (4 tokens)
    a.fork(1, 2)
    _, cows = a.append_tokens(2, 1)  # partial shared block 1 -> copy into 2
    assert cows == [(1, 2)] and a.tables == {1: [0, 1], 2: [0, 2]}
    # seq 2 alone: block 0 stays with seq 1, block 2 is released
    assert a.swap_out([2]) == [(0, 0), (2, 1)]
    assert a.state() == ([3, 4, 5, 6, 7, 2], [1, 1, 0, 0, 0, 0, 0, 0])
    assert a.host_state() == ([2, 3], [1, 1, 0, 0])
    assert a.swapped_table(2) == ([0, 1], 21)
    with pytest.raises(RefAllocError):
        a.append_slot(2)
    with pytest.raises(RefAllocError):
        a.fork(2, 3)
    assert a.swap_in([2]) == [(0, 3), (1, 4)]
    assert a.tables[2] == [3, 4] and a.lengths[2] == 21
    assert a.state() == ([5, 6, 7, 2], [1, 1, 0, 1, 1, 0, 0, 0])
    assert a.host_state() == ([2, 3, 0, 1], [0, 0, 0, 0])
    check_invariants(a)


def test_group_swap_keeps_sharing():
    """Siblings swapped together share one host copy of their common blocks
    and come back sharing device blocks (a later append still copies)."""
    a = RefAllocator(10, num_host_blocks=10)
    a.add_seq(0)
    a.append_tokens(0, 40)           # 0, 1, 2 (8 tokens in 2)
    a.fork(0, 1)
    pairs = a.swap_out([0, 1])
    assert pairs == [(0, 0), (1, 1), (2, 2)]
    assert a.host_state()[1][:3] == [2, 2, 2]
    assert a.state()[0] == [3, 4, 5, 6, 7, 8, 9, 0, 1, 2]
    pairs = a.swap_in([1, 0])
    assert pairs == [(0, 3), (1, 4), (2, 5)]
    assert a.tables == {1: [3, 4, 5], 0: [3, 4, 5]}
    _, cow = a.append_slot(0)
    assert cow == (5, 6)
    check_invariants(a)


def test_failed_swaps_change_nothing():
    a = RefAllocator(6, num_host_blocks=2)
    a.add_seq(0)
    a.append_tokens(0, 48)           # 3 blocks > 2 host blocks
    a.add_seq(1)
    before = (a.state(), a.host_state(), dict(a.tables), dict(a.swapped))
    for bad in ([0], [0, 0], [7], []):
        if bad == []:
            assert a.swap_out(bad) == []
            continue
        with pytest.raises(RefAllocError) as e:
            a.swap_out(bad)
        assert e.value.kind == ("nomem" if bad == [0] else "inval")
        assert (a.state(), a.host_state(), dict(a.tables), dict(a.swapped)) == before
    assert a.swap_out([1]) == []     # an empty sequence moves no block
    with pytest.raises(RefAllocError):
        a.swap_in([0])               # not swapped
    # swap in needs device room: fill the device pool first
    a2 = RefAllocator(3, num_host_blocks=3)
    a2.add_seq(0)
    a2.append_tokens(0, 40)
    a2.swap_out([0])
    a2.add_seq(1)
    a2.append_tokens(1, 17)          # 2 of the 3 device blocks
    with pytest.raises(RefAllocError) as e:
        a2.swap_in([0])
    assert e.value.kind == "nomem"
    a2.free_seq(0)                   # a swapped sequence can be dropped
    assert a2.host_state() == ([0, 1, 2], [0, 0, 0])
    check_invariants(a2)


def random_ops(rng, n_ops, with_swaps=True):
    ops, live, swapped, nxt = [], [], [], 0
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.12 or not live:
            ops.append(("add", nxt)); live.append(nxt); nxt += 1
        elif r < 0.20:
            ops.append(("fork", int(rng.choice(live)), nxt)); live.append(nxt); nxt += 1
        elif r < 0.26:
            s = int(rng.choice(live)); ops.append(("free", s)); live.remove(s)
        elif r < 0.40:
            k = int(rng.integers(1, min(len(live), 6) + 1))
            ops.append(("step", [int(x) for x in rng.choice(live, size=k, replace=False)]))
        elif r < 0.52 and with_swaps:
            k = int(rng.integers(1, min(len(live), 3) + 1))
            ids = [int(x) for x in rng.choice(live, size=k, replace=False)]
            ops.append(("out", ids))
            for s in ids:
                live.remove(s); swapped.append(s)
        elif r < 0.62 and with_swaps and swapped:
            k = int(rng.integers(1, min(len(swapped), 3) + 1))
            ids = [int(x) for x in rng.choice(swapped, size=k, replace=False)]
            ops.append(("in", ids))
            for s in ids:
                swapped.remove(s); live.append(s)
        elif r < 0.65 and swapped:
            s = int(rng.choice(swapped)); ops.append(("free", s)); swapped.remove(s)
        else:
            ops.append(("append", int(rng.choice(live)), int(rng.integers(0, 40))))
    return ops


def apply_ref(a, op):
    kind = op[0]
    if kind == "add":
        return a.add_seq(op[1])
    if kind == "fork":
        return a.fork(op[1], op[2])
    if kind == "free":
        return a.free_seq(op[1])
    if kind == "step":
        return a.step(op[1])
    if kind == "out":
        return a.swap_out(op[1])
    if kind == "in":
        return a.swap_in(op[1])
    return a.append_tokens(op[1], op[2])


@pytest.mark.parametrize("seed", range(6))
def test_oracle_invariants_under_random_swaps(seed):
    rng = np.random.default_rng(500 + seed)
    nb, nh = int(rng.integers(20, 60)), int(rng.integers(10, 60))
    a = RefAllocator(nb, rng.permutation(nb), num_host_blocks=nh)
    for op in random_ops(rng, 300):
        state = (a.state(), a.host_state(), {k: list(v) for k, v in a.tables.items()}, dict(a.swapped))
        try:
            apply_ref(a, op)
        except RefAllocError:
            assert (a.state(), a.host_state(), {k: list(v) for k, v in a.tables.items()},
                    dict(a.swapped)) == state
        check_invariants(a)


def test_content_round_trip_is_bit_exact():
    """Swap a group out, let another sequence overwrite the released device
    blocks, swap the group back in: every swapped sequence attends to the
    same K/V as before (bit-identical decode output, fp16 storage)."""
    rng = np.random.default_rng(7)
    Hkv, D, nb, nh = 2, 64, 12, 12
    a = RefAllocator(nb, rng.permutation(nb), num_host_blocks=nh)
    dev = RefCache(nb, Hkv, D, "f16")
    host = RefCache(nh, Hkv, D, "f16")

    def write(sid, n):
        slots, cows = a.append_tokens(sid, n)
        dev.copy_blocks(cows)
        vals = rng.standard_normal((2, n, Hkv, D)).astype(np.float16)
        dev.append(vals[0], vals[1], np.array(slots))

    a.add_seq(0); write(0, 37)
    a.fork(0, 1); write(1, 5)
    a.add_seq(2); write(2, 20)

    def decode(sids):
        tables = [a.block_table(s)[0] for s in sids]
        lens = np.array([a.block_table(s)[1] for s in sids], dtype=np.int32)
        w = max(len(t) for t in tables)
        bt = np.array([t + [nb + 99] * (w - len(t)) for t in tables], dtype=np.int32)
        q = np.random.default_rng(3).standard_normal((len(sids), 4, D)).astype(np.float16)
        return paged_decode(q, dev.k, dev.v, bt, lens, 0.125, "f16")

    before = decode([0, 1])
    swap_blocks(host, dev, a.swap_out([0, 1]))
    write(2, 60)                     # takes (and overwrites) the released blocks
    swap_blocks(dev, host, a.swap_in([0, 1]))
    after = decode([0, 1])
    assert np.array_equal(before, after)
    # and a planted slip -- a swap-in that copies only K -- is caught
    swap_blocks(host, dev, a.swap_out([0, 1]))
    write(2, 16)
    pairs = a.swap_in([0, 1])
    for s, d in pairs:
        dev.k[d] = host.k[s]
    assert not np.array_equal(before, decode([0, 1]))


# ---- the library's allocator against the oracle's ------------------------
@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_365_b200 as m
    return m


def same(lib_a, ref):
    assert lib_a.state() == ref.state()
    assert lib_a.host_state() == ref.host_state()
    assert lib_a.num_seqs == len(ref.tables)
    assert lib_a.num_swapped == len(ref.swapped)
    for sid in ref.tables:
        assert lib_a.block_table(sid) == ref.block_table(sid)
    for sid in ref.swapped:
        assert lib_a.swapped_table(sid) == ref.swapped_table(sid)


@pytest.mark.parametrize("seed", range(8))
def test_library_swaps_match_oracle(pkv, seed):
    rng = np.random.default_rng(900 + seed)
    nb, nh = int(rng.integers(20, 80)), int(rng.integers(8, 80))
    order = rng.permutation(nb).astype(np.int32)
    lib_a = pkv.BlockAllocator(nb, order)
    lib_a.set_host_pool(nh)
    ref = RefAllocator(nb, order, num_host_blocks=nh)
    for op in random_ops(rng, 400):
        r_err = l_err = r_out = l_out = None
        try:
            r_out = apply_ref(ref, op)
        except RefAllocError as e:
            r_err = {"inval": 1, "nomem": 2}[e.kind]
        try:
            kind = op[0]
            if kind == "out":
                l_out = lib_a.swap_out(op[1])
            elif kind == "in":
                l_out = lib_a.swap_in(op[1])
            elif kind == "step":
                l_out = lib_a.step(op[1])
            elif kind == "append":
                l_out = lib_a.append_tokens(op[1], op[2])
            elif kind == "add":
                lib_a.add_seq(op[1])
            elif kind == "fork":
                lib_a.fork(op[1], op[2])
            else:
                lib_a.free_seq(op[1])
        except pkv.PkvError as e:
            l_err = e.status
        assert r_err == l_err, (op, r_err, l_err)
        if r_err is None and op[0] in ("out", "in"):
            assert [tuple(int(x) for x in p) for p in l_out] == r_out
        if r_err is None and op[0] in ("step", "append"):
            assert list(l_out[0]) == list(r_out[0])
            assert [tuple(p) for p in l_out[1]] == [tuple(p) for p in r_out[1]]
        same(lib_a, ref)


def test_library_swap_rejections(pkv):
    a = pkv.BlockAllocator(8)
    a.set_host_pool(2)
    a.add_seq(0)
    a.append_tokens(0, 40)
    with pytest.raises(pkv.PkvError) as e:
        a.swap_out([0])              # 3 blocks, 2 host blocks
    assert e.value.status == 2
    a.set_host_pool(4)               # allowed while nothing is swapped
    a.swap_out([0])
    with pytest.raises(pkv.PkvError):
        a.set_host_pool(8)           # not while a sequence is swapped
    with pytest.raises(pkv.PkvError):
        a.block_table(0)
    with pytest.raises(pkv.PkvError):
        a.step([0])
    with pytest.raises(pkv.PkvError):
        a.add_seq(0)
    a.swap_in([0])
    assert a.block_table(0)[1] == 40


@pytest.mark.parametrize("pairs,ok", [
    ([[0, 1], [2, 3]], True),
    ([[5, 1], [5, 3]], True),        # one source twice is fine
    ([[0, 1], [2, 1]], False),       # duplicate dst
    ([[9, 1]], False),               # src outside its pool
    ([[0, 4]], False),               # dst outside its pool
])
def test_swap_pairs_host_check(pkv, pairs, ok):
    p = np.array(pairs, dtype=np.int32).reshape(-1, 2)
    if ok:
        pkv.swap_blocks_check(p, 8, 4)
    else:
        with pytest.raises(pkv.PkvError):
            pkv.swap_blocks_check(p, 8, 4)
