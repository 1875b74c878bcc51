"""PagedKVCache.run_step over many consecutive steps with host inputs and
host outputs: the staged path the end-to-end figure times.

run_step uploads a step's pinned host inputs on a side stream into one of
two device buffer sets (set i % 2) and downloads its output on another side
stream.  Two events keep the sets apart:

* ``computed[s]`` -- the upload of step i + 2 into set s waits until the
  kernels of step i, which read set s, have run.  Without it, step i + 2's
  q / k_new / v_new / tables would overwrite set s before step i's kernels
  read them, and step i's output would be attention with step i + 2's
  inputs;
* ``downloaded[s]`` -- the kernels of step i + 2 write set s's output buffer
  only after step i's download of it has finished.  Without it, step i's
  host output could receive step i + 2's result.

The test holds the compute stream back (a bounded spin kernel of ~0.1 s)
before the first step, so every step is enqueued while nothing has run:
the upload stream would then race ahead of the compute stream at once if
either wait were missing, and the outputs below would not match.  Each of
the steps has its own pinned inputs and its own pinned output; all of them
are compared with the fp64 oracle after the last download, and the pool is
compared token row by token row with the oracle's pool.  Plain and cascade
steps alternate, and a fork between steps brings copy-on-write copies back
into a later step.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}


def _draw(rng, shape, dtype):
    return workloads._to_storage(rng.standard_normal(shape).astype(np.float32), dtype)


def _pinned(arr, dtype):
    from paged_kv_cache_365_b200.replay import to_torch
    return to_torch(arr, dtype, "cpu").pin_memory()


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_consecutive_staged_steps_match_oracle(dtype):
    import paged_kv_cache_365_b200 as pkv
    from paged_kv_cache_365_b200.replay import to_torch
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    Hq, Hkv, D, NB = 8, 2, 128, 600
    scale = 1.0 / np.sqrt(D)
    rng = np.random.default_rng(77)
    free_order = rng.permutation(NB).astype(np.int32)
    cache = pkv.PagedKVCache(NB, Hkv, D, tdt, "cuda", free_order)
    ref_alloc = oracle.RefAllocator(NB, free_order)
    ref = oracle.RefCache(NB, Hkv, D, dtype)

    def prefill(sid, n):
        k, v = _draw(rng, (n, Hkv, D), dtype), _draw(rng, (n, Hkv, D), dtype)
        cache.prefill(sid, to_torch(k, dtype, "cuda"), to_torch(v, dtype, "cuda"))
        slots, pairs = ref_alloc.append_tokens(sid, n)
        ref.copy_blocks(pairs)
        ref.append_many(k, v, np.array(slots))

    # a root of 8 full pages + 5 tokens, forked into 6 sequences that grow
    # private suffixes: >= 4 sequences share >= 8 full pages (cascade)
    root = 100
    cache.add_seq(root)
    ref_alloc.add_seq(root)
    prefill(root, 8 * 16 + 5)
    ids = []
    for i in range(6):
        cache.fork(root, i)
        ref_alloc.fork(root, i)
        ids.append(i)
    cache.free_seq(root)
    ref_alloc.free_seq(root)
    for i in ids:
        if i % 2:
            prefill(i, int(rng.integers(1, 40)))   # odd ones leave the shared partial block
    # the first step copies every sequence still sharing the partial block

    n_steps = 8
    outs, wants = [], []
    hold = torch.cuda.current_stream()
    torch.cuda.synchronize()
    torch.cuda._sleep(200_000_000)  # hold the compute stream (~0.1 s): all steps enqueue before any runs
    for step in range(n_steps):
        if step == 4:  # a fork between steps: both siblings append into a shared partial block
            cache.fork(0, 6)
            ref_alloc.fork(0, 6)
            ids.append(6)
        slots, pairs, tables, lens = cache.plan_step(ids)
        r_slots, r_pairs = ref_alloc.step(ids)
        assert slots.tolist() == list(r_slots) and [tuple(p) for p in pairs.tolist()] == list(r_pairs)
        copies = pkv.cow_copy_rows(pairs, slots)
        q = _draw(rng, (len(ids), Hq, D), dtype)
        kn, vn = _draw(rng, (len(ids), Hkv, D), dtype), _draw(rng, (len(ids), Hkv, D), dtype)
        ref.copy_rows_then_append([tuple(int(x) for x in c) for c in copies], kn, vn, np.array(slots))
        r_tables = np.full((len(ids), tables.shape[1]), NB + 7, dtype=np.int32)
        r_lens = np.zeros(len(ids), dtype=np.int32)
        for b, sid in enumerate(ids):
            t, n = ref_alloc.block_table(sid)
            r_tables[b, :len(t)] = t
            r_lens[b] = n
        assert np.array_equal(lens, r_lens)
        wants.append(oracle.paged_decode(q, ref.k, ref.v, r_tables, r_lens, scale, dtype))
        cascade = step % 2 == 1
        pp = pkv.cascade_prefix_pages(tables, lens, tdt) if cascade else 0
        if cascade:
            assert pp >= 8
        out = torch.full((len(ids), Hq, D), float("nan"), dtype=tdt).pin_memory()
        outs.append(out)
        cache.run_step(torch.from_numpy(slots).pin_memory(), torch.from_numpy(copies).pin_memory(),
                       torch.from_numpy(np.ascontiguousarray(tables)).pin_memory(),
                       torch.from_numpy(lens).pin_memory(), int(lens.max()), _pinned(q, dtype), _pinned(kn, dtype),
                       _pinned(vn, dtype), out=out, scale=scale, stream=hold,
                       prefix_blocks=(torch.from_numpy(np.ascontiguousarray(tables[0, :pp])).pin_memory()
                                      if pp else None))
    cache.wait_downloads(hold)
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    for step, (out, want) in enumerate(zip(outs, wants)):
        err = float(np.abs(out.float().numpy().astype(np.float64) - want).max())
        assert err <= TOL[dtype], (step, err)
    # the pool: every token row of every sequence, bit for bit
    gk = cache.k.cpu().view(torch.int16).numpy()
    gv = cache.v.cpu().view(torch.int16).numpy()
    for sid in ids:
        t, n = ref_alloc.block_table(sid)
        tok = np.arange(n)
        blk, off = np.asarray(t)[tok // 16], tok % 16
        assert np.array_equal(gk[blk, :, off], ref.k[blk, :, off].view(np.int16))
        assert np.array_equal(gv[blk, :, off], ref.v[blk, :, off].view(np.int16))
