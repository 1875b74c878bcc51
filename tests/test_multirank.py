"""The N>1 path of the bench on CPU: two gloo ranks, each with its own
replica batch (no data-path collective), timings combined as the max over
ranks, whole-job throughput = all ranks' bytes / the slowest rank's time."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads
        from oracle import RefAllocator
        import paged_kv_cache_365_b200 as pkv
        wl = workloads.named("tiny", bench.replica_seed(0, rank))
        # the host half of a replica step: both allocators agree on its plan
        ref = RefAllocator(wl.num_blocks, wl.free_order)
        lib_a = pkv.BlockAllocator(wl.num_blocks, wl.free_order)
        for op in wl.ops:
            getattr(ref, {"add": "add_seq", "append": "append_tokens"}[op[0]])(*op[1:])
            getattr(lib_a, {"add": "add_seq", "append": "append_tokens"}[op[0]])(*op[1:])
        r_slots, _ = ref.step(list(wl.step_seqs))
        l_slots, _ = lib_a.step(list(wl.step_seqs))
        assert list(l_slots) == r_slots
        # per-rank timings: rank r is slower in the first entry
        mine = [1.0 + rank, 5.0 - rank]
        got = bench.max_over_ranks(mine, world, "cpu")
        q.put((rank, got, list(wl.free_order[:8]), r_slots))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = dict((r, (g, fo, sl)) for r, g, fo, sl in (q.get() for _ in range(world)))
    assert res[0][0] == res[1][0] == [2.0, 5.0]
    # distinct replicas: different seeds give different placements
    assert res[0][1] != res[1][1]


def test_job_throughput_counts_every_rank():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_throughput(1e9, 2, 10, 4.0) == pytest.approx(5.0)
    assert bench.job_throughput(1e9, 1, 10, 2.0) == pytest.approx(5.0)
