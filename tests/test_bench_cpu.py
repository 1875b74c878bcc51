"""bench.py's host side: the reference arm (the oracle on the host cores)
prints the contract's JSON line, for the decode step and the next rows."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


@pytest.mark.parametrize("row", ["step", "swap", "multi"])
def test_reference_arm_line(row):
    workload = "tiny" if row == "step" else "llama7b_compact"
    d = run("--impl", "reference", "--row", row, "--workload", workload, "--steps", "2", "--warmup", "3")
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "GB/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_warmup_floor():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                         text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0 and "warmup" in out.stderr


def test_bench_reports_the_library_auto_partitions():
    """bench.py names the partition the library picks for partition=0 (its
    own copy of the rule, so the reference arm needs no CUDA library)."""
    import bench
    import paged_kv_cache_365_b200 as pkv
    for n in (1, 512, 4096, 4097, 16384, 16385, 131072):
        assert bench.auto_partition(n, False) == pkv.api.auto_partition(n)
        assert bench.auto_partition(n, True) == pkv.api.auto_partition_fp8(n)
        assert bench.auto_partition(n, False, True) == pkv.api.auto_partition_multi(n)
    # the 16-bit rule is also the one the workspace size follows
    B, Hq, D = 3, 8, 128
    for n in (700, 3000, 5000, 9000):
        P = -(-n // pkv.api.auto_partition(n))
        assert pkv.decode_workspace_bytes(B, Hq, D, n, 0) == B * Hq * P * (D + 2) * 4
        # the multi-token path's workspace follows its own rule (T query rows)
        T = 7
        Pm = -(-n // pkv.api.auto_partition_multi(n))
        want = 0 if Pm <= 1 else -(-(T * Hq * Pm * D * 4) // 16) * 16 + T * Hq * Pm * 8
        assert pkv.multi_workspace_bytes(T, Hq, D, n, 0) == want


def test_multi_flops_and_roofline_choice():
    """The multi-token row's flop count against a brute-force count of
    (query, key) pairs, and the binding roofline picked by the longer of the
    memory and math times."""
    import bench
    lens, n_new, Hq, D = [5, 40, 3], 4, 2, 8
    pairs = 0
    for L in lens:
        n = min(n_new, L)
        for i in range(n):
            pos = L - n + i
            pairs += sum(1 for j in range(L) if j <= pos)
    assert bench.multi_useful_flops(lens, n_new, Hq, D) == pairs * Hq * D * 4
    r = bench.roofline_of(1e9, 1e12, 1e-3, 5000.0, 1000.0)   # 0.2 ms of bytes, 1 ms of math
    assert r["bound"] == "tensor" and abs(r["frac"] - 1.0) < 1e-12 and r["unit"] == "TFLOP/s"
    r = bench.roofline_of(1e9, 1e9, 4e-4, 5000.0, 1000.0)    # 0.2 ms of bytes, 1 us of math
    assert r["bound"] == "hbm" and abs(r["frac"] - 0.5) < 1e-12 and abs(r["achieved"] - 2500.0) < 1e-9


def test_multi_line_builds_the_contract_json():
    """multi_line (the multi-token row's JSON) from a timing record, without
    a GPU: the contract's keys and the roofline's fields."""
    import argparse
    import numpy as np
    import bench
    import workloads
    wl = workloads.named("tiny", 0)
    lens = wl.context_lens.astype(np.int64) + 4
    r = dict(wl=wl, K=10, T=5 * wl.B, kv=int(lens.sum()) * wl.kv_bytes_per_token, att_bytes=10 ** 6,
             total_ms=1.0, att_ms=0.8, e2e_ms=1.5, h2d=1000, d2h=2000, clocks={"sm_mhz": 1800.0}, P=1,
             launches=30, lens=lens)
    args = argparse.Namespace(warmup=3, partition=0, seed=0, gpus=1, new_tokens=5, no_cpu_baseline=True)
    d = bench.multi_line(args, r, 1)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "clocks", "e2e", "gpu_launches", "roofline"):
        assert key in d, key
    roof = d["roofline"]
    assert roof["bound"] in ("hbm", "tensor") and roof["frac"] > 0
    assert roof["useful_flops_per_launch"] == bench.multi_useful_flops(lens, 5, wl.Hq, wl.D)
    json.dumps(d)
