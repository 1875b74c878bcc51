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


def test_library_partition_rule_and_workspace_sizes():
    """pkv_partition_tokens (the one copy of the auto rules, read by the
    binding and the bench) against the rules pkv.h states, and the workspace
    sizes that follow from it."""
    import paged_kv_cache_365_b200 as pkv
    from paged_kv_cache_365_b200 import _lib
    pt = pkv.partition_tokens
    for n in (1, 512, 4096):
        assert pt(_lib.OP_DECODE, n) == 512
        assert pt(_lib.OP_MULTI, n) == 2048
    for n in (4097, 16384, 131072):
        assert pt(_lib.OP_DECODE, n) == 1024
        assert pt(_lib.OP_MULTI, n) == 1024
    for n in (1, 4096):
        assert pt(_lib.OP_DECODE_FP8, n) == 768
    for n in (4097, 16384):
        assert pt(_lib.OP_DECODE_FP8, n) == 1024
    assert pt(_lib.OP_DECODE_FP8, 16385) == 2048
    # never more FP8 partitions than 16-bit ones (one workspace serves both)
    for n in (1, 700, 769, 1537, 4096, 4097, 9000, 16385, 131072):
        assert -(-n // pt(_lib.OP_DECODE_FP8, n)) <= -(-n // pt(_lib.OP_DECODE, n))
    # the tcgen05 multi-token kernel (more than 32 rows per kv-head, or an
    # FP8 pool): 8192 tokens at any length; up to 32 rows the rules above
    for n in (1, 4097, 131072):
        assert pt(_lib.OP_MULTI, n, rows=33) == 8192
        assert pt(_lib.OP_MULTI_FP8, n) == 8192
        assert pt(_lib.OP_MULTI, n, rows=32) == (2048 if n <= 4096 else 1024)
    assert pt(_lib.OP_MULTI, 9000, 48, rows=128) == 48
    # cascade suffix pass: longest suffix rounded up to a page, in [512, 2048]
    assert pt(_lib.OP_DECODE_PREFIX, 1024 + 100, 0, 64) == 512
    assert pt(_lib.OP_DECODE_PREFIX, 1024 + 600, 0, 64) == 608
    assert pt(_lib.OP_DECODE_PREFIX, 1024 + 5000, 0, 64) == 2048
    for op in (_lib.OP_DECODE, _lib.OP_DECODE_FP8, _lib.OP_MULTI):
        assert pt(op, 9000, 48) == 48          # an explicit partition is kept
        for bad in (8, 17, 4096):
            with pytest.raises(ValueError):
                pt(op, 9000, bad)
    with pytest.raises(ValueError):
        pt(_lib.OP_DECODE_PREFIX, 2000, 0, 0)   # the cascade needs a prefix
    with pytest.raises(ValueError):
        pt(7, 2000)
    # the workspaces follow the rule
    B, Hq, D = 3, 8, 128
    for n in (700, 3000, 5000, 9000):
        P = -(-n // pt(_lib.OP_DECODE, n))
        assert pkv.decode_workspace_bytes(B, Hq, D, n, 0) == (0 if P <= 1 else B * Hq * P * (D + 2) * 4)
        T = 7
        Pm = -(-n // pt(_lib.OP_MULTI, n))
        part = 0 if Pm <= 1 else -(-(T * Hq * Pm * D * 4) // 16) * 16 + T * Hq * Pm * 8
        # then the tcgen05 kernel's claim counter and work list
        want = -(-part // 16) * 16 + 16 + 2 * T * Pm * 8
        assert pkv.multi_workspace_bytes(T, Hq, D, n, 0) == want


def test_step_line_builds_the_contract_json():
    """step_line and the per_config entries from a timing record, without a
    GPU: the contract's keys, the roofline arithmetic, the e2e bytes."""
    import argparse
    import bench
    import workloads
    wl = workloads.named("llama7b", 0)
    r = dict(wl=wl, K=20, total_ms=20 * 0.18, e2e_ms=20 * 0.19, dec_avg_ms=0.175, roof_calls=2800,
             launches=60, h2d=1606400, d2h=524288, clocks={"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []},
             P=4, partition_tokens=512, n_pairs=0, cascade_pages=0, graph=False, cascade_overlap=False)
    args = argparse.Namespace(warmup=5, partition=0, seed=0, gpus=1, kv_fp8=False)
    line = bench.step_line(args, r, 1)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "clocks", "e2e", "gpu_launches", "roofline"):
        assert key in line, key
    assert line["config"]["workload"] == "llama7b" and "partition_tokens" not in line["config"]
    peak = bench.measured_peak()[0]
    dec = bench.decode_algorithmic_bytes(wl)
    assert abs(line["roofline"]["frac"] - dec / 0.175e-3 / 1e9 / peak) < 1e-12
    assert abs(line["value"] - bench.kv_bytes(wl, False) / 0.18e-3 / 1e9) < 1e-6
    e = bench.config_entry(args, r, 1)
    for key in ("us_per_step", "pct_hbm_peak", "roofline", "e2e", "clocks", "config"):
        assert key in e, key
    json.dumps(line)


def test_both_arms_quote_the_same_config():
    """The reference arm's config object is the one the CUDA arm prints."""
    import argparse
    import bench
    import workloads
    args = argparse.Namespace(seed=0, gpus=1)
    wl = workloads.named("tiny", 0)
    d = run("--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3")
    assert d["config"] == json.loads(json.dumps(bench.config_of(wl, args)))


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
