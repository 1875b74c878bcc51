"""Benchmark of the paged decode step: KV-cache GB/s (% of HBM peak),
sequence-steps/s and us per step.

One step = the whole device path for one batch: the copy-on-write block
copies (when the step has any), the slot-mapped append of the new tokens'
K/V, and paged decode attention (partition kernel, plus the merge kernel
when a sequence spans several partitions).  A plain 16-bit step is one
fused launch (pkv_decode_step) plus the merge; --unfused runs the append as
its own launch (the cascade always does).  The host allocator's step is
planned before the timed region (host microseconds, not device work); the
same planned step is replayed every iteration (its copies and appends are
idempotent).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
      (default: the JSON line is quoted on the long-context workload -- the
      largest single-GPU configuration -- and carries a ``per_config``
      object with the same figures for tiny, llama7b, gqa8b and prefix13b,
      each timed with the same --steps / --warmup)
  python bench.py --impl reference ...   (the fp64 CPU oracle, bounded sample)
  python bench.py --row swap ...         (preemption by swapping: one step =
      swap a quarter of the batch out to pinned host memory and back in;
      GB/s over the host link against cudaMemcpyAsync of the same bytes)
  python bench.py --row multi [--new-tokens N] ...  (one step = append N new
      tokens per sequence + causal attention of all of them over the paged
      context: a speculative-verification pass, N = drafted + 1)

N > 1: one process per GPU (torchrun), each rank decoding its own replica
batch (different seed), no collective on the data path; value = all ranks'
KV bytes / the slowest rank's time.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import gc
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "paged decode attention: KV-cache HBM GB/s (% of peak), seq-steps/s"
FP8_SCALE = 6.0 / 448.0  # --kv-fp8: one scale for K and V (448 = E4M3's largest value)
SWAP_METRIC = "block swap device<->pinned host (preempt + resume): GB/s over the host link"
MULTI_METRIC = ("paged multi-token attention (several new tokens per sequence, causal): KV-cache HBM GB/s "
                "(% of peak), query-tokens/s")
UNIT = "GB/s"
# the headline workload of the default run (the largest single-GPU
# configuration: 8 sequences of 32k-131k tokens, 2.2 GB of K/V a step) and
# the workloads reported beside it in ``per_config``
DEFAULT_WORKLOAD = "long"
PER_CONFIG = ["tiny", "llama7b", "gqa8b", "prefix13b"]
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1400.0
STORAGE = {"f32": 4, "f16": 2, "bf16": 2}
DTYPE_NAME = {"f32": "fp32", "f16": "fp16", "bf16": "bf16"}
# the decode kernels and their launch configuration: a committed ncu traffic
# figure counts only while these are unchanged
DECODE_SOURCES = ["paged_kv_cache_365_b200/csrc/decode.cuh", "paged_kv_cache_365_b200/csrc/decode_mma.cuh",
                  "paged_kv_cache_365_b200/csrc/decode_prefix.cuh", "paged_kv_cache_365_b200/csrc/common.cuh",
                  "paged_kv_cache_365_b200/csrc/decode_launch.cuh"]


# ---------------------------------------------------------------------------
# workload accounting (algorithmic bytes)
# ---------------------------------------------------------------------------
def kv_bytes(wl, unique: bool, fp8: bool = False) -> int:
    """K+V bytes the decode must read: each token once per kv-head.

    With ``unique`` a block shared by several sequences counts once (the
    shared prefix of the prefix workload); otherwise per sequence.  ``fp8``:
    the cache holds one-byte E4M3 codes instead of the workload's dtype.
    """
    per_tok = wl.kv_bytes_per_token // (STORAGE[wl.dtype] if fp8 else 1)
    logical = int(np.sum(wl.context_lens.astype(np.int64))) * per_tok
    if not unique or wl.name != "prefix13b":
        return logical
    prefix = 1024
    return logical - (wl.B - 1) * prefix * per_tok


def decode_algorithmic_bytes(wl, unique: bool = True, fp8: bool = False) -> int:
    """Bytes one decode launch must move: K/V + q in + out + tables + lengths."""
    es = STORAGE[wl.dtype]
    pages = int(np.sum((wl.context_lens.astype(np.int64) + 15) // 16))
    return kv_bytes(wl, unique, fp8) + 2 * wl.B * wl.Hq * wl.D * es + 4 * pages + 4 * wl.B


def source_digest() -> str:
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor-core TFLOP/s: the sustained figure (the kernels are
    timed inside a long step loop)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), "measured (MEASURED_PEAKS bf16_tflops_sustained)"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def multi_useful_flops(lens, n_new: int, Hq: int, D: int) -> int:
    """Flops of one multi-token attention call: new token i of a sequence of
    (post-append) length L sits at L - n + i and meets L - n + i + 1 keys; per
    key and head, q.k and p.v cost 2 D flops each."""
    keys = 0
    for L in np.asarray(lens, dtype=np.int64):
        n = min(int(n_new), int(L))
        keys += n * (int(L) - n) + n * (n + 1) // 2
    return keys * Hq * D * 4


def roofline_of(nbytes: float, flops: float, secs: float, hbm_gbs: float, tensor_tflops: float):
    """The binding roofline of a call: whichever of its bytes at the copy
    bandwidth and its flops at the tensor peak takes longer."""
    t_mem = nbytes / (hbm_gbs * 1e9)
    t_math = flops / (tensor_tflops * 1e12)
    if t_math > t_mem:
        return {"bound": "tensor", "achieved": flops / secs / 1e12, "peak": tensor_tflops, "unit": "TFLOP/s",
                "frac": t_math / secs}
    return {"bound": "hbm", "achieved": nbytes / secs / 1e9, "peak": hbm_gbs, "unit": "GB/s", "frac": t_mem / secs}


def recorded_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it
    was taken on the current decode source (else None)."""
    path = os.path.join(ROOT, "profiles", f"paged_decode_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    s = re.search(r"decode_source_digest:\s*([0-9a-f]+)", text)
    if not m or not s or s.group(1) != source_digest():
        return None
    return int(m.group(1))


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read-only)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = pynvml
            self.max_mhz = int(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.ok = True
        except Exception as e:  # pragma: no cover - reported in the JSON
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(int(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# ranks: every rank decodes its own replica batch; the job's time is the
# slowest rank's
# ---------------------------------------------------------------------------
def replica_seed(seed: int, rank: int) -> int:
    return seed + rank


def max_over_ranks(values, world, device):
    """Element-wise max of per-rank timings (the job ends with its slowest rank)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(bytes_per_rank_step, world, steps, max_total_s):
    """Whole-job GB/s: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_rank_step * steps / max_total_s / 1e9


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
def device_values(wl, seed, device):
    """Seeded synthetic N(0,1) values drawn on the device (fast at full size)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 7919 + 17)
    dt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[wl.dtype]
    shapes = {"q": (wl.B, wl.Hq, wl.D), "k_new": (wl.B, wl.Hkv, wl.D), "v_new": (wl.B, wl.Hkv, wl.D),
              "k_tokens": (wl.n_prefill_tokens, wl.Hkv, wl.D), "v_tokens": (wl.n_prefill_tokens, wl.Hkv, wl.D)}
    out = {}
    for k, shp in shapes.items():
        t = torch.empty(shp, dtype=dt, device=device)
        n = t.numel()
        flat = t.view(-1)
        chunk = 1 << 26
        for s in range(0, n, chunk):
            e = min(n, s + chunk)
            flat[s:e] = torch.randn(e - s, generator=g, device=device, dtype=torch.float32).to(dt)
        out[k] = t
    return out


ROOFLINE_LEG_S = 0.5  # least device time of the decode-call leg (several clock samples)


def run_cuda(args, rank, world, local_rank, workload=None, graph=None):
    """One workload's decode step: the timed K-step region, the decode call
    alone (event-bracketed, at least ROOFLINE_LEG_S of calls) and the same
    step end to end through PagedKVCache.run_step.  ``workload`` / ``graph``
    override args.workload / args.graph."""
    import torch
    from paged_kv_cache_365_b200.replay import build_step
    import paged_kv_cache_365_b200 as pkv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    use_graph = bool(args.graph if graph is None else graph)
    wl = workloads.named(workload or args.workload, replica_seed(args.seed, rank))
    vals = device_values(wl, replica_seed(args.seed, rank), dev)
    st = build_step(wl, {}, dev, device_values=vals)
    del vals
    cache = st["cache"]
    stream = torch.cuda.current_stream(dev)
    B, Hq, D = wl.B, wl.Hq, wl.D
    max_ctx = st["max_context_len"]
    n_pairs = int(st["cow_pairs"].shape[0])
    ws = cache.workspace(pkv.decode_workspace_bytes(B, Hq, D, max_ctx, args.partition))
    out = torch.empty_like(st["q"])
    part_tokens = pkv.partition_tokens(pkv._lib.OP_DECODE_FP8 if args.kv_fp8 else pkv._lib.OP_DECODE, max_ctx,
                                       args.partition)
    P = max(1, math.ceil(max_ctx / part_tokens))
    scale = 1.0 / math.sqrt(D)
    # a batch that shares leading blocks is decoded with the cascade (the
    # shared prefix is read once per kv-head) when the library says so
    pp = pkv.cascade_prefix_pages(st["host"]["block_tables"], st["host"]["context_lens"], cache.dtype)
    use_cascade = pp > 0 and not args.no_cascade
    if use_cascade:
        part_tokens = pkv.partition_tokens(pkv._lib.OP_DECODE_PREFIX, max_ctx, args.partition, pp)
    fp8 = bool(args.kv_fp8)
    if fp8:
        if wl.dtype == "f32":
            raise SystemExit("--kv-fp8 needs an fp16 / bf16 workload")
        to_fp8_pool(cache, dev)
    prefix = torch.from_numpy(np.ascontiguousarray(st["host"]["block_tables"][0, :pp])).to(dev) if use_cascade else None
    # the step through pkv_decode_step (pkv_decode_step_fp8 over an FP8
    # pool): a plain step is one launch (+ merge); the cascade keeps its
    # copies and append in a launch of their own, which it overlaps (it waits
    # for it only at each sequence's last page)
    fused_step = wl.dtype != "f32" and not args.unfused and not args.cascade_overlap
    if use_cascade and fp8:
        # the FP8 cascade: the prefix widened to 16 bits, the prefix pass,
        # the suffix pass beside it (making the step's copies and append when
        # fused), the merge
        if args.cascade_overlap:
            raise SystemExit("--cascade-overlap takes a 16-bit pool")
        ws = cache.workspace(pkv.decode_prefix_fp8_workspace_bytes(B, Hq, wl.Hkv, D, max_ctx, pp, args.partition))
        launches_per_step = (0 if fused_step else (1 if n_pairs else 0) + 1) + 4
    elif use_cascade:
        ws = cache.workspace(pkv.decode_prefix_workspace_bytes(B, Hq, D, max_ctx, pp, args.partition))
        # copies + append (one launch), cascade (one launch, or prefix + suffix passes), merge
        launches_per_step = 1 + (3 if args.cascade_overlap else 2)
    else:
        launches_per_step = ((0 if fused_step else 1) + 1 + (1 if (n_pairs and fp8 and not fused_step) else 0) +
                             (1 if P > 1 else 0))

    # every call goes to the current stream at call time (so that a CUDA
    # graph capture records it)
    # the step's copy-on-write copies cut to the rows that hold tokens, in
    # one launch with the append (16-bit pools)
    copies_host = pkv.cow_copy_rows(st["host"]["cow_pairs"], st["host"]["step_slots"])
    copies = torch.from_numpy(copies_host).to(dev)

    def pre_decode():
        if fp8:
            if n_pairs:
                pkv.copy_blocks(cache.k, cache.v, st["cow_pairs"])
            pkv.kv_append_fp8(st["k_new"], st["v_new"], cache.k, cache.v, st["slot_mapping"], FP8_SCALE, FP8_SCALE)
        elif n_pairs:
            pkv.kv_append_copy(st["k_new"], st["v_new"], cache.k, cache.v, st["slot_mapping"], copies)
        else:
            pkv.kv_append(st["k_new"], st["v_new"], cache.k, cache.v, st["slot_mapping"])

    side = torch.cuda.Stream(dev) if use_cascade else None
    fork, join = torch.cuda.Event(), torch.cuda.Event()
    overlap = use_cascade and args.cascade_overlap

    def cascade(phase, s):
        pkv.paged_attention_decode_prefix(st["q"], cache.k, cache.v, st["block_tables"], st["context_lens"],
                                          max_ctx, prefix, scale, out=out, workspace=ws, partition=args.partition,
                                          stream=s, phase=phase)

    def overlapped(pre):
        # the prefix pass (q and the shared, full prefix blocks only) on a
        # second stream beside the step's copies and append
        cur = torch.cuda.current_stream(dev)
        fork.record(cur)
        side.wait_event(fork)
        with torch.cuda.stream(side):
            cascade(0, side)
            join.record(side)
        if pre:
            pre_decode()
        cascade(1, cur)
        cur.wait_event(join)
        cascade(2, cur)

    def decode():
        if overlap:
            overlapped(False)
            return
        if fp8 and use_cascade:
            pkv.paged_attention_decode_prefix_fp8(st["q"], cache.k, cache.v, st["block_tables"], st["context_lens"],
                                                  max_ctx, prefix, scale, FP8_SCALE, FP8_SCALE, out=out, workspace=ws,
                                                  partition=args.partition)
        elif fp8:
            pkv.paged_attention_decode_fp8(st["q"], cache.k, cache.v, st["block_tables"], st["context_lens"],
                                           max_ctx, scale, FP8_SCALE, FP8_SCALE, out=out, workspace=ws,
                                           partition=args.partition)
        elif use_cascade:
            pkv.paged_attention_decode_prefix(st["q"], cache.k, cache.v, st["block_tables"], st["context_lens"],
                                              max_ctx, prefix, scale, out=out, workspace=ws,
                                              partition=args.partition)
        else:
            pkv.paged_attention_decode(st["q"], cache.k, cache.v, st["block_tables"], st["context_lens"], max_ctx,
                                       scale, out=out, workspace=ws, partition=args.partition)

    fused = fused_step

    def eager_step():
        if overlap:
            overlapped(True)
            return
        if fused and fp8:
            pkv.decode_step_fp8(st["q"], cache.k, cache.v, st["k_new"], st["v_new"], st["slot_mapping"],
                                copies if n_pairs else None, st["block_tables"], st["context_lens"], max_ctx, scale,
                                FP8_SCALE, FP8_SCALE, prefix_blocks=prefix if use_cascade else None, out=out,
                                workspace=ws, partition=args.partition)
            return
        if fused:
            pkv.decode_step(st["q"], cache.k, cache.v, st["k_new"], st["v_new"], st["slot_mapping"],
                            copies if n_pairs else None, st["block_tables"], st["context_lens"], max_ctx, scale,
                            prefix_blocks=prefix if use_cascade else None, out=out, workspace=ws,
                            partition=args.partition)
            return
        pre_decode()
        decode()

    run_step = eager_step
    if use_graph:
        # one whole step captured once, replayed every iteration
        for _ in range(3):
            eager_step()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            eager_step()
        torch.cuda.synchronize()
        run_step = graph.replay

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    if pkv.get_error() != 0:
        raise RuntimeError("device error flags raised during warm-up")
    barrier()
    torch.cuda.synchronize()

    K = args.steps
    with ClockSampler(local_rank) as clocks:
        # (1) the step, K times back to back: events only around the whole
        #     run (an event between two kernels would break their overlap)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(K):
            run_step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        total_ms = t0.elapsed_time(t1)
        # (2) the decode call alone, each launch bracketed by events
        #     (roofline), for at least ROOFLINE_LEG_S of device time; every
        #     rank makes the same number of calls
        n_roof = max(K, int(math.ceil(ROOFLINE_LEG_S * 1e3 / max(total_ms / K, 1e-3))))
        n_roof = int(max_over_ranks([n_roof], world, dev)[0])
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_roof)]
        for i in range(n_roof):
            ev[i][0].record(stream)
            decode()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    dec_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(n_roof)]
    dec_avg_ms = sum(dec_ms) / n_roof
    barrier()

    # e2e: the same step with its inputs in pinned host memory, copied in
    # every step, and the output read back every step
    host = {k: st[k].cpu().pin_memory() for k in ("q", "k_new", "v_new", "slot_mapping", "cow_pairs",
                                                    "block_tables", "context_lens")}
    if n_pairs and (fused_step or not fp8):
        host["cow_pairs"] = torch.from_numpy(copies_host).pin_memory()
    if use_cascade:
        host["prefix_blocks"] = prefix.cpu().pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()

    def e2e_step():
        cache.run_step(host["slot_mapping"], host["cow_pairs"], host["block_tables"], host["context_lens"],
                       max_ctx, host["q"], host["k_new"], host["v_new"], out=out_host, scale=scale,
                       partition=args.partition, stream=stream, prefix_blocks=host.get("prefix_blocks"))

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cache.staging_after(stream)   # the first upload starts after e0
    for _ in range(K):
        e2e_step()
    cache.wait_downloads(stream)  # the last download ends before e1
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    if pkv.get_error() != 0:
        raise RuntimeError("device error flags raised during timing")

    total_ms, e2e_ms, dec_avg_ms = max_over_ranks([total_ms, e2e_ms, dec_avg_ms], world, dev)

    res = dict(wl=wl, K=K, total_ms=total_ms, e2e_ms=e2e_ms, dec_avg_ms=dec_avg_ms, roof_calls=n_roof,
               launches=launches_per_step * K, h2d=h2d, d2h=d2h, clocks=clocks.summary(), P=P,
               partition_tokens=part_tokens, n_pairs=n_pairs, cascade_pages=pp if use_cascade else 0,
               graph=use_graph, cascade_overlap=bool(use_cascade and args.cascade_overlap), fused=fused)
    return res


# ---------------------------------------------------------------------------
# several new tokens per sequence (speculative verification)
# ---------------------------------------------------------------------------
def to_fp8_pool(cache, dev):
    """The cache's pool quantised once to E4M3 codes (one scale for K, one
    for V, covering ~6 standard deviations of the N(0,1) values); the 16-bit
    pool is released."""
    import torch
    import paged_kv_cache_365_b200 as pkv
    NB, Hkv, D = cache.k.shape[0], cache.k.shape[1], cache.k.shape[3]
    k8 = torch.empty(cache.k.shape, dtype=torch.uint8, device=dev)
    v8 = torch.empty(cache.v.shape, dtype=torch.uint8, device=dev)
    all_slots = torch.arange(NB * 16, dtype=torch.int64, device=dev)
    for src, dst in ((cache.k, k8), (cache.v, v8)):
        rows = src.permute(0, 2, 1, 3).reshape(NB * 16, Hkv, D).contiguous()
        pkv.kv_append_fp8(rows, rows, dst, dst, all_slots, FP8_SCALE, FP8_SCALE)
        del rows
    cache.k, cache.v = k8, v8
    cache.fp8 = (FP8_SCALE, FP8_SCALE)
    torch.cuda.synchronize()


def run_multi(args, rank, world, local_rank):
    import torch
    from paged_kv_cache_365_b200.replay import build_multi_step
    import paged_kv_cache_365_b200 as pkv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = workloads.named(args.workload, replica_seed(args.seed, rank))
    if wl.dtype == "f32":
        raise SystemExit("--row multi needs an fp16 / bf16 workload")
    vals = device_values(wl, replica_seed(args.seed, rank), dev)
    st = build_multi_step(wl, args.new_tokens, dev, device_values=vals, seed=replica_seed(args.seed, rank))
    del vals
    cache = st["cache"]
    fp8 = bool(args.kv_fp8)
    if fp8:
        to_fp8_pool(cache, dev)
    stream = torch.cuda.current_stream(dev)
    lens = st["host"]["context_lens"]
    T = int(st["q"].shape[0])
    max_ctx, max_q = st["max_context_len"], st["max_query_len"]
    ws = cache.workspace(pkv.multi_workspace_bytes(T, wl.Hq, wl.D, max_ctx, args.partition))
    out = torch.empty_like(st["q"])
    scale = 1.0 / math.sqrt(wl.D)
    n_pairs = int(st["cow_pairs"].shape[0])
    part_tokens = pkv.partition_tokens(pkv._lib.OP_MULTI_FP8 if fp8 else pkv._lib.OP_MULTI, max_ctx, args.partition,
                                       rows=max_q * wl.Hq // wl.Hkv)
    P = max(1, math.ceil(max_ctx / part_tokens))

    def pre():
        if n_pairs:
            pkv.copy_blocks(cache.k, cache.v, st["cow_pairs"])
        if fp8:
            pkv.kv_append_fp8(st["k_new"], st["v_new"], cache.k, cache.v, st["slot_mapping"], FP8_SCALE, FP8_SCALE)
        else:
            pkv.kv_append(st["k_new"], st["v_new"], cache.k, cache.v, st["slot_mapping"])

    def attend():
        if fp8:
            pkv.paged_attention_multi_fp8(st["q"], cache.k, cache.v, st["block_tables"], st["context_lens"],
                                          st["query_start"], max_ctx, max_q, scale, FP8_SCALE, FP8_SCALE, out=out,
                                          workspace=ws, partition=args.partition)
        else:
            pkv.paged_attention_multi(st["q"], cache.k, cache.v, st["block_tables"], st["context_lens"],
                                      st["query_start"], max_ctx, max_q, scale, out=out, workspace=ws,
                                      partition=args.partition)

    def step():
        pre()
        attend()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if pkv.get_error() != 0:
        raise RuntimeError("device error flags raised during warm-up")
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        t0.record(stream)
        for _ in range(K):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    total_ms = t0.elapsed_time(t1)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for i in range(K):
        ev[i][0].record(stream)
        attend()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    att_ms = sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(K)) / K
    # e2e: inputs from pinned host memory every step, output read back
    host = {k: st[k].cpu().pin_memory() for k in ("q", "k_new", "v_new", "slot_mapping", "cow_pairs",
                                                    "block_tables", "context_lens", "query_start")}
    out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()

    def e2e_step():
        cache.run_multi_step(host["slot_mapping"], host["cow_pairs"], host["block_tables"], host["context_lens"],
                             max_ctx, host["query_start"], max_q, host["q"], host["k_new"], host["v_new"],
                             out=out_host, scale=scale, partition=args.partition, stream=stream)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cache.staging_after(stream)   # the first upload starts after e0
    for _ in range(K):
        e2e_step()
    cache.wait_downloads(stream)  # the last download ends before e1
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if pkv.get_error() != 0:
        raise RuntimeError("device error flags raised during timing")
    total_ms, att_ms, e2e_ms = max_over_ranks([total_ms, att_ms, e2e_ms], world, dev)
    es = STORAGE[wl.dtype]
    kv = int(np.asarray(lens, dtype=np.int64).sum()) * wl.Hkv * wl.D * 2 * (1 if fp8 else es)
    att_bytes = kv + 2 * T * wl.Hq * wl.D * es + int(sum(-(-int(n) // 16) for n in lens)) * 4 + 8 * wl.B + 4
    # the tcgen05 kernel (more than 32 rows per kv-head, or an FP8 pool) adds
    # its one-CTA plan kernel
    tc = fp8 or max_q * wl.Hq // wl.Hkv > 32
    launches = (1 + (1 if n_pairs else 0) + (2 if tc else 1) + (1 if P > 1 else 0)) * K
    return dict(wl=wl, K=K, T=T, kv=kv, att_bytes=att_bytes, total_ms=total_ms, att_ms=att_ms, e2e_ms=e2e_ms, tc=tc,
                h2d=h2d, d2h=d2h, clocks=clocks.summary(), P=P, launches=launches, lens=lens,
                partition_tokens=part_tokens)


def multi_cpu_baseline(wl, n_new, budget_s=10.0, seed=0):
    """The oracle's multi-token attention, one thread, on sampled sequences
    of the same workload (n_new new tokens each, the last of the context)."""
    import oracle
    limits = blas_threads()
    ctx = limits(limits=1) if limits else None
    if ctx:
        ctx.__enter__()
    try:
        vals, ref = oracle_setup(wl)
        rng = np.random.default_rng(seed)
        order = rng.permutation(wl.B)
        es = STORAGE[wl.dtype]
        secs, nbytes, done = 0.0, 0, 0
        for b in order:
            qs = np.array([0, n_new], dtype=np.int32)
            qrows = workloads._to_storage(rng.standard_normal((n_new, wl.Hq, wl.D)).astype(np.float32), wl.dtype)
            t0 = time.perf_counter()
            oracle.paged_multi(qrows, ref["cache"].k, ref["cache"].v, ref["block_tables"][b:b + 1],
                               ref["context_lens"][b:b + 1], qs, wl.scale, wl.dtype)
            secs += time.perf_counter() - t0
            nbytes += int(ref["context_lens"][b]) * wl.Hkv * wl.D * 2 * es
            done += 1
            if secs >= budget_s:
                break
    finally:
        if ctx:
            ctx.__exit__(None, None, None)
    return {"value": nbytes / secs / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{done} sequences of workload {wl.name} seed {wl.seed}, {n_new} new tokens each, "
                      f"{nbytes / 1e6:.1f} MB of K/V, fp64 numpy, BLAS limited to 1 thread, {secs:.1f} s"}


def multi_line(args, r, world):
    wl = r["wl"]
    K = r["K"]
    peak, peak_kind = measured_peak()
    tpeak, tpeak_kind = measured_tensor_peak()
    step_s = r["total_ms"] / 1e3 / K
    flops = multi_useful_flops(r["lens"], args.new_tokens, wl.Hq, wl.D)
    roof = roofline_of(r["att_bytes"], flops, r["att_ms"] / 1e3, peak, tpeak)
    line = {
        "metric": MULTI_METRIC, "value": job_throughput(r["kv"], world, K, r["total_ms"] / 1e3), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": r["total_ms"] / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded N(0,1) q/K/V on the device, seeded lengths and placement)",
        "config": {"workload": f"{wl.name} + {args.new_tokens} new tokens per sequence", "global_batch": wl.B,
                   "new_tokens": args.new_tokens, "query_tokens": r["T"], "num_q_heads": wl.Hq,
                   "num_kv_heads": wl.Hkv, "head_dim": wl.D, "block_size": 16,
                   "context_lens": {"min": int(np.min(r["lens"])), "max": int(np.max(r["lens"])),
                                    "sum": int(np.sum(r["lens"]))},
                   "seed": args.seed,
                   "parallelism": f"replicas{args.gpus}" if args.gpus > 1 else "single-gpu",
                   "l2": "inputs larger than L2 (no flush)" if r["kv"] > 126e6 else "inputs fit in L2"},
        "us_per_step": 1e3 * r["total_ms"] / K,
        "query_tokens_per_s": world * r["T"] / step_s,
        "pct_hbm_peak": 100.0 * (r["kv"] / step_s / 1e9) / peak,
        "clocks": r["clocks"],
        "e2e": {"value": job_throughput(r["kv"], world, K, r["e2e_ms"] / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "us_per_step": 1e3 * r["e2e_ms"] / K},
        "gpu_launches": r["launches"],
        "launch": {"partition_tokens": r.get("partition_tokens"), "partition_auto": not args.partition,
                   "partitions_max": r["P"]},
        "roofline": {"kernel": ("paged_multi_tc (plan + persistent tcgen05 kernel" if r.get("tc") else
                                "paged_multi (partition kernel") + (" + merge)" if r["P"] > 1 else ")"), **roof,
                     "peak_kind": (tpeak_kind if roof["bound"] == "tensor" else
                                   f"{peak_kind} (MEASURED_PEAKS hbm_gbs)" if peak_kind == "measured" else "fallback"),
                     "traffic": None, "algorithmic_bytes_per_launch": r["att_bytes"],
                     "useful_flops_per_launch": flops, "avg_launch_us": 1e3 * r["att_ms"]},
    }
    fp8 = bool(getattr(args, "kv_fp8", False))
    if fp8:
        line["config"]["kv_cache"] = "e4m3 (FP8) codes, scale %.6g for K and V" % FP8_SCALE
        line["roofline"]["kernel"] = line["roofline"]["kernel"].replace("paged_multi_tc", "paged_multi_fp8", 1)
    if world == 1 and not args.no_cpu_baseline and not fp8:
        line["cpu_baseline"] = multi_cpu_baseline(wl, args.new_tokens, seed=args.seed)
    return line


# ---------------------------------------------------------------------------
# preemption by swapping: a quarter of the batch out to pinned host memory
# and back in
# ---------------------------------------------------------------------------
def swap_plan(wl):
    """Sequences a swap step preempts: the first quarter of the step batch."""
    ids = [int(s) for s in wl.step_seqs]
    return ids[:max(1, len(ids) // 4)]


def run_swap(args, rank, world, local_rank):
    import torch
    from paged_kv_cache_365_b200.replay import build_step
    import paged_kv_cache_365_b200 as pkv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = workloads.named(args.workload, replica_seed(args.seed, rank))
    vals = device_values(wl, replica_seed(args.seed, rank), dev)
    st = build_step(wl, {}, dev, device_values=vals)
    del vals
    cache = st["cache"]
    stream = torch.cuda.current_stream(dev)
    ids = swap_plan(wl)
    n_host = sum(len(cache.alloc.block_table(s)[0]) for s in ids)
    cache.enable_swap(n_host)
    # one preempt/resume cycle planned on the host; its copies replayed
    out_pairs = cache.alloc.swap_out(ids)
    in_pairs = cache.alloc.swap_in(ids)
    d_out = torch.from_numpy(np.ascontiguousarray(out_pairs)).to(dev)
    d_in = torch.from_numpy(np.ascontiguousarray(in_pairs)).to(dev)
    es = STORAGE[wl.dtype]
    block_bytes = 2 * wl.Hkv * 16 * wl.D * es  # K and V
    out_bytes, in_bytes = len(out_pairs) * block_bytes, len(in_pairs) * block_bytes

    def swap_out():
        pkv.swap_blocks(cache.host_k, cache.host_v, cache.k, cache.v, d_out, stream, dev)

    def swap_in():
        pkv.swap_blocks(cache.k, cache.v, cache.host_k, cache.host_v, d_in, stream, dev)

    # the copy engine over the same link and bytes: cudaMemcpyAsync of one
    # contiguous pinned buffer each way (the roofline's denominator)
    dbuf = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
    hbuf = torch.empty(out_bytes, dtype=torch.uint8, pin_memory=True)

    def timed(fn, K):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    K = args.steps
    with ClockSampler(local_rank) as clocks:
        total_ms = timed(lambda: (swap_out(), swap_in()), K)
    out_ms = timed(swap_out, K)
    in_ms = timed(swap_in, K)
    ce_d2h_ms = timed(lambda: hbuf.copy_(dbuf, non_blocking=True), K)
    ce_h2d_ms = timed(lambda: dbuf.copy_(hbuf, non_blocking=True), K)
    if pkv.get_error() != 0:
        raise RuntimeError("device error flags raised during the swap timing")
    # end to end through the public API: allocator plan + pairs upload +
    # copies, every step (alternating device blocks, all valid)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        cache.swap_out(ids, stream)
        cache.swap_in(ids, stream)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(K):
        cache.swap_out(ids, stream)
        cache.swap_in(ids, stream)
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = t0.elapsed_time(t1)
    total_ms, out_ms, in_ms, ce_d2h_ms, ce_h2d_ms, e2e_ms = max_over_ranks(
        [total_ms, out_ms, in_ms, ce_d2h_ms, ce_h2d_ms, e2e_ms], world, dev)
    return dict(wl=wl, K=K, ids=ids, out_bytes=out_bytes, in_bytes=in_bytes, total_ms=total_ms, out_ms=out_ms,
                in_ms=in_ms, ce_d2h_ms=ce_d2h_ms, ce_h2d_ms=ce_h2d_ms, e2e_ms=e2e_ms, clocks=clocks.summary(),
                n_pairs=(len(out_pairs), len(in_pairs)), block_bytes=block_bytes)


def swap_cpu_baseline(wl, budget_s=3.0):
    """The oracle's swap_blocks (numpy block copies) on a bounded sample."""
    import oracle
    n = 64
    dev = oracle.RefCache(n, wl.Hkv, wl.D, wl.dtype)
    host = oracle.RefCache(n, wl.Hkv, wl.D, wl.dtype)
    pairs = [(i, (i * 7) % n) for i in range(n)]
    block_bytes = 2 * wl.Hkv * 16 * wl.D * STORAGE[wl.dtype]
    reps, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        oracle.swap_blocks(host, dev, pairs)
        reps += 1
    secs = time.perf_counter() - t0
    return {"value": reps * n * block_bytes / secs / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{reps} x {n} blocks of workload {wl.name}'s shape copied between two numpy pools, "
                      f"one thread, {secs:.1f} s"}


def swap_line(args, r, world):
    wl = r["wl"]
    K = r["K"]
    step_bytes = r["out_bytes"] + r["in_bytes"]
    gbs = lambda b, ms: b * K / (ms / 1e3) / 1e9  # noqa: E731
    # the memcpy buffers hold out_bytes; scale the inbound copy to in_bytes
    ce_ms = r["ce_d2h_ms"] + r["ce_h2d_ms"] * r["in_bytes"] / max(1, r["out_bytes"])
    achieved = gbs(step_bytes, r["out_ms"] + r["in_ms"])
    peak = gbs(step_bytes, ce_ms)
    line = {
        "metric": SWAP_METRIC, "value": world * gbs(step_bytes, r["total_ms"]), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": r["total_ms"] / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded N(0,1) K/V on the device, seeded lengths and placement)",
        "config": {"workload": f"{wl.name} preempt+resume", "swapped_seqs": len(r["ids"]),
                   "blocks_out": r["n_pairs"][0], "blocks_in": r["n_pairs"][1], "block_bytes_kv": r["block_bytes"],
                   "bytes_per_step": step_bytes, "num_kv_heads": wl.Hkv, "head_dim": wl.D, "seed": args.seed,
                   "parallelism": f"replicas{args.gpus}" if args.gpus > 1 else "single-gpu",
                   "l2": "device side larger than L2 (no flush)" if r["out_bytes"] > 126e6 else "fits in L2"},
        "swap_out_gbs": gbs(r["out_bytes"], r["out_ms"]), "swap_in_gbs": gbs(r["in_bytes"], r["in_ms"]),
        "memcpy_d2h_gbs": gbs(r["out_bytes"], r["ce_d2h_ms"]), "memcpy_h2d_gbs": gbs(r["out_bytes"], r["ce_h2d_ms"]),
        "clocks": r["clocks"],
        "e2e": {"value": world * gbs(step_bytes, r["e2e_ms"]), "unit": UNIT,
                "h2d_bytes_per_step": r["in_bytes"] + 8 * sum(r["n_pairs"]),
                "d2h_bytes_per_step": r["out_bytes"], "us_per_step": 1e3 * r["e2e_ms"] / K},
        "gpu_launches": 2 * K,
        "roofline": {"kernel": "swap_blocks_kernel (out + in)", "bound": "host link", "achieved": achieved,
                     "peak": peak, "peak_kind": "cudaMemcpyAsync of the same bytes each way, this run",
                     "unit": "GB/s", "frac": achieved / peak, "traffic": None,
                     "algorithmic_bytes_per_launch": step_bytes / 2, "avg_launch_us": 1e3 * (r["out_ms"] + r["in_ms"]) / (2 * K)},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = swap_cpu_baseline(wl)
    return line


# ---------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------
def oracle_units_timed(wl, ref, vals, units):
    """Time the oracle on a list of (sequence, kv-head) units; return
    (seconds, KV bytes the units read)."""
    import oracle
    G = wl.Hq // wl.Hkv
    t0 = time.perf_counter()
    nbytes = 0
    for b, g in units:
        n = int(ref["context_lens"][b])
        pages = -(-n // 16)
        tbl = ref["block_tables"][b, :pages].astype(np.int64)
        keys = oracle.widen(ref["cache"].k[tbl, g].reshape(-1, wl.D)[:n], wl.dtype)
        values = oracle.widen(ref["cache"].v[tbl, g].reshape(-1, wl.D)[:n], wl.dtype)
        qb = oracle.widen(vals["q"][b], wl.dtype)
        for h in range(g * G, (g + 1) * G):
            oracle.decode_head(qb[h], keys, values, wl.scale)
        nbytes += 2 * n * wl.D * STORAGE[wl.dtype]
    return time.perf_counter() - t0, nbytes


def oracle_setup(wl):
    import oracle
    vals = workloads.draw_values(wl)
    ref = oracle.replay(wl, vals)
    return vals, ref


def pick_units(wl, rng, budget_s, per_byte_s):
    """Random (sequence, kv-head) units whose estimated oracle time fills
    ``budget_s`` (the whole workload, repeated, when it is smaller)."""
    units, est = [], 0.0
    cand = [(b, g) for b in range(wl.B) for g in range(wl.Hkv) if wl.context_lens[b] > 0]
    while est < budget_s:
        added = False
        for i in rng.permutation(len(cand)):
            b, g = cand[i]
            cost = 2 * int(wl.context_lens[b]) * wl.D * STORAGE[wl.dtype] * per_byte_s
            if units and est + cost > budget_s:
                continue
            units.append((b, g))
            est += cost
            added = True
            if est >= budget_s:
                break
        if not added:
            break
    return units


def calibrate(wl, ref, vals):
    b = int(np.argmax(wl.context_lens))
    s, nb = oracle_units_timed(wl, ref, vals, [(b, 0)])
    return s / max(nb, 1)


def blas_threads():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits
    except Exception:  # pragma: no cover
        return None


def cpu_baseline(wl, budget_s=12.0, seed=0):
    """The oracle as it stands, one host thread, on a bounded sample."""
    limits = blas_threads()
    ctx = limits(limits=1) if limits else None
    if ctx:
        ctx.__enter__()
    try:
        vals, ref = oracle_setup(wl)
        per_byte = calibrate(wl, ref, vals)
        units = pick_units(wl, np.random.default_rng(seed), budget_s, per_byte)
        secs, nbytes = oracle_units_timed(wl, ref, vals, units)
    finally:
        if ctx:
            ctx.__exit__(None, None, None)
    return {"value": nbytes / secs / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{len(units)} (sequence, kv-head) units of workload {wl.name} seed {wl.seed}, "
                      f"{nbytes / 1e6:.1f} MB of K/V, fp64 numpy, BLAS limited to 1 thread, {secs:.1f} s"}


def config_of(wl, args):
    """The workload the line is quoted on (the same object on both arms)."""
    return {"workload": wl.name, "global_batch": wl.B, "num_q_heads": wl.Hq, "num_kv_heads": wl.Hkv,
            "head_dim": wl.D, "block_size": 16, "num_blocks": wl.num_blocks,
            "context_lens": {"min": int(wl.context_lens.min()), "max": int(wl.context_lens.max()),
                             "sum": int(wl.context_lens.astype(np.int64).sum())},
            "seed": args.seed,
            "parallelism": f"replicas{args.gpus}" if args.gpus > 1 else "single-gpu",
            "l2": "inputs larger than L2 (no flush)" if kv_bytes(wl, True) > 126e6 else "inputs fit in L2"}


def launch_of(args, r):
    """How the CUDA path ran the workload (partition, graph, cascade)."""
    return {"partition_tokens": r["partition_tokens"], "partition_auto": not args.partition,
            "partitions_max": r["P"], "cuda_graph": r["graph"], "fused_step": r.get("fused", False),
            "cascade": None if not r["cascade_pages"] else
            ("prefix pass on a second stream beside copies + append" if r["cascade_overlap"] else "one launch")}


def run_reference(args, rank, world):
    """The oracle timed on the host cores, every step a bounded sample."""
    if rank != 0:
        return
    wl = workloads.named(args.workload or DEFAULT_WORKLOAD, args.seed)
    if getattr(args, "row", "step") == "multi":
        b = multi_cpu_baseline(wl, args.new_tokens, budget_s=min(60.0, 0.5 * (args.steps + args.warmup)),
                               seed=args.seed)
        print(json.dumps({"impl": "reference", "metric": MULTI_METRIC, "value": b["value"], "unit": UNIT,
                          "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic",
                          "config": {"workload": f"{wl.name} + {args.new_tokens} new tokens per sequence"},
                          "cpu_baseline": b,
                          "e2e": {"value": b["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}), flush=True)
        return
    if getattr(args, "row", "step") == "swap":
        b = swap_cpu_baseline(wl, budget_s=min(60.0, 0.5 * (args.steps + args.warmup)))
        print(json.dumps({"impl": "reference", "metric": SWAP_METRIC, "value": b["value"], "unit": UNIT,
                          "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
                          "data": "synthetic", "config": {"workload": f"{wl.name} preempt+resume"},
                          "cpu_baseline": b,
                          "e2e": {"value": b["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}), flush=True)
        return
    limits = blas_threads()
    ctx = limits(limits=1) if limits else None
    if ctx:
        ctx.__enter__()
    try:
        vals, ref = oracle_setup(wl)
        per_byte = calibrate(wl, ref, vals)
        per_step = min(1.0, 150.0 / max(1, args.steps + args.warmup))
        rng = np.random.default_rng(args.seed)
        for _ in range(args.warmup):
            oracle_units_timed(wl, ref, vals, pick_units(wl, rng, per_step, per_byte))
        tot_s, tot_b, n_units = 0.0, 0, 0
        for _ in range(args.steps):
            units = pick_units(wl, rng, per_step, per_byte)
            s, nb = oracle_units_timed(wl, ref, vals, units)
            tot_s += s
            tot_b += nb
            n_units += len(units)
    finally:
        if ctx:
            ctx.__exit__(None, None, None)
    value = tot_b / tot_s / 1e9
    sample = (f"each step: ~{n_units / max(1, args.steps):.1f} random (sequence, kv-head) units of workload "
              f"{wl.name} ({tot_b / max(1, args.steps) / 1e6:.1f} MB of K/V), fp64 numpy, one thread")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default 2000; 20 with --row swap)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, choices=sorted(workloads.NAMED),
                    help=f"one workload alone (default: {DEFAULT_WORKLOAD} headline + per_config entries for "
                         f"{', '.join(PER_CONFIG)}; --row swap / multi default to llama7b)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="the headline workload alone (no per_config entries)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--partition", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="capture one step in a CUDA graph and replay it (launch-bound batches)")
    ap.add_argument("--no-cascade", action="store_true",
                    help="decode a shared-prefix batch with the plain paged kernel")
    ap.add_argument("--cascade-overlap", action="store_true",
                    help="run the cascade's prefix pass on a second stream beside the copies and append "
                         "(three launches instead of one; no faster on B200 so far)")
    ap.add_argument("--unfused", action="store_true",
                    help="run a 16-bit step as separate copy/append and decode launches")
    ap.add_argument("--kv-fp8", action="store_true",
                    help="the step over an FP8 (E4M3) cache: quantising append + FP8 decode")
    ap.add_argument("--row", choices=["step", "swap", "multi"], default="step",
                    help="step: the decode step (default); swap: preemption by swapping; "
                         "multi: several new tokens per sequence")
    ap.add_argument("--new-tokens", type=int, default=5,
                    help="--row multi: new tokens per sequence (drafted + 1)")
    args = ap.parse_args(argv)
    if args.steps is None:
        args.steps = 20 if args.row == "swap" else 2000
    if args.workload is None and args.row != "step":
        args.workload = "llama7b"
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0

    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    if args.row == "multi":
        r = run_multi(args, rank, world, local_rank)
        if world > 1:
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(multi_line(args, r, world)), flush=True)
        return 0
    if args.row == "swap":
        r = run_swap(args, rank, world, local_rank)
        if world > 1:
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(swap_line(args, r, world)), flush=True)
        return 0
    headline = args.workload or DEFAULT_WORKLOAD
    others = [] if (args.workload or args.no_per_config) else [w for w in PER_CONFIG if w != headline]
    if args.kv_fp8:  # an FP8 cache holds 16-bit workloads' values only
        others = [w for w in others if workloads.named(w, args.seed).dtype != "f32"]
    r = run_cuda(args, rank, world, local_rank, workload=headline)
    per = {}
    for name in others:
        gc.collect()
        torch.cuda.empty_cache()
        # the tiny batch (319 KB of K/V) is launch-bound: its step runs as one
        # captured CUDA graph
        rr = run_cuda(args, rank, world, local_rank, workload=name, graph=True if name == "tiny" else None)
        per[name] = config_entry(args, rr, world)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    line = step_line(args, r, world)
    if per:
        line["per_config"] = per
    if world == 1 and not args.no_cpu_baseline and not args.kv_fp8:
        line["cpu_baseline"] = cpu_baseline(r["wl"], seed=args.seed)
    print(json.dumps(line), flush=True)
    return 0


def step_figures(args, r, world):
    """The decode step's figures from one run_cuda record: throughput, % of
    the measured HBM peak on unique bytes, the decode call's roofline, e2e."""
    wl = r["wl"]
    peak, peak_kind = measured_peak()
    K = r["K"]
    step_s = r["total_ms"] / 1e3 / K
    fp8 = bool(args.kv_fp8)
    kv_unique = kv_bytes(wl, True, fp8)
    kv_logical = kv_bytes(wl, False, fp8)
    dec_bytes = decode_algorithmic_bytes(wl, unique=True, fp8=fp8)
    achieved = dec_bytes / (r["dec_avg_ms"] / 1e3) / 1e9
    e2e_step_s = r["e2e_ms"] / 1e3 / K
    kernel = ("paged_decode_fp8 cascade (prefix widening, prefix pass, suffix pass, merge kernels)"
              if r["cascade_pages"] and fp8
              else "paged_decode cascade (prefix/suffix kernel + merge kernel)" if r["cascade_pages"]
              else "paged_decode_fp8 (partition + merge kernels)" if fp8
              else "paged_decode (partition + merge kernels)")
    return {
        "value": job_throughput(kv_logical, world, K, r["total_ms"] / 1e3),
        "ms_per_step": r["total_ms"] / K,
        "us_per_step": 1e3 * r["total_ms"] / K,
        "seq_steps_per_s": world * wl.B / step_s,
        "pct_hbm_peak": 100.0 * (world * kv_unique / step_s / 1e9) / (peak * world),
        "kv_bytes_per_step": {"logical": kv_logical, "unique": kv_unique},
        "clocks": r["clocks"],
        "e2e": {"value": job_throughput(kv_logical, world, K, r["e2e_ms"] / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "us_per_step": 1e6 * e2e_step_s},
        "gpu_launches": r["launches"],
        "launch": launch_of(args, r),
        "cascade_prefix_pages": r["cascade_pages"],
        "roofline": {"kernel": kernel, "bound": "hbm", "achieved": achieved, "peak": peak,
                     "peak_kind": f"{peak_kind} (MEASURED_PEAKS hbm_gbs)" if peak_kind == "measured" else "fallback",
                     "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None if fp8 else recorded_traffic(wl.name),
                     "algorithmic_bytes_per_launch": dec_bytes, "avg_launch_us": 1e3 * r["dec_avg_ms"],
                     "calls_timed": r["roof_calls"]},
    }


def config_entry(args, r, world):
    """One workload's entry of ``per_config``."""
    wl = r["wl"]
    f = step_figures(args, r, world)
    return {"config": config_of(wl, args), "dtype": wl.dtype, "unit": UNIT, "steps": r["K"], **f}


def step_line(args, r, world):
    """The contract's JSON line for the decode step on one workload."""
    wl = r["wl"]
    f = step_figures(args, r, world)
    line = {
        "metric": METRIC, "value": f.pop("value"), "unit": UNIT, "n_gpus": world, "steps": r["K"],
        "warmup": args.warmup, "ms_per_step": f.pop("ms_per_step"), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded N(0,1) q/K/V on the device, seeded lengths and placement)",
        "config": config_of(wl, args),
        "kv_cache": "e4m3 (FP8) codes, scale %.6g for K and V" % FP8_SCALE if args.kv_fp8 else wl.dtype,
    }
    line.update(f)
    return line


if __name__ == "__main__":
    sys.exit(main())
