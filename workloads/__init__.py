"""Seeded synthetic decode workloads for the paged KV-cache decode path.

This module draws random numbers and lays out the *structure* of one decode
batch: how many sequences, their context lengths, the pool size, the initial
order of the free-block list and the order of the cache operations (add a
sequence, append tokens, fork, free).  It holds none of the method's
arithmetic -- no slot or block-table arithmetic, no allocator policy and no
attention.  Each side (the CUDA library and the CPU oracle) replays the op log
through its own allocator, writes the drawn token values through its own
append and runs its own decode.

Shapes follow the pages' statement of the problem: K/V held in fixed
16-token blocks of a shared pool and reached through a per-sequence block
table ("PagedAttention 与 vLLM 推理加速", §2.2-§2.3).  The five named
workloads are

  tiny       B=4, ctx {7,16,33,100}, Hq=Hkv=4, D=64, fp32, 64-block pool
  llama7b    B=64, ctx U[128,2048], Hq=Hkv=32, D=128, fp16, 16384-block pool
  gqa8b      B=256, ctx lognormal(median 1024, sigma 1) clipped to
             [16,8192], Hq=32, Hkv=8, D=128, bf16, pool 1.1x the blocks used
  prefix13b  128 sequences sharing a 1024-token prefix (64 blocks), private
             suffix U[16,512], each forked once before the step so that
             the step copies-on-write every partially filled last block;
             Hq=Hkv=40, D=128, fp16
  long       B=8, ctx U[32768,131072], Hq=64, Hkv=8, D=128, bf16

"ctx" is the context length *after* the step's append: every sequence in
the step appends one new token and then attends over all ``ctx`` tokens,
itself included.  The prefill writes the first ``ctx - 1`` tokens.

Values: q, K and V are N(0,1) drawn in float32 and cast once to the
storage format (fp16 by numpy's round-to-nearest-even cast, bf16 by
round-to-nearest-even on the float32 bit pattern; bf16 arrays are carried
as their uint16 bit patterns because numpy has no bf16 type).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

BLOCK_SIZE = 16

# sequence-id bases used by the op logs (any distinct int64 ids would do)
ROOT_SEQ = 1_000_000
SIBLING_BASE = 2_000_000

STORAGE_BYTES = {"f32": 4, "f16": 2, "bf16": 2}

Op = Tuple  # ('add', sid) | ('append', sid, n) | ('fork', parent, child) | ('free', sid)


@dataclasses.dataclass
class Workload:
    """Structure of one decode batch.

    ``ops`` is the op log that builds the cache state before the step; the
    i-th token appended by the log (counting across every ``append`` op in
    order) carries the values ``k_tokens[i]`` / ``v_tokens[i]``.  The step
    then appends one token to each of ``step_seqs`` (values ``k_new[b]``,
    ``v_new[b]``) and decodes query ``q[b]`` for each of them.
    """

    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    dtype: str
    num_blocks: int
    free_order: np.ndarray  # int32 [num_blocks]
    ops: List[Op]
    step_seqs: np.ndarray  # int64 [B]
    context_lens: np.ndarray  # int32 [B], after the step's append
    seed: int
    block_size: int = BLOCK_SIZE

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def n_prefill_tokens(self) -> int:
        return int(sum(op[2] for op in self.ops if op[0] == "append"))

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.B else 0

    @property
    def step_append_mask(self) -> np.ndarray:
        """True where the step appends a token (a post-append length of 0
        marks a padded entry that appends nothing)."""
        return self.context_lens > 0

    @property
    def kv_bytes_per_token(self) -> int:
        """Bytes of K plus V one token holds across all kv-heads."""
        return 2 * self.Hkv * self.D * STORAGE_BYTES[self.dtype]


# --------------------------------------------------------------------------
# value drawing
# --------------------------------------------------------------------------

def _to_storage(x32: np.ndarray, dtype: str) -> np.ndarray:
    """Cast float32 draws to the storage format (bf16 as uint16 bits)."""
    if dtype == "f32":
        return x32
    if dtype == "f16":
        return x32.astype(np.float16)
    if dtype == "bf16":
        bits = x32.view(np.uint32)
        # round to nearest even on the upper 16 bits (draws are finite)
        rounded = bits + np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))
        return (rounded >> np.uint32(16)).astype(np.uint16)
    raise ValueError(dtype)


def draw_values(wl: Workload, chunk: int = 1 << 24) -> Dict[str, np.ndarray]:
    """Draw q, k_new, v_new and the prefill tokens for ``wl`` (numpy PCG64).

    Returns storage-format arrays: q [B,Hq,D], k_new/v_new [B,Hkv,D],
    k_tokens/v_tokens [n_prefill_tokens,Hkv,D].
    """
    rng = np.random.default_rng([wl.seed, 1])
    out = {}
    shapes = [
        ("q", (wl.B, wl.Hq, wl.D)),
        ("k_new", (wl.B, wl.Hkv, wl.D)),
        ("v_new", (wl.B, wl.Hkv, wl.D)),
        ("k_tokens", (wl.n_prefill_tokens, wl.Hkv, wl.D)),
        ("v_tokens", (wl.n_prefill_tokens, wl.Hkv, wl.D)),
    ]
    for name, shape in shapes:
        n = int(np.prod(shape))
        sdt = np.uint16 if wl.dtype == "bf16" else (np.float16 if wl.dtype == "f16" else np.float32)
        arr = np.empty(n, dtype=sdt)
        for s in range(0, n, chunk):
            e = min(n, s + chunk)
            arr[s:e] = _to_storage(rng.standard_normal(e - s, dtype=np.float32), wl.dtype)
        out[name] = arr.reshape(shape)
    return out


# --------------------------------------------------------------------------
# structures
# --------------------------------------------------------------------------

def _blocks_for(n_tokens: int) -> int:
    return -(-int(n_tokens) // BLOCK_SIZE)


def _independent(name, B, Hq, Hkv, D, dtype, ctx, num_blocks, seed, rng) -> Workload:
    ctx = np.asarray(ctx, dtype=np.int64)
    ops: List[Op] = []
    for b in range(B):
        ops.append(("add", b))
        if ctx[b] > 1:
            ops.append(("append", b, int(ctx[b]) - 1))
    free_order = rng.permutation(num_blocks).astype(np.int32)
    return Workload(name=name, B=B, Hq=Hq, Hkv=Hkv, D=D, dtype=dtype,
                    num_blocks=int(num_blocks), free_order=free_order, ops=ops,
                    step_seqs=np.arange(B, dtype=np.int64),
                    context_lens=ctx.astype(np.int32), seed=seed)


def tiny(seed: int = 0) -> Workload:
    rng = np.random.default_rng(seed)
    return _independent("tiny", 4, 4, 4, 64, "f32", [7, 16, 33, 100], 64, seed, rng)


def llama7b(seed: int = 0) -> Workload:
    rng = np.random.default_rng(seed)
    ctx = rng.integers(128, 2048, size=64, endpoint=True)
    return _independent("llama7b", 64, 32, 32, 128, "f16", ctx, 16384, seed, rng)


def llama7b_compact(seed: int = 0) -> Workload:
    """llama7b's lengths, heads and dtype in a pool of 1.1x the blocks used
    (about 1.3 GB instead of 4.3 GB): the small case for full profiler
    captures of the same kernel."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(128, 2048, size=64, endpoint=True)
    need = sum(_blocks_for(c) for c in ctx)
    return _independent("llama7b_compact", 64, 32, 32, 128, "f16", ctx, math.ceil(1.1 * need), seed, rng)


def gqa8b(seed: int = 0, sigma: float = 1.0) -> Workload:
    rng = np.random.default_rng(seed)
    raw = rng.lognormal(mean=math.log(1024.0), sigma=sigma, size=256)
    ctx = np.clip(np.rint(raw), 16, 8192).astype(np.int64)
    need = sum(_blocks_for(c) for c in ctx)
    return _independent("gqa8b", 256, 32, 8, 128, "bf16", ctx, math.ceil(1.1 * need), seed, rng)


def long(seed: int = 0) -> Workload:
    rng = np.random.default_rng(seed)
    ctx = rng.integers(32768, 131072, size=8, endpoint=True)
    need = sum(_blocks_for(c) for c in ctx)
    return _independent("long", 8, 64, 8, 128, "bf16", ctx, math.ceil(1.1 * need), seed, rng)


def prefix13b(seed: int = 0, B: int = 128, prefix_tokens: int = 1024,
              suffix_range: Tuple[int, int] = (16, 512), Hq: int = 40, Hkv: int = 40,
              D: int = 128, dtype: str = "f16", name: str = "prefix13b") -> Workload:
    """Shared system prefix, private suffixes, one sibling fork per sequence.

    Op log: a root sequence prefills the prefix; every batch sequence forks
    from it (sharing the prefix blocks); the root is freed; each sequence
    prefills its private suffix; each sequence is forked once more (a
    parallel-sampling sibling) so its private blocks are shared too.  In the
    step, a sequence whose suffix ends mid-block must copy that shared
    block before it can append.
    """
    rng = np.random.default_rng(seed)
    lo, hi = suffix_range
    suffix = rng.integers(lo, hi, size=B, endpoint=True)
    ops: List[Op] = [("add", ROOT_SEQ)]
    if prefix_tokens:
        ops.append(("append", ROOT_SEQ, prefix_tokens))
    for b in range(B):
        ops.append(("fork", ROOT_SEQ, b))
    ops.append(("free", ROOT_SEQ))
    for b in range(B):
        if suffix[b]:
            ops.append(("append", b, int(suffix[b])))
    for b in range(B):
        ops.append(("fork", b, SIBLING_BASE + b))
    # blocks: shared prefix + private suffix blocks + one new/CoW block per
    # sequence in the step; pool 1.1x that
    need = _blocks_for(prefix_tokens) + sum(_blocks_for(s) for s in suffix) + B
    num_blocks = math.ceil(1.1 * need)
    free_order = rng.permutation(num_blocks).astype(np.int32)
    ctx = (prefix_tokens + suffix + 1).astype(np.int32)
    return Workload(name=name, B=B, Hq=Hq, Hkv=Hkv, D=D, dtype=dtype,
                    num_blocks=num_blocks, free_order=free_order, ops=ops,
                    step_seqs=np.arange(B, dtype=np.int64), context_lens=ctx, seed=seed)


def custom(ctx: Sequence[int], Hq: int, Hkv: int, D: int, dtype: str,
           num_blocks: Optional[int] = None, seed: int = 0, name: str = "custom") -> Workload:
    """Independent sequences with the given post-append context lengths.

    A context length of 0 adds the sequence without any token and without a
    step append (the sequence is decoded with nothing to attend to); the
    step's new-token values are still drawn for it but no slot is written.
    """
    rng = np.random.default_rng(seed)
    ctx = np.asarray(list(ctx), dtype=np.int64)
    need = sum(_blocks_for(c) for c in ctx)
    nb = int(num_blocks) if num_blocks is not None else max(4, math.ceil(1.25 * need) + 4)
    return _independent(name, len(ctx), Hq, Hkv, D, dtype, ctx, nb, seed, rng)


NAMED = {
    "tiny": tiny,
    "llama7b": llama7b,
    "llama7b_compact": llama7b_compact,
    "gqa8b": gqa8b,
    "prefix13b": prefix13b,
    "long": long,
}


def named(name: str, seed: int = 0) -> Workload:
    return NAMED[name](seed)
