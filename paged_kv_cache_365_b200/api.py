"""Python binding of libpkv: torch tensors in, C-ABI calls out.

Argument marshalling only -- shape/dtype/device checks, raw pointers, the
current CUDA stream.  Every step of the path runs in the library's CUDA
kernels (device ops) or its C++ allocator (host bookkeeping).  PyTorch
provides device memory and streams.
"""
from __future__ import annotations

import contextlib
import ctypes
import functools
import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np
import torch


@contextlib.contextmanager
def nvtx_range(name: str):
    """An NVTX range around host code (shows in Nsight timelines; a no-op
    without a profiler attached)."""
    torch.cuda.nvtx.range_push(name)
    try:
        yield
    finally:
        torch.cuda.nvtx.range_pop()


def _traced(name: str):
    def wrap(fn):
        @functools.wraps(fn)
        def inner(*a, **kw):
            with nvtx_range(name):
                return fn(*a, **kw)
        return inner
    return wrap

from . import _lib
from ._lib import check, lib

BLOCK_SIZE = 16
DEFAULT_PARTITION = 512


def partition_tokens(op: int, max_context_len: int, partition: int = 0, prefix_pages: int = 0,
                     rows: int = 0) -> int:
    """Tokens per split-K partition that call ``op`` (``_lib.OP_*``) makes
    with this ``partition`` argument (0 = its auto rule): the library's own
    rule (pkv_partition_tokens).  ``prefix_pages``: the cascade's shared
    pages (OP_DECODE_PREFIX); ``rows``: rows per kv-head of a multi-token
    call, max_query_len * Hq / Hkv (OP_MULTI)."""
    extra = prefix_pages if int(op) == _lib.OP_DECODE_PREFIX else rows
    p = int(lib.pkv_partition_tokens(int(op), int(partition), int(max_context_len), int(extra)))
    if p < 0:
        raise ValueError(f"invalid partition {partition} for op {op}")
    return p


def auto_partition(max_context_len: int) -> int:
    """The decode's partition for partition=0 (pkv_partition_tokens)."""
    return partition_tokens(_lib.OP_DECODE, max_context_len)


def auto_partition_multi(max_context_len: int) -> int:
    """The multi-token path's partition for partition=0."""
    return partition_tokens(_lib.OP_MULTI, max_context_len)


def auto_partition_fp8(max_context_len: int) -> int:
    """The FP8 decode's partition for partition=0."""
    return partition_tokens(_lib.OP_DECODE_FP8, max_context_len)


# an FP8 cache holds E4M3 codes: torch.float8_e4m3fn, or uint8 bytes
_DT = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2, torch.float8_e4m3fn: 3, torch.uint8: 3}
_FP8 = (torch.float8_e4m3fn, torch.uint8)


def _i32p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _i64p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def kv_cache_bytes(num_layers: int, num_heads: int, head_dim: int, seq_len: int, dtype_bytes: int) -> int:
    """Bytes of K plus V for one sequence: 2 * L * H * D * S * dtype_size
    ("PagedAttention 与 vLLM 推理加速" §1)."""
    return 2 * num_layers * num_heads * head_dim * seq_len * dtype_bytes


def _stream(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _cache_dims(k_cache: torch.Tensor, v_cache: torch.Tensor):
    if k_cache.dim() != 4 or k_cache.shape != v_cache.shape or k_cache.dtype != v_cache.dtype:
        raise ValueError("k_cache/v_cache must both be [num_blocks, Hkv, 16, D] of one dtype")
    nb, hkv, bs, d = k_cache.shape
    if bs != BLOCK_SIZE:
        raise ValueError(f"block size must be {BLOCK_SIZE}")
    if k_cache.dtype not in _DT:
        raise ValueError(f"unsupported dtype {k_cache.dtype}")
    return nb, hkv, d


def kv_append(k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              slot_mapping: torch.Tensor, stream=None) -> None:
    """Write each new token's K/V into its slot (slot < 0: skipped).

    k_new/v_new [N, Hkv, D]; slot_mapping int64 [N] on the device.
    """
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if k_new.shape != v_new.shape or k_new.dim() != 3 or tuple(k_new.shape[1:]) != (hkv, d):
        raise ValueError("k_new/v_new must be [N, Hkv, D] matching the cache")
    n = k_new.shape[0]
    if slot_mapping.shape != (n,):
        raise ValueError("slot_mapping must be [N]")
    check(lib.pkv_kv_append(_dev(k_new, "k_new", k_cache.dtype), _dev(v_new, "v_new", k_cache.dtype),
                            _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                            _dev(slot_mapping, "slot_mapping", torch.int64), n, hkv, d, nb,
                            _DT[k_cache.dtype], _stream(stream, k_cache.device)), "pkv_kv_append")


def copy_blocks_check(pairs_host: np.ndarray, num_blocks: int) -> None:
    """Host check of copy pairs (ids in range, distinct dst, no dst is a src)."""
    p = np.ascontiguousarray(pairs_host, dtype=np.int32).reshape(-1, 2)
    check(lib.pkv_copy_blocks_check(p.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), p.shape[0], num_blocks),
          "pkv_copy_blocks_check")


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, pairs: torch.Tensor, stream=None) -> None:
    """cache[dst] = cache[src] for each (src, dst) row of int32 ``pairs`` [n, 2] (device)."""
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be [n, 2]")
    n = pairs.shape[0]
    if n == 0:
        return
    check(lib.pkv_copy_blocks(_dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                              _dev(pairs, "pairs", torch.int32), n, hkv, d, nb, _DT[k_cache.dtype],
                              _stream(stream, k_cache.device)), "pkv_copy_blocks")


def _any(t: torch.Tensor, name: str, dtype=None) -> int:
    """Device tensor, or page-locked host tensor (the library maps it)."""
    if not isinstance(t, torch.Tensor) or not (t.is_cuda or t.is_pinned()):
        raise ValueError(f"{name} must be a CUDA tensor or a pinned host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def swap_blocks_check(pairs_host: np.ndarray, src_blocks: int, dst_blocks: int) -> None:
    """Host check of swap pairs (ids in range, distinct dst)."""
    p = np.ascontiguousarray(pairs_host, dtype=np.int32).reshape(-1, 2)
    check(lib.pkv_swap_blocks_check(p.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), p.shape[0], src_blocks,
                                    dst_blocks), "pkv_swap_blocks_check")


def swap_blocks(dst_k: torch.Tensor, dst_v: torch.Tensor, src_k: torch.Tensor, src_v: torch.Tensor,
                pairs: torch.Tensor, stream=None, device=None) -> None:
    """dst[d] = src[s] for each (s, d) row of int32 ``pairs`` [n, 2], K and V.

    Each pool is [blocks, Hkv, 16, D] on the device or in pinned host memory
    (preemption by swapping); ``pairs`` on the device or pinned.  Runs on the
    current stream of ``device`` (default: the device of a CUDA operand)."""
    dnb, hkv, d = _cache_dims(dst_k, dst_v)
    snb, shkv, sd = _cache_dims(src_k, src_v)
    if (shkv, sd) != (hkv, d) or src_k.dtype != dst_k.dtype:
        raise ValueError("source and destination pools must share Hkv, D and dtype")
    if pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be [n, 2]")
    n = pairs.shape[0]
    if n == 0:
        return
    if device is None:
        cuda = [t for t in (dst_k, src_k, pairs) if t.is_cuda]
        device = cuda[0].device if cuda else torch.device("cuda", torch.cuda.current_device())
    check(lib.pkv_swap_blocks(_any(dst_k, "dst_k"), _any(dst_v, "dst_v"), dnb, _any(src_k, "src_k"),
                              _any(src_v, "src_v"), snb, _any(pairs, "pairs", torch.int32), n, hkv, d,
                              _DT[dst_k.dtype], _stream(stream, device)), "pkv_swap_blocks")


def kv_append_fp8(k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  slot_mapping: torch.Tensor, k_scale: float, v_scale: float, stream=None) -> None:
    """Quantise each new token's K/V (fp16/bf16 [N, Hkv, D]) into its slot of
    an FP8 cache: code = E4M3(x / scale), one scale for K and one for V."""
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if k_cache.dtype not in _FP8:
        raise ValueError("kv_append_fp8 writes an FP8 cache (float8_e4m3fn or uint8)")
    if k_new.shape != v_new.shape or k_new.dim() != 3 or tuple(k_new.shape[1:]) != (hkv, d):
        raise ValueError("k_new/v_new must be [N, Hkv, D] matching the cache")
    if k_new.dtype not in (torch.float16, torch.bfloat16) or v_new.dtype != k_new.dtype:
        raise ValueError("k_new/v_new must be fp16 or bf16")
    n = k_new.shape[0]
    if slot_mapping.shape != (n,):
        raise ValueError("slot_mapping must be [N]")
    check(lib.pkv_kv_append_fp8(_dev(k_new, "k_new"), _dev(v_new, "v_new"), _dev(k_cache, "k_cache"),
                                _dev(v_cache, "v_cache"), _dev(slot_mapping, "slot_mapping", torch.int64), n, hkv, d,
                                nb, _DT[k_new.dtype], float(k_scale), float(v_scale),
                                _stream(stream, k_cache.device)), "pkv_kv_append_fp8")


def paged_attention_decode_fp8(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                               block_tables: torch.Tensor, context_lens: torch.Tensor, max_context_len: int,
                               scale: float, k_scale: float, v_scale: float, out: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None, partition: int = 0,
                               stream=None) -> torch.Tensor:
    """paged_attention_decode over an FP8 cache (E4M3 codes, one scale for K
    and one for V); q and the output in fp16 or bf16."""
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if k_cache.dtype not in _FP8:
        raise ValueError("an FP8 cache (float8_e4m3fn or uint8) is required")
    if q.dim() != 3 or q.shape[2] != d or q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("q must be [B, Hq, D] in fp16 or bf16")
    B, hq, _ = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    if out is None:
        out = torch.empty_like(q)
    need = decode_workspace_bytes(B, hq, d, max_context_len, partition)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if need else None
    ws_len = workspace.numel() * workspace.element_size() if need else 0
    check(lib.pkv_paged_attention_decode_fp8(
        _dev(out, "out", q.dtype), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len), B, hq, hkv, d, nb, float(scale),
        float(k_scale), float(v_scale), int(partition), _DT[q.dtype], ws_ptr, ws_len, _stream(stream, q.device)),
        "pkv_paged_attention_decode_fp8")
    return out


def cow_copy_rows(pairs: np.ndarray, slots: np.ndarray) -> np.ndarray:
    """(src, dst, rows) for each copy-on-write pair of a step
    (pkv_cow_copy_rows): rows = the first row a slot of the step writes into
    dst (16 when none does), the rows of dst that hold tokens."""
    p = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    s = np.ascontiguousarray(np.asarray(slots, dtype=np.int64).reshape(-1))
    out = np.empty((max(p.shape[0], 1), 3), dtype=np.int32)
    check(lib.pkv_cow_copy_rows(_i32p(p), p.shape[0], _i64p(s), s.shape[0], _i32p(out)), "pkv_cow_copy_rows")
    return out[:p.shape[0]]


def kv_append_copy(k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   slot_mapping: torch.Tensor, copies: torch.Tensor, stream=None) -> None:
    """The step's copy-on-write copies and append in one launch: int32
    ``copies`` [n, 3] = (src, dst, rows) (``cow_copy_rows``): rows 0..rows-1
    of dst from src, then every token into its slot."""
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if k_new.shape != v_new.shape or k_new.dim() != 3 or tuple(k_new.shape[1:]) != (hkv, d):
        raise ValueError("k_new/v_new must be [N, Hkv, D] matching the cache")
    n = k_new.shape[0]
    if slot_mapping.shape != (n,) or copies.dim() != 2 or copies.shape[1] != 3:
        raise ValueError("slot_mapping must be [N] and copies [n, 3]")
    check(lib.pkv_kv_append_copy(_dev(k_new, "k_new", k_cache.dtype), _dev(v_new, "v_new", k_cache.dtype),
                                 _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                 _dev(slot_mapping, "slot_mapping", torch.int64), n,
                                 _dev(copies, "copies", torch.int32) if copies.shape[0] else None, copies.shape[0],
                                 hkv, d, nb, _DT[k_cache.dtype], _stream(stream, k_cache.device)),
          "pkv_kv_append_copy")


def decode_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int, max_context_len: int,
                           partition: int = 0) -> int:
    return int(lib.pkv_decode_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len, partition))


def paged_attention_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                           block_tables: torch.Tensor, context_lens: torch.Tensor, max_context_len: int,
                           scale: float, out: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None, partition: int = 0,
                           stream=None) -> torch.Tensor:
    """Single-query attention of each sequence over its paged K/V.

    q [B, Hq, D]; block_tables int32 [B, max_blocks]; context_lens int32 [B]
    (lengths after this step's append); max_context_len: host bound on
    context_lens.  Returns ``out`` [B, Hq, D] in q's dtype.  ``workspace``
    (uint8, >= decode_workspace_bytes) is allocated here when not given.
    """
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if q.dim() != 3 or q.shape[2] != d or q.dtype != k_cache.dtype:
        raise ValueError("q must be [B, Hq, D] in the cache dtype")
    B, hq, _ = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    if out is None:
        out = torch.empty_like(q)
    need = decode_workspace_bytes(B, hq, d, max_context_len, partition)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if need else None
    ws_len = workspace.numel() * workspace.element_size() if need else 0
    check(lib.pkv_paged_attention_decode(
        _dev(out, "out", q.dtype), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len), B, hq, hkv, d, nb,
        float(scale), int(partition), _DT[k_cache.dtype], ws_ptr, ws_len,
        _stream(stream, q.device)), "pkv_paged_attention_decode")
    return out


def decode_step(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, k_new: torch.Tensor,
                v_new: torch.Tensor, slot_mapping: torch.Tensor, copies: Optional[torch.Tensor],
                block_tables: torch.Tensor, context_lens: torch.Tensor, max_context_len: int, scale: float,
                prefix_blocks: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, partition: int = 0, stream=None) -> torch.Tensor:
    """One decode step in one launch (pkv_decode_step): the step's
    copy-on-write copies (int32 ``copies`` [n, 3] = (src, dst, rows), from
    ``cow_copy_rows``) and append of one new token per sequence (k_new /
    v_new [B, Hkv, D], slot_mapping int64 [B]), then the decode -- the
    cascade when ``prefix_blocks`` (int32, the shared leading blocks) is
    given.  16-bit pools."""
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if q.dim() != 3 or q.shape[2] != d or q.dtype != k_cache.dtype:
        raise ValueError("q must be [B, Hq, D] in the cache dtype")
    B, hq, _ = q.shape
    if k_new.shape != (B, hkv, d) or v_new.shape != k_new.shape or slot_mapping.shape != (B,):
        raise ValueError("k_new/v_new must be [B, Hkv, D] and slot_mapping [B]")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    n_copies = 0 if copies is None else int(copies.shape[0])
    if n_copies and (copies.dim() != 2 or copies.shape[1] != 3):
        raise ValueError("copies must be [n, 3]")
    pp = 0 if prefix_blocks is None else int(prefix_blocks.numel())
    if out is None:
        out = torch.empty_like(q)
    need = (decode_prefix_workspace_bytes(B, hq, d, max_context_len, pp, partition) if pp else
            decode_workspace_bytes(B, hq, d, max_context_len, partition))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    check(lib.pkv_decode_step(
        _dev(out, "out", q.dtype), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(k_new, "k_new", k_cache.dtype), _dev(v_new, "v_new", k_cache.dtype),
        _dev(slot_mapping, "slot_mapping", torch.int64), _dev(copies, "copies", torch.int32) if n_copies else None,
        n_copies, _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len),
        _dev(prefix_blocks, "prefix_blocks", torch.int32) if pp else None, pp, B, hq, hkv, d, nb, float(scale),
        int(partition), _DT[k_cache.dtype], _dev(workspace, "workspace") if need else None,
        workspace.numel() * workspace.element_size() if need else 0, _stream(stream, q.device)),
        "pkv_decode_step")
    return out


def decode_step_fp8(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, k_new: torch.Tensor,
                    v_new: torch.Tensor, slot_mapping: torch.Tensor, copies: Optional[torch.Tensor],
                    block_tables: torch.Tensor, context_lens: torch.Tensor, max_context_len: int, scale: float,
                    k_scale: float, v_scale: float, prefix_blocks: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, partition: int = 0,
                    stream=None) -> torch.Tensor:
    """decode_step over an FP8 cache (pkv_decode_step_fp8): the copies
    (int32 [n, 3] from ``cow_copy_rows``) and the append of one new token
    per sequence (k_new / v_new [B, Hkv, D] in q's dtype, quantised with
    k_scale / v_scale) made by the decode's CTAs -- the FP8 cascade's when
    ``prefix_blocks`` (int32, the shared leading blocks) is given."""
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if k_cache.dtype not in _FP8:
        raise ValueError("an FP8 cache (float8_e4m3fn or uint8) is required")
    if q.dim() != 3 or q.shape[2] != d or q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("q must be [B, Hq, D] in fp16 or bf16")
    B, hq, _ = q.shape
    if k_new.shape != (B, hkv, d) or v_new.shape != k_new.shape or slot_mapping.shape != (B,):
        raise ValueError("k_new/v_new must be [B, Hkv, D] and slot_mapping [B]")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    n_copies = 0 if copies is None else int(copies.shape[0])
    if n_copies and (copies.dim() != 2 or copies.shape[1] != 3):
        raise ValueError("copies must be [n, 3]")
    pp = 0 if prefix_blocks is None else int(prefix_blocks.numel())
    if out is None:
        out = torch.empty_like(q)
    need = (decode_prefix_fp8_workspace_bytes(B, hq, hkv, d, max_context_len, pp, partition) if pp else
            decode_workspace_bytes(B, hq, d, max_context_len, partition))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    check(lib.pkv_decode_step_fp8(
        _dev(out, "out", q.dtype), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(k_new, "k_new", q.dtype), _dev(v_new, "v_new", q.dtype), _dev(slot_mapping, "slot_mapping", torch.int64),
        _dev(copies, "copies", torch.int32) if n_copies else None, n_copies,
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len),
        _dev(prefix_blocks, "prefix_blocks", torch.int32) if pp else None, pp, B, hq, hkv, d, nb, float(scale),
        float(k_scale), float(v_scale), int(partition), _DT[q.dtype], _dev(workspace, "workspace") if need else None,
        workspace.numel() * workspace.element_size() if need else 0, _stream(stream, q.device)),
        "pkv_decode_step_fp8")
    return out


def decode_prefix_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int, max_context_len: int,
                                  prefix_pages: int, partition: int = 0) -> int:
    return int(lib.pkv_decode_prefix_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len,
                                                     prefix_pages, partition))


def _tables_lens(block_tables, context_lens):
    bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    if bt.ndim != 2:
        raise ValueError("block_tables must be [B, W]")
    lens = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32).reshape(-1))
    if lens.shape[0] != bt.shape[0]:
        raise ValueError("context_lens must be [B]")
    return bt, lens


def common_prefix_pages(block_tables: np.ndarray, context_lens: np.ndarray) -> int:
    """Leading pages that every sequence of the batch shares (same physical
    blocks) and fills completely (pkv_common_prefix_pages).  Host arrays:
    tables [B, W], lengths [B]."""
    bt, lens = _tables_lens(block_tables, context_lens)
    n = ctypes.c_int(0)
    check(lib.pkv_common_prefix_pages(_i32p(bt), bt.shape[0], bt.shape[1], _i32p(lens), ctypes.byref(n)),
          "pkv_common_prefix_pages")
    return int(n.value)


def cascade_prefix_pages(block_tables: np.ndarray, context_lens: np.ndarray, dtype: torch.dtype) -> int:
    """The shared prefix pages the cascade decode should read once, or 0 when
    the plain decode is the better call (pkv_cascade_prefix_pages)."""
    bt, lens = _tables_lens(block_tables, context_lens)
    n = ctypes.c_int(0)
    check(lib.pkv_cascade_prefix_pages(_i32p(bt), bt.shape[0], bt.shape[1], _i32p(lens), _DT[dtype],
                                       ctypes.byref(n)), "pkv_cascade_prefix_pages")
    return int(n.value)


def paged_attention_decode_prefix(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                  block_tables: torch.Tensor, context_lens: torch.Tensor, max_context_len: int,
                                  prefix_blocks: torch.Tensor, scale: float, out: Optional[torch.Tensor] = None,
                                  workspace: Optional[torch.Tensor] = None, partition: int = 0,
                                  stream=None, phase: int = -1) -> torch.Tensor:
    """Cascade decode for a batch sharing the blocks ``prefix_blocks``
    (int32 [prefix_pages], device) at the start of every table: the shared
    pages are read once per kv-head.  Same result as paged_attention_decode.

    ``phase`` -1 runs the whole cascade; 0 / 1 / 2 run its prefix pass,
    suffix pass and merge alone (same arguments and workspace for all three;
    the caller orders them across streams)."""
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if q.dim() != 3 or q.shape[2] != d or q.dtype != k_cache.dtype:
        raise ValueError("q must be [B, Hq, D] in the cache dtype")
    B, hq, _ = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    pp = int(prefix_blocks.numel())
    if out is None:
        out = torch.empty_like(q)
    need = decode_prefix_workspace_bytes(B, hq, d, max_context_len, pp, partition)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        if phase != -1:
            raise ValueError("the phases of one cascade must share a workspace the caller provides")
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    args = (_dev(out, "out", q.dtype), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
            _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
            _dev(context_lens, "context_lens", torch.int32), int(max_context_len),
            _dev(prefix_blocks, "prefix_blocks", torch.int32), pp, B, hq, hkv, d, nb, float(scale), int(partition),
            _DT[k_cache.dtype], _dev(workspace, "workspace"), workspace.numel() * workspace.element_size())
    if phase == -1:
        check(lib.pkv_paged_attention_decode_prefix(*args, _stream(stream, q.device)),
              "pkv_paged_attention_decode_prefix")
    else:
        check(lib.pkv_paged_attention_decode_prefix_phase(*args, int(phase), _stream(stream, q.device)),
              "pkv_paged_attention_decode_prefix_phase")
    return out


def decode_prefix_fp8_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                                      max_context_len: int, prefix_pages: int, partition: int = 0) -> int:
    return int(lib.pkv_decode_prefix_fp8_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                         max_context_len, prefix_pages, partition))


def paged_attention_decode_prefix_fp8(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                      block_tables: torch.Tensor, context_lens: torch.Tensor, max_context_len: int,
                                      prefix_blocks: torch.Tensor, scale: float, k_scale: float, v_scale: float,
                                      out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                                      partition: int = 0, stream=None) -> torch.Tensor:
    """The shared-prefix decode over an FP8 cache (E4M3 codes, one scale for
    K and one for V): the prefix blocks ``prefix_blocks`` (int32, device)
    every table starts with are read once per kv-head.  q / out fp16 or
    bf16."""
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if k_cache.dtype not in _FP8:
        raise ValueError("an FP8 cache (float8_e4m3fn or uint8) is required")
    if q.dim() != 3 or q.shape[2] != d or q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("q must be [B, Hq, D] in fp16 or bf16")
    B, hq, _ = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    pp = int(prefix_blocks.numel())
    if out is None:
        out = torch.empty_like(q)
    need = decode_prefix_fp8_workspace_bytes(B, hq, hkv, d, max_context_len, pp, partition)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    check(lib.pkv_paged_attention_decode_prefix_fp8(
        _dev(out, "out", q.dtype), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len),
        _dev(prefix_blocks, "prefix_blocks", torch.int32), pp, B, hq, hkv, d, nb, float(scale), float(k_scale),
        float(v_scale), int(partition), _DT[q.dtype], _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream, q.device)),
        "pkv_paged_attention_decode_prefix_fp8")
    return out


def multi_workspace_bytes(total_query_tokens: int, num_q_heads: int, head_dim: int, max_context_len: int,
                          partition: int = 0) -> int:
    return int(lib.pkv_multi_workspace_bytes(total_query_tokens, num_q_heads, head_dim, max_context_len, partition))


def paged_attention_multi(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                          block_tables: torch.Tensor, context_lens: torch.Tensor, query_start: torch.Tensor,
                          max_context_len: int, max_query_len: int, scale: float,
                          out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                          partition: int = 0, stream=None) -> torch.Tensor:
    """Several query tokens per sequence, each attending causally over its
    sequence's paged K/V up to its own position.

    q [T, Hq, D] (fp16/bf16); query_start int32 [B + 1] (sequence b's rows
    are query_start[b] .. query_start[b+1]-1, its last n_b tokens, already
    appended); block_tables int32 [B, W]; context_lens int32 [B].
    max_context_len / max_query_len: host bounds.  Returns out [T, Hq, D].
    """
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if q.dim() != 3 or q.shape[2] != d or q.dtype != k_cache.dtype:
        raise ValueError("q must be [T, Hq, D] in the cache dtype")
    T, hq, _ = q.shape
    B = block_tables.shape[0]
    if block_tables.dim() != 2 or context_lens.shape != (B,) or query_start.shape != (B + 1,):
        raise ValueError("block_tables [B, W], context_lens [B] and query_start [B + 1] required")
    if out is None:
        out = torch.empty_like(q)
    need = multi_workspace_bytes(T, hq, d, max_context_len, partition)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if need else None
    ws_len = workspace.numel() * workspace.element_size() if need else 0
    check(lib.pkv_paged_attention_multi(
        _dev(out, "out", q.dtype), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len),
        _dev(query_start, "query_start", torch.int32), int(max_query_len), T, B, hq, hkv, d, nb, float(scale),
        int(partition), _DT[k_cache.dtype], ws_ptr, ws_len, _stream(stream, q.device)),
        "pkv_paged_attention_multi")
    return out


def paged_attention_multi_fp8(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                              block_tables: torch.Tensor, context_lens: torch.Tensor, query_start: torch.Tensor,
                              max_context_len: int, max_query_len: int, scale: float, k_scale: float,
                              v_scale: float, out: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None, partition: int = 0,
                              stream=None) -> torch.Tensor:
    """paged_attention_multi over an FP8 cache (E4M3 codes, one scale for K
    and one for V); q and the output in fp16 or bf16."""
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if k_cache.dtype not in _FP8:
        raise ValueError("an FP8 cache (float8_e4m3fn or uint8) is required")
    if q.dim() != 3 or q.shape[2] != d or q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("q must be [T, Hq, D] in fp16 or bf16")
    T, hq, _ = q.shape
    B = block_tables.shape[0]
    if block_tables.dim() != 2 or context_lens.shape != (B,) or query_start.shape != (B + 1,):
        raise ValueError("block_tables [B, W], context_lens [B] and query_start [B + 1] required")
    if out is None:
        out = torch.empty_like(q)
    need = multi_workspace_bytes(T, hq, d, max_context_len, partition)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if need else None
    ws_len = workspace.numel() * workspace.element_size() if need else 0
    check(lib.pkv_paged_attention_multi_fp8(
        _dev(out, "out", q.dtype), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len),
        _dev(query_start, "query_start", torch.int32), int(max_query_len), T, B, hq, hkv, d, nb, float(scale),
        float(k_scale), float(v_scale), int(partition), _DT[q.dtype], ws_ptr, ws_len, _stream(stream, q.device)),
        "pkv_paged_attention_multi_fp8")
    return out


def get_error(stream=None, device=None) -> int:
    """Read and clear the device error word (PKV_ERR_* bits); synchronises."""
    v = ctypes.c_uint32(0)
    check(lib.pkv_get_error(ctypes.byref(v), _stream(stream, device)), "pkv_get_error")
    return int(v.value)


def selftest_bounded_wait(limit_cycles: int, stream=None, device=None) -> None:
    """Run the kernels' bounded staged-copy wait on a barrier nothing
    completes (pkv_selftest_bounded_wait); get_error() then shows
    ERR_TIMEOUT."""
    check(lib.pkv_selftest_bounded_wait(int(limit_cycles), _stream(stream, device)), "pkv_selftest_bounded_wait")


# ---------------------------------------------------------------------------
# host allocator
# ---------------------------------------------------------------------------
class BlockAllocator:
    """The library's host block allocator (FIFO free list, refcounts, CoW)."""

    def __init__(self, num_blocks: int, free_order: Optional[Sequence[int]] = None):
        h = ctypes.c_void_p()
        order = None if free_order is None else np.ascontiguousarray(free_order, dtype=np.int32)
        check(lib.pkv_alloc_create(int(num_blocks), None if order is None else _i32p(order), ctypes.byref(h)),
              "pkv_alloc_create")
        self._h = h
        self.num_blocks = int(num_blocks)

    def close(self) -> None:
        if self._h:
            lib.pkv_alloc_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, sid: int) -> None:
        check(lib.pkv_alloc_add_seq(self._h, int(sid)), "pkv_alloc_add_seq")

    def fork(self, parent: int, child: int) -> None:
        check(lib.pkv_alloc_fork(self._h, int(parent), int(child)), "pkv_alloc_fork")

    def free_seq(self, sid: int) -> None:
        check(lib.pkv_alloc_free_seq(self._h, int(sid)), "pkv_alloc_free_seq")

    def append_slot(self, sid: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        slot, s, d = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        check(lib.pkv_alloc_append_slot(self._h, int(sid), ctypes.byref(slot), ctypes.byref(s), ctypes.byref(d)),
              "pkv_alloc_append_slot")
        return slot.value, (None if s.value < 0 else (s.value, d.value))

    def append_tokens(self, sid: int, n: int) -> Tuple[np.ndarray, np.ndarray]:
        slots = np.empty(max(n, 1), dtype=np.int64)
        pairs = np.empty(2, dtype=np.int32)
        nc = ctypes.c_int()
        check(lib.pkv_alloc_append_tokens(self._h, int(sid), int(n), _i64p(slots), _i32p(pairs), ctypes.byref(nc)),
              "pkv_alloc_append_tokens")
        return slots[:n], pairs[:2 * nc.value].reshape(-1, 2)

    def step(self, sids: Iterable[int]) -> Tuple[np.ndarray, np.ndarray]:
        ids = np.ascontiguousarray(list(sids), dtype=np.int64)
        n = ids.shape[0]
        slots = np.empty(max(n, 1), dtype=np.int64)
        pairs = np.empty(max(2 * n, 2), dtype=np.int32)
        nc = ctypes.c_int()
        check(lib.pkv_alloc_step(self._h, _i64p(ids), n, _i64p(slots), _i32p(pairs), ctypes.byref(nc)),
              "pkv_alloc_step")
        return slots[:n], pairs[:2 * nc.value].reshape(-1, 2)

    def step_copies(self, sids: Iterable[int]) -> Tuple[np.ndarray, np.ndarray]:
        """``step`` with the copy pairs cut to rows (pkv_alloc_step_copies):
        slots [n] and (src, dst, rows) copies [k, 3] for kv_append_copy."""
        ids = np.ascontiguousarray(list(sids), dtype=np.int64)
        n = ids.shape[0]
        slots = np.empty(max(n, 1), dtype=np.int64)
        copies = np.empty((max(n, 1), 3), dtype=np.int32)
        nc = ctypes.c_int()
        check(lib.pkv_alloc_step_copies(self._h, _i64p(ids), n, _i64p(slots), _i32p(copies), ctypes.byref(nc)),
              "pkv_alloc_step_copies")
        return slots[:n], copies[:nc.value]

    def block_table(self, sid: int) -> Tuple[List[int], int]:
        nb, ln = ctypes.c_int(), ctypes.c_int64()
        check(lib.pkv_alloc_block_table(self._h, int(sid), None, 0, ctypes.byref(nb), ctypes.byref(ln)),
              "pkv_alloc_block_table")
        out = np.empty(max(nb.value, 1), dtype=np.int32)
        check(lib.pkv_alloc_block_table(self._h, int(sid), _i32p(out), nb.value, ctypes.byref(nb),
                                        ctypes.byref(ln)), "pkv_alloc_block_table")
        return [int(x) for x in out[:nb.value]], int(ln.value)

    def block_tables(self, sids: Sequence[int], width: int, pad: int) -> Tuple[np.ndarray, np.ndarray]:
        ids = np.ascontiguousarray(list(sids), dtype=np.int64)
        n = ids.shape[0]
        tables = np.empty((max(n, 1), max(width, 1)), dtype=np.int32)
        lens = np.empty(max(n, 1), dtype=np.int32)
        check(lib.pkv_alloc_block_tables(self._h, _i64p(ids), n, _i32p(tables), int(width), int(pad), _i32p(lens)),
              "pkv_alloc_block_tables")
        return tables[:n, :width], lens[:n]

    def state(self) -> Tuple[List[int], List[int]]:
        free = np.empty(self.num_blocks, dtype=np.int32)
        rc = np.empty(self.num_blocks, dtype=np.int32)
        nf = ctypes.c_int()
        check(lib.pkv_alloc_state(self._h, _i32p(free), ctypes.byref(nf), _i32p(rc)), "pkv_alloc_state")
        return [int(x) for x in free[:nf.value]], [int(x) for x in rc]

    @property
    def num_free(self) -> int:
        return int(lib.pkv_alloc_num_free(self._h))

    @property
    def num_seqs(self) -> int:
        """Resident sequences (swapped ones not counted)."""
        return int(lib.pkv_alloc_num_seqs(self._h))

    # -- preemption by swapping --------------------------------------------
    def set_host_pool(self, num_host_blocks: int) -> None:
        check(lib.pkv_alloc_set_host_pool(self._h, int(num_host_blocks)), "pkv_alloc_set_host_pool")
        self.num_host_blocks = int(num_host_blocks)

    def _swap(self, fn, name, sids) -> np.ndarray:
        ids = np.ascontiguousarray(list(sids), dtype=np.int64)
        cap = max(self.num_blocks, getattr(self, "num_host_blocks", 0), 1)
        pairs = np.empty((cap, 2), dtype=np.int32)
        n = ctypes.c_int()
        check(fn(self._h, _i64p(ids), ids.shape[0], _i32p(pairs), cap, ctypes.byref(n)), name)
        return pairs[:n.value]

    def swap_out(self, sids: Iterable[int]) -> np.ndarray:
        """Move resident sequences to the host pool; (device, host) pairs [n, 2]."""
        return self._swap(lib.pkv_alloc_swap_out, "pkv_alloc_swap_out", sids)

    def swap_in(self, sids: Iterable[int]) -> np.ndarray:
        """Bring swapped sequences back; (host, device) pairs [n, 2]."""
        return self._swap(lib.pkv_alloc_swap_in, "pkv_alloc_swap_in", sids)

    def host_state(self) -> Tuple[List[int], List[int]]:
        nh = getattr(self, "num_host_blocks", 0)
        free = np.empty(max(nh, 1), dtype=np.int32)
        rc = np.empty(max(nh, 1), dtype=np.int32)
        nf = ctypes.c_int()
        check(lib.pkv_alloc_host_state(self._h, _i32p(free), ctypes.byref(nf), _i32p(rc)), "pkv_alloc_host_state")
        return [int(x) for x in free[:nf.value]], [int(x) for x in rc[:nh]]

    def swapped_table(self, sid: int) -> Tuple[List[int], int]:
        nb, ln = ctypes.c_int(), ctypes.c_int64()
        check(lib.pkv_alloc_swapped_table(self._h, int(sid), None, 0, ctypes.byref(nb), ctypes.byref(ln)),
              "pkv_alloc_swapped_table")
        out = np.empty(max(nb.value, 1), dtype=np.int32)
        check(lib.pkv_alloc_swapped_table(self._h, int(sid), _i32p(out), nb.value, ctypes.byref(nb),
                                          ctypes.byref(ln)), "pkv_alloc_swapped_table")
        return [int(x) for x in out[:nb.value]], int(ln.value)

    @property
    def num_swapped(self) -> int:
        return int(lib.pkv_alloc_num_swapped(self._h))


# ---------------------------------------------------------------------------
# host <-> device staging of a step's inputs and output
# ---------------------------------------------------------------------------
class _Staging:
    """Double-buffered device copies of a step's host inputs and of its
    output, on two side streams: the uploads of step i+1 and the download of
    step i run while the compute stream runs step i / i+1.  Buffer set i % 2
    is reused only after the compute that read it (inputs) and the download
    that read it (output) have finished."""

    def __init__(self, device):
        self.device = device
        self.h2d = torch.cuda.Stream(device)
        self.d2h = torch.cuda.Stream(device)
        self.slot = 0
        self.bufs = [{}, {}]
        self.computed = [None, None]    # compute that last read set s is done
        self.downloaded = [None, None]  # download that last read set s's output is done
        # one event of each kind per buffer set, recorded again each time the
        # set comes round (every wait on the previous record is queued by then)
        self.ev_ready = [torch.cuda.Event(), torch.cuda.Event()]
        self.ev_done = [torch.cuda.Event(), torch.cuda.Event()]
        self.ev_dl = [torch.cuda.Event(), torch.cuda.Event()]

    def _buf(self, key, shape, dtype, st):
        b = self.bufs[self.slot].get(key)
        if b is None or tuple(b.shape) != tuple(shape) or b.dtype != dtype:
            b = torch.empty(tuple(shape), dtype=dtype, device=self.device)
            b.record_stream(st)
            b.record_stream(self.h2d)
            b.record_stream(self.d2h)
            self.bufs[self.slot][key] = b
        return b

    def upload(self, st, named):
        """Device tensors for ``named``: device inputs as they are, host ones
        copied on the upload stream; ``st`` waits for the copies."""
        s = self.slot
        out, host = {}, {}
        for k, t in named.items():
            if t is None or t.device == self.device:
                out[k] = t
            else:
                host[k] = t
        if host:
            if self.computed[s] is not None:
                self.h2d.wait_event(self.computed[s])
            for k, t in host.items():
                out[k] = self._buf(k, t.shape, t.dtype, st)
            with torch.cuda.stream(self.h2d):
                for k, t in host.items():
                    out[k].copy_(t, non_blocking=True)
                ready = self.ev_ready[s]
                ready.record(self.h2d)
            st.wait_event(ready)
        return out

    def output(self, st, shape, dtype):
        """This step's device output buffer (free of any pending download)."""
        s = self.slot
        if self.downloaded[s] is not None:
            st.wait_event(self.downloaded[s])
        return self._buf("_out", shape, dtype, st)

    def finish(self, st, res, out):
        """After the step's kernels on ``st``: download into a host ``out`` on
        the download stream; flip to the other buffer set."""
        s = self.slot
        done = self.ev_done[s]
        done.record(st)
        self.computed[s] = done
        if out is not None and out.device != self.device:
            self.d2h.wait_event(done)
            with torch.cuda.stream(self.d2h):
                out.copy_(res, non_blocking=True)
                ev = self.ev_dl[s]
                ev.record(self.d2h)
            self.downloaded[s] = ev
        self.slot ^= 1


# ---------------------------------------------------------------------------
# a paged KV cache: the pool (torch device memory) plus the allocator
# ---------------------------------------------------------------------------
class PagedKVCache:
    """One layer's paged K/V pool on a device, with its block allocator.

    ``step(seq_ids, q, k_new, v_new)`` is one decode step of the hot path:
    the allocator hands out each sequence's slot (and copy-on-write pairs),
    the shared blocks are copied, the new K/V are appended and every
    sequence's query attends over its whole context.  Inputs may live on
    the host (they are copied in) or on the device; the result is returned
    on the inputs' device.
    """

    def __init__(self, num_blocks: int, num_kv_heads: int, head_dim: int, dtype: torch.dtype,
                 device="cuda", free_order: Optional[Sequence[int]] = None, fill=float("nan"),
                 fp8_scales: Optional[Tuple[float, float]] = None):
        """``dtype``: the queries' (and, without ``fp8_scales``, the pool's)
        dtype.  With ``fp8_scales`` = (k_scale, v_scale) the pool holds FP8
        E4M3 codes (half the bytes) written by the quantising append; new
        K/V still arrive in ``dtype``."""
        self.device = torch.device(device)
        self.dtype = dtype
        self.num_blocks, self.Hkv, self.D = int(num_blocks), int(num_kv_heads), int(head_dim)
        shape = (self.num_blocks, self.Hkv, BLOCK_SIZE, self.D)
        self.fp8 = None if fp8_scales is None else (float(fp8_scales[0]), float(fp8_scales[1]))
        if self.fp8 is None:
            self.k = torch.full(shape, fill, dtype=dtype, device=self.device)
            self.v = torch.full(shape, fill, dtype=dtype, device=self.device)
        else:  # unwritten slots hold the NaN code
            self.k = torch.full(shape, 0x7F, dtype=torch.uint8, device=self.device)
            self.v = torch.full(shape, 0x7F, dtype=torch.uint8, device=self.device)
        self.alloc = BlockAllocator(num_blocks, free_order)
        self._ws = torch.empty(0, dtype=torch.uint8, device=self.device)

    def _copy_append(self, pair_shape, x, st) -> None:
        """The step's copy-on-write copies and append: (src, dst, rows)
        copies with a 16-bit pool go in one launch with the append, cut to
        the rows that hold tokens; (src, dst) pairs copy whole blocks."""
        n = pair_shape[0]
        if n and pair_shape[1] == 3 and self.fp8 is None:
            kv_append_copy(x["k"], x["v"], self.k, self.v, x["slots"], x["pairs"], st)
            return
        if n:
            copy_blocks(self.k, self.v, x["pairs"][:, :2].contiguous(), st)
        self._append(x["k"], x["v"], x["slots"], st)

    def _append(self, k: torch.Tensor, v: torch.Tensor, slots: torch.Tensor, stream) -> None:
        if self.fp8 is None:
            kv_append(k, v, self.k, self.v, slots, stream)
        else:
            kv_append_fp8(k, v, self.k, self.v, slots, self.fp8[0], self.fp8[1], stream)

    def workspace(self, nbytes: int) -> torch.Tensor:
        if self._ws.numel() < nbytes:
            self._ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self._ws

    # bookkeeping passthroughs
    def add_seq(self, sid):
        self.alloc.add_seq(sid)

    def fork(self, parent, child):
        self.alloc.fork(parent, child)

    def free_seq(self, sid):
        self.alloc.free_seq(sid)

    # preemption by swapping
    def enable_swap(self, num_host_blocks: int) -> None:
        """Give the cache a pinned host pool of ``num_host_blocks`` blocks."""
        shape = (int(num_host_blocks), self.Hkv, BLOCK_SIZE, self.D)
        self.host_k = torch.empty(shape, dtype=self.k.dtype, pin_memory=True)
        self.host_v = torch.empty(shape, dtype=self.k.dtype, pin_memory=True)
        self.alloc.set_host_pool(num_host_blocks)

    @_traced("pkv.swap_out")
    def swap_out(self, seq_ids: Sequence[int], stream=None) -> np.ndarray:
        """Preempt sequences: their blocks go to the host pool (copied on the
        stream before anything later on it can reuse the released blocks)."""
        pairs = self.alloc.swap_out(seq_ids)
        if len(pairs):
            swap_blocks(self.host_k, self.host_v, self.k, self.v,
                        torch.from_numpy(np.ascontiguousarray(pairs)).to(self.device), stream, self.device)
        return pairs

    @_traced("pkv.swap_in")
    def swap_in(self, seq_ids: Sequence[int], stream=None) -> np.ndarray:
        """Bring preempted sequences back into the device pool."""
        pairs = self.alloc.swap_in(seq_ids)
        if len(pairs):
            swap_blocks(self.k, self.v, self.host_k, self.host_v,
                        torch.from_numpy(np.ascontiguousarray(pairs)).to(self.device), stream, self.device)
        return pairs

    def prefill(self, sid: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> np.ndarray:
        """Append n tokens' K/V ([n, Hkv, D]) to one sequence."""
        slots, pairs = self.alloc.append_tokens(sid, k.shape[0])
        if len(pairs):
            copy_blocks(self.k, self.v, torch.from_numpy(pairs).to(self.device), stream)
        self._append(k.to(self.device), v.to(self.device), torch.from_numpy(slots).to(self.device), stream)
        return slots

    @_traced("pkv.plan_step")
    def plan_step(self, seq_ids: Sequence[int], width: Optional[int] = None):
        """Host part of a decode step: slots, CoW pairs, tables, lengths."""
        slots, pairs = self.alloc.step(seq_ids)
        copy_blocks_check(pairs, self.num_blocks)
        if width is None:
            width = max(1, max(len(self.alloc.block_table(s)[0]) for s in seq_ids)) if len(seq_ids) else 1
        tables, lens = self.alloc.block_tables(seq_ids, width, self.num_blocks)
        return slots, pairs, tables, lens

    @_traced("pkv.run_step")
    def run_step(self, slot_mapping: torch.Tensor, cow_pairs: torch.Tensor, block_tables: torch.Tensor,
                 context_lens: torch.Tensor, max_context_len: int, q: torch.Tensor, k_new: torch.Tensor,
                 v_new: torch.Tensor, out: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                 partition: int = 0, stream=None, prefix_blocks: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Device part of a decode step: copy-on-write copies, append, decode.

        ``cow_pairs``: int32 [n, 2] (src, dst) whole-block copies, or [n, 3]
        (src, dst, rows) from ``cow_copy_rows``: the copies cut to the rows
        that hold tokens.  With [n, 3] copies (or none) the step goes through
        pkv_decode_step (16-bit pools) or pkv_decode_step_fp8: without a
        shared prefix it is one decode launch, each sequence's copy and
        append made by the warp that then stages its last page (so too in
        the FP8 cascade's suffix pass).
        Inputs may be host tensors (pinned for asynchronous copies) or
        device tensors.  Host inputs are uploaded, and a host ``out`` is
        filled, on two side streams with double-buffered device copies, so a
        step's transfers overlap the previous / next step's kernels; call
        ``wait_downloads`` (or synchronise the device) before reading a host
        ``out``.  With ``prefix_blocks`` (int32, the blocks every sequence's
        table starts with) the cascade decode reads that shared prefix once.
        Returns the device output (valid until the call after next reuses
        its buffer, unless ``out`` is a device tensor).
        """
        dev = self.device
        st = torch.cuda.current_stream(dev) if stream is None else stream
        stg = self._staging()
        x = stg.upload(st, {"slots": slot_mapping, "pairs": cow_pairs, "tables": block_tables,
                            "lens": context_lens, "q": q, "k": k_new, "v": v_new, "prefix": prefix_blocks})
        with torch.cuda.stream(st):
            B, hq = q.shape[0], q.shape[1]
            res = out if (out is not None and out.device == dev) else stg.output(st, q.shape, self.dtype)
            sc = (1.0 / math.sqrt(self.D)) if scale is None else scale
            # the step through pkv_decode_step: a plain decode takes its copies
            # and append into its own launch; the cascade overlaps their
            # launch, waiting for it only at each sequence's last page
            cut = cow_pairs.shape[0] == 0 or cow_pairs.shape[1] == 3
            fused = self.fp8 is None and self.dtype != torch.float32 and cut
            pp = 0 if prefix_blocks is None else int(prefix_blocks.numel())
            if self.fp8 is not None and cut:
                ws = self.workspace(decode_prefix_fp8_workspace_bytes(B, hq, self.Hkv, self.D, max_context_len, pp,
                                                                      partition) if pp
                                    else decode_workspace_bytes(B, hq, self.D, max_context_len, partition))
                decode_step_fp8(x["q"], self.k, self.v, x["k"], x["v"], x["slots"],
                                x["pairs"] if cow_pairs.shape[0] else None, x["tables"], x["lens"], max_context_len,
                                sc, self.fp8[0], self.fp8[1], prefix_blocks=x["prefix"] if pp else None, out=res,
                                workspace=ws, partition=partition, stream=st)
                stg.finish(st, res, out)
                return res
            if fused:
                ws = self.workspace(decode_prefix_workspace_bytes(B, hq, self.D, max_context_len, pp, partition) if pp
                                    else decode_workspace_bytes(B, hq, self.D, max_context_len, partition))
                decode_step(x["q"], self.k, self.v, x["k"], x["v"], x["slots"],
                            x["pairs"] if cow_pairs.shape[0] else None, x["tables"], x["lens"], max_context_len, sc,
                            prefix_blocks=x["prefix"] if pp else None, out=res, workspace=ws, partition=partition,
                            stream=st)
                stg.finish(st, res, out)
                return res
            self._copy_append(cow_pairs.shape, x, st)
            if self.fp8 is not None and prefix_blocks is not None and prefix_blocks.numel() > 0:
                ws = self.workspace(decode_prefix_fp8_workspace_bytes(B, hq, self.Hkv, self.D, max_context_len,
                                                                      prefix_blocks.numel(), partition))
                paged_attention_decode_prefix_fp8(x["q"], self.k, self.v, x["tables"], x["lens"], max_context_len,
                                                  x["prefix"], sc, self.fp8[0], self.fp8[1], out=res, workspace=ws,
                                                  partition=partition, stream=st)
            elif self.fp8 is not None:
                ws = self.workspace(decode_workspace_bytes(B, hq, self.D, max_context_len, partition))
                paged_attention_decode_fp8(x["q"], self.k, self.v, x["tables"], x["lens"], max_context_len, sc,
                                           self.fp8[0], self.fp8[1], out=res, workspace=ws, partition=partition,
                                           stream=st)
            elif prefix_blocks is not None and prefix_blocks.numel() > 0:
                ws = self.workspace(decode_prefix_workspace_bytes(B, hq, self.D, max_context_len,
                                                                  prefix_blocks.numel(), partition))
                paged_attention_decode_prefix(x["q"], self.k, self.v, x["tables"], x["lens"], max_context_len,
                                              x["prefix"], sc, out=res, workspace=ws, partition=partition,
                                              stream=st)
            else:
                ws = self.workspace(decode_workspace_bytes(B, hq, self.D, max_context_len, partition))
                paged_attention_decode(x["q"], self.k, self.v, x["tables"], x["lens"], max_context_len, sc,
                                       out=res, workspace=ws, partition=partition, stream=st)
        stg.finish(st, res, out)
        return res

    def _staging(self) -> "_Staging":
        stg = getattr(self, "_stg", None)
        if stg is None:
            stg = _Staging(self.device)
            self._stg = stg
        return stg

    def staging_after(self, stream=None) -> None:
        """Order the staging streams' next copies after the work already on
        ``stream`` (default: current), e.g. after a timing event."""
        st = torch.cuda.current_stream(self.device) if stream is None else stream
        stg = self._staging()
        stg.h2d.wait_stream(st)
        stg.d2h.wait_stream(st)

    def wait_downloads(self, stream=None) -> None:
        """Make ``stream`` (default: current) wait for the outputs that
        run_step / run_multi_step are still copying to host tensors."""
        stg = getattr(self, "_stg", None)
        if stg is not None:
            st = torch.cuda.current_stream(self.device) if stream is None else stream
            st.wait_stream(stg.d2h)

    @_traced("pkv.plan_multi_step")
    def plan_multi_step(self, seq_ids: Sequence[int], n_new: Sequence[int], width: Optional[int] = None):
        """Host part of a multi-token step: append n_new[i] tokens to each
        sequence (in order); returns slots [sum n], CoW pairs [k, 2],
        query_start [B + 1], tables and lengths.  Each sequence's append is
        all or nothing; a failure leaves earlier sequences' appends done."""
        slots, pairs = [], []
        for sid, n in zip(seq_ids, n_new):
            s_, p_ = self.alloc.append_tokens(sid, int(n))
            slots.append(s_)
            if len(p_):
                pairs.append(p_)
        slots = np.concatenate(slots) if slots else np.zeros(0, dtype=np.int64)
        pairs = np.concatenate(pairs).astype(np.int32) if pairs else np.zeros((0, 2), dtype=np.int32)
        copy_blocks_check(pairs, self.num_blocks)
        qs = np.concatenate([[0], np.cumsum(np.asarray(n_new, dtype=np.int64))]).astype(np.int32)
        if width is None:
            width = max(1, max(len(self.alloc.block_table(s)[0]) for s in seq_ids)) if len(seq_ids) else 1
        tables, lens = self.alloc.block_tables(seq_ids, width, self.num_blocks)
        return slots, pairs, qs, tables, lens

    @_traced("pkv.run_multi_step")
    def run_multi_step(self, slot_mapping: torch.Tensor, cow_pairs: torch.Tensor, block_tables: torch.Tensor,
                       context_lens: torch.Tensor, max_context_len: int, query_start: torch.Tensor,
                       max_query_len: int, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                       out: Optional[torch.Tensor] = None, scale: Optional[float] = None, partition: int = 0,
                       stream=None) -> torch.Tensor:
        """Device part of a multi-token step (speculative verification or a
        prefill chunk): copy-on-write copies, append of every new token,
        causal attention of each new token over its sequence.  Host inputs
        are copied in (pinned: asynchronously); a host ``out`` receives the
        result asynchronously.  Returns the device output [T, Hq, D]."""
        dev = self.device
        st = torch.cuda.current_stream(dev) if stream is None else stream
        stg = self._staging()
        x = stg.upload(st, {"slots": slot_mapping, "pairs": cow_pairs, "tables": block_tables, "lens": context_lens,
                            "qs": query_start, "q": q, "k": k_new, "v": v_new})
        with torch.cuda.stream(st):
            self._copy_append(cow_pairs.shape, x, st)
            res = out if (out is not None and out.device == dev) else stg.output(st, q.shape, self.dtype)
            sc = (1.0 / math.sqrt(self.D)) if scale is None else scale
            ws = self.workspace(multi_workspace_bytes(q.shape[0], q.shape[1], self.D, max_context_len, partition))
            if self.fp8 is not None:
                paged_attention_multi_fp8(x["q"], self.k, self.v, x["tables"], x["lens"], x["qs"], max_context_len,
                                          max_query_len, sc, self.fp8[0], self.fp8[1], out=res, workspace=ws,
                                          partition=partition, stream=st)
            else:
                paged_attention_multi(x["q"], self.k, self.v, x["tables"], x["lens"], x["qs"], max_context_len,
                                      max_query_len, sc, out=res, workspace=ws, partition=partition, stream=st)
        stg.finish(st, res, out)
        return res

    @_traced("pkv.step")
    def step(self, seq_ids: Sequence[int], q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
             scale: Optional[float] = None, partition: int = 0, stream=None) -> torch.Tensor:
        """Host plan (allocator) + device step; returns the output on q's device."""
        slots, pairs, tables, lens = self.plan_step(seq_ids)
        max_ctx = int(lens.max()) if len(lens) else 0
        pp = cascade_prefix_pages(tables, lens, self.dtype)
        prefix = torch.from_numpy(np.ascontiguousarray(tables[0, :pp])) if pp else None
        copies = cow_copy_rows(pairs, slots)  # copy only the rows that hold tokens
        out = self.run_step(torch.from_numpy(slots), torch.from_numpy(copies),
                            torch.from_numpy(np.ascontiguousarray(tables)), torch.from_numpy(lens), max_ctx,
                            q, k_new, v_new, scale=scale, partition=partition, stream=stream,
                            prefix_blocks=prefix)
        return out.clone() if q.device == self.device else out.to(q.device)


def paged_attention_decode_static_ws(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                     block_tables: torch.Tensor, context_lens: torch.Tensor,
                                     max_context_len: int, scale: float, out: Optional[torch.Tensor] = None,
                                     partition: int = 0, stream=None) -> torch.Tensor:
    """``paged_attention_decode`` for callers that must not allocate device
    memory: the split-K scratch is a fixed area the library holds on each
    device (``_lib.STATIC_WORKSPACE_BYTES``), shared by all calls on that
    device.  Raises PkvError (invalid argument) when the call needs more
    scratch than that.  Pass ``out`` to avoid the one allocation this
    wrapper would otherwise make."""
    nb, hkv, d = _cache_dims(k_cache, v_cache)
    if q.dim() != 3 or q.shape[2] != d or q.dtype != k_cache.dtype:
        raise ValueError("q must be [B, Hq, D] in the cache dtype")
    B, hq, _ = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    if out is None:
        out = torch.empty_like(q)
    check(lib.pkv_paged_attention_decode_static_ws(
        _dev(out, "out", q.dtype), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len), B, hq, hkv, d, nb,
        float(scale), int(partition), _DT[k_cache.dtype], _stream(stream, q.device)),
        "pkv_paged_attention_decode_static_ws")
    return out
