"""Paged decode attention, the plain definition, in float64 (oracle only).

For sequence b and query head h (kv-head g = h // (Hq // Hkv)), with
n = context_lens[b] tokens:

  K_j = k_cache[block_tables[b][j // bs], g, j % bs, :]     (V_j likewise)
  s_j = scale * sum_d q[b,h,d] * K_j[d]
  out[b,h,:] = sum_j softmax(s)_j * V_j

"PagedAttention 与 vLLM 推理加速" §2.3: the block table maps each logical
page to a physical block, the kernel reads every K of the sequence's blocks
through it and Q x K gives the attention scores; §1: decode step t attends
over the K/V of every token so far, itself included.  The softmax is the
standard one, computed max-subtracted so exp never overflows.  A sequence
with no tokens yields zeros.  Block-table entries past the sequence's last
page, and the unused slots of its last block, are never read.

Several query tokens per sequence (``paged_multi``): "PagedAttention 与 vLLM
推理加速" §6 (the large model verifies the small model's guessed tokens --
several new tokens of one sequence scored in one pass) and "LLM Systems 24
..." §2.2.1.3 (batches that mix prefill chunks and decode steps).  Query
token i of a sequence with n new tokens sits at position ctx - n + i and,
by §1's rule (a token attends over every token so far, itself included),
attends over positions 0..ctx - n + i and no later ones.
"""
import numpy as np

from .storage import widen


def _gather(cache: np.ndarray, pages: np.ndarray, g: int, n: int, bs: int) -> np.ndarray:
    """Rows 0..n-1 of kv-head g in logical order: page j//bs, offset j%bs."""
    tiles = cache[pages, g]  # [n_pages, bs, D]
    return tiles.reshape(-1, tiles.shape[-1])[:n]


def decode_head(q_row: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float) -> np.ndarray:
    """Single-query softmax attention over float64 rows ``keys``/``values``."""
    if keys.shape[0] == 0:
        return np.zeros(values.shape[-1], dtype=np.float64)
    s = scale * (keys @ q_row)
    s = s - s.max()
    p = np.exp(s)
    p = p / p.sum()
    return p @ values


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale, dtype,
                 block_size=16, seqs=None, kv_dtype=None, k_scale=1.0, v_scale=1.0):
    """float64 output [B, Hq, D] (rows not in ``seqs`` are left NaN).

    q: [B,Hq,D]; k_cache/v_cache: [num_blocks,Hkv,block_size,D] in the
    storage format ``dtype`` ('f32', 'f16', or 'bf16' as uint16 bits);
    block_tables: int [B, max_blocks]; context_lens: int [B].
    ``seqs`` restricts the work to those sequence indices (sampled checks).
    An FP8 cache: ``kv_dtype='e4m3'`` (q stays in ``dtype``); a stored K
    value is its code's value times ``k_scale`` (V alike).
    """
    kvd = dtype if kv_dtype is None else kv_dtype
    B, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    out = np.full((B, Hq, D), np.nan, dtype=np.float64)
    for b in (range(B) if seqs is None else seqs):
        n = int(context_lens[b])
        n_pages = -(-n // block_size)
        pages = np.asarray(block_tables[b][:n_pages], dtype=np.int64)
        qb = widen(q[b], dtype)
        for g in range(Hkv):
            keys = widen(_gather(k_cache, pages, g, n, block_size), kvd) * k_scale
            values = widen(_gather(v_cache, pages, g, n, block_size), kvd) * v_scale
            for h in range(g * G, (g + 1) * G):
                out[b, h] = decode_head(qb[h], keys, values, scale)
    return out


def paged_multi(q, k_cache, v_cache, block_tables, context_lens, query_start, scale, dtype,
                block_size=16, seqs=None, kv_dtype=None, k_scale=1.0, v_scale=1.0):
    """float64 output [T, Hq, D] for T = query_start[-1] query tokens.

    Rows query_start[b] .. query_start[b+1]-1 of q [T, Hq, D] are sequence
    b's n_b new tokens, the last n_b of its context_lens[b] tokens; row
    query_start[b] + i attends over the sequence's tokens 0 .. ctx - n_b + i.
    A row whose position would be negative (n_b > ctx) yields zeros.
    ``seqs`` restricts the work to those sequences (other rows stay NaN).
    An FP8 cache as in ``paged_decode``: ``kv_dtype='e4m3'`` (q stays in
    ``dtype``), a stored K value is its code's value times ``k_scale`` (V
    alike).
    """
    kvd = dtype if kv_dtype is None else kv_dtype
    T, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    out = np.full((T, Hq, D), np.nan, dtype=np.float64)
    B = len(context_lens)
    for b in (range(B) if seqs is None else seqs):
        n = int(context_lens[b])
        r0, r1 = int(query_start[b]), int(query_start[b + 1])
        nq = r1 - r0
        n_pages = -(-n // block_size)
        pages = np.asarray(block_tables[b][:n_pages], dtype=np.int64)
        for g in range(Hkv):
            keys = widen(_gather(k_cache, pages, g, n, block_size), kvd) * k_scale
            values = widen(_gather(v_cache, pages, g, n, block_size), kvd) * v_scale
            for i in range(nq):
                pos = n - nq + i
                qi = widen(q[r0 + i], dtype)
                for h in range(g * G, (g + 1) * G):
                    if pos < 0:
                        out[r0 + i, h] = 0.0
                    else:
                        out[r0 + i, h] = decode_head(qi[h], keys[:pos + 1], values[:pos + 1], scale)
    return out
