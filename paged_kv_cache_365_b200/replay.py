"""Rebuild a paged cache on the device from an op log.

An op log is a list of ``('add', sid)``, ``('append', sid, n)``,
``('fork', parent, child)`` and ``('free', sid)``; the i-th token appended
by the log carries ``k_tokens[i]`` / ``v_tokens[i]``.  The log goes through
the library's allocator; appends are batched into as few ``kv_append``
launches as possible (a copy-on-write pair flushes the pending appends so
the copy sees every token written before it).
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from .api import PagedKVCache, copy_blocks, kv_append

_TORCH = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def to_torch(arr: np.ndarray, dtype: str, device) -> torch.Tensor:
    """Storage array (bf16 as uint16 bits) -> torch tensor of that dtype."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr))
    return t.to(device)


def replay_ops(cache: PagedKVCache, ops, k_tokens: torch.Tensor, v_tokens: torch.Tensor,
               stream=None) -> np.ndarray:
    """Apply ``ops``; return every appended token's slot (in log order)."""
    dev = cache.device
    n_total = sum(op[2] for op in ops if op[0] == "append")
    all_slots = np.empty(n_total, dtype=np.int64)
    cursor = 0
    pending_from = 0

    def flush(upto: int):
        nonlocal pending_from
        if upto > pending_from:
            kv_append(k_tokens[pending_from:upto], v_tokens[pending_from:upto], cache.k, cache.v,
                      torch.from_numpy(all_slots[pending_from:upto]).to(dev), stream)
            pending_from = upto

    for op in ops:
        kind = op[0]
        if kind == "add":
            cache.add_seq(op[1])
        elif kind == "fork":
            cache.fork(op[1], op[2])
        elif kind == "free":
            cache.free_seq(op[1])
        elif kind == "append":
            sid, n = op[1], op[2]
            slots, pairs = cache.alloc.append_tokens(sid, n)
            if len(pairs):
                flush(cursor)
                copy_blocks(cache.k, cache.v, torch.from_numpy(np.ascontiguousarray(pairs)).to(dev), stream)
            all_slots[cursor:cursor + n] = slots
            cursor += n
        else:
            raise ValueError(op)
    flush(cursor)
    return all_slots


def build_step(wl, values: Dict[str, np.ndarray], device="cuda", fill=float("nan"),
               device_values: Optional[Dict[str, torch.Tensor]] = None, stream=None):
    """Rebuild ``wl``'s cache on the device and plan its decode step.

    Returns a dict with the cache, the step's device inputs (q, k_new, v_new,
    slot_mapping, cow pairs, block_tables, context_lens) and host copies of
    the plan.  The step's copy / append / decode are NOT run.
    """
    dt = _TORCH[wl.dtype]
    cache = PagedKVCache(wl.num_blocks, wl.Hkv, wl.D, dt, device, wl.free_order, fill=fill)
    dv = device_values or {}
    get = lambda k: dv[k] if k in dv else to_torch(values[k], wl.dtype, device)  # noqa: E731
    k_tok, v_tok = get("k_tokens"), get("v_tokens")
    prefill_slots = replay_ops(cache, wl.ops, k_tok, v_tok, stream)
    del k_tok, v_tok
    mask = np.asarray(wl.step_append_mask)
    ids = [int(s) for s, m in zip(wl.step_seqs, mask) if m]
    slots, pairs = cache.alloc.step(ids)
    step_slots = np.full(wl.B, -1, dtype=np.int64)
    step_slots[mask] = slots
    all_ids = [int(s) for s in wl.step_seqs]
    width = max(1, max(len(cache.alloc.block_table(s)[0]) for s in all_ids))
    tables, lens = cache.alloc.block_tables(all_ids, width, wl.num_blocks + 12345)
    dev = cache.device
    return {
        "cache": cache,
        "q": get("q"),
        "k_new": get("k_new"),
        "v_new": get("v_new"),
        "slot_mapping": torch.from_numpy(step_slots).to(dev),
        "cow_pairs": torch.from_numpy(np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)).to(dev),
        "block_tables": torch.from_numpy(np.ascontiguousarray(tables)).to(dev),
        "context_lens": torch.from_numpy(np.ascontiguousarray(lens)).to(dev),
        "max_context_len": int(lens.max()) if len(lens) else 0,
        "host": {"step_slots": step_slots, "cow_pairs": pairs, "block_tables": tables,
                 "context_lens": lens, "prefill_slots": prefill_slots},
    }


def build_multi_step(wl, n_new: int, device="cuda", fill=float("nan"),
                     device_values: Optional[Dict[str, torch.Tensor]] = None, stream=None, seed: int = 0):
    """Rebuild ``wl``'s cache on the device (its op log, without the decode
    step) and plan a multi-token step: ``n_new`` new tokens for each of the
    step's sequences.  New q / K / V are seeded N(0,1) draws on the device.
    The step's copy / append / attention are NOT run."""
    dt = _TORCH[wl.dtype]
    cache = PagedKVCache(wl.num_blocks, wl.Hkv, wl.D, dt, device, wl.free_order, fill=fill)
    dv = device_values or {}
    replay_ops(cache, wl.ops, dv["k_tokens"], dv["v_tokens"], stream)
    ids = [int(s) for s in wl.step_seqs]
    slots, pairs, qs, tables, lens = cache.plan_multi_step(ids, [n_new] * len(ids), None)
    dev = cache.device
    T = int(qs[-1])
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed) * 104729 + 3)
    draw = lambda *shape: torch.randn(*shape, generator=g, device=dev, dtype=torch.float32).to(dt)  # noqa: E731
    return {
        "cache": cache,
        "q": draw(T, wl.Hq, wl.D),
        "k_new": draw(T, wl.Hkv, wl.D),
        "v_new": draw(T, wl.Hkv, wl.D),
        "slot_mapping": torch.from_numpy(slots).to(dev),
        "cow_pairs": torch.from_numpy(np.ascontiguousarray(pairs)).to(dev),
        "block_tables": torch.from_numpy(np.ascontiguousarray(tables)).to(dev),
        "context_lens": torch.from_numpy(np.ascontiguousarray(lens)).to(dev),
        "query_start": torch.from_numpy(qs).to(dev),
        "max_context_len": int(lens.max()) if len(lens) else 0,
        "max_query_len": int(n_new),
        "host": {"slots": slots, "cow_pairs": pairs, "block_tables": tables, "context_lens": lens,
                 "query_start": qs},
    }
