"""Replay a workload's op log through the reference allocator and cache
(oracle only).

``replay`` takes any object with the workload attributes (num_blocks,
free_order, block_size, Hkv, D, dtype, ops, step_seqs, context_lens) and the
drawn values, and returns the state right after the step's appends: the
reference allocator, the reference cache, the step's slots and copy pairs,
and the block tables / context lengths of the step's sequences.
"""
import numpy as np

from .allocator import RefAllocator
from .cache import RefCache

# value written into block-table entries past a sequence's last page; it is
# out of range on purpose, so a reader that strays past the last page fails
TABLE_PAD_OFFSET = 12345


def replay(wl, values):
    alloc = RefAllocator(wl.num_blocks, wl.free_order, wl.block_size)
    cache = RefCache(wl.num_blocks, wl.Hkv, wl.D, wl.dtype, wl.block_size)
    k_tok, v_tok = values["k_tokens"], values["v_tokens"]
    cursor = 0
    prefill_slots = np.empty(wl.n_prefill_tokens, dtype=np.int64)
    for op in wl.ops:
        kind = op[0]
        if kind == "add":
            alloc.add_seq(op[1])
        elif kind == "append":
            sid, n = op[1], op[2]
            slots, cows = alloc.append_tokens(sid, n)
            cache.copy_blocks(cows)
            cache.append_many(k_tok[cursor:cursor + n], v_tok[cursor:cursor + n], slots)
            prefill_slots[cursor:cursor + n] = slots
            cursor += n
        elif kind == "fork":
            alloc.fork(op[1], op[2])
        elif kind == "free":
            alloc.free_seq(op[1])
        else:
            raise ValueError(op)

    mask = np.asarray(wl.step_append_mask)
    step_ids = [int(s) for s, m in zip(wl.step_seqs, mask) if m]
    slots, cows = alloc.step(step_ids)
    step_slots = np.full(len(wl.step_seqs), -1, dtype=np.int64)
    step_slots[mask] = slots
    cow_pairs = np.asarray(cows, dtype=np.int32).reshape(-1, 2)
    cache.copy_blocks(cow_pairs)
    cache.append(values["k_new"], values["v_new"], step_slots)

    tables, lens = [], []
    for sid in wl.step_seqs:
        t, n = alloc.block_table(int(sid))
        tables.append(t)
        lens.append(n)
    width = max(1, max(len(t) for t in tables))
    bt = np.full((len(tables), width), wl.num_blocks + TABLE_PAD_OFFSET, dtype=np.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = t
    return {
        "alloc": alloc,
        "cache": cache,
        "prefill_slots": prefill_slots,
        "step_slots": step_slots,
        "cow_pairs": cow_pairs,
        "block_tables": bt,
        "context_lens": np.asarray(lens, dtype=np.int32),
    }
