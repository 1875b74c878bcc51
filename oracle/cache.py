"""Reference paged KV cache: the slot-mapped append and the block copy
(oracle only).

Layout: k_cache / v_cache [num_blocks, Hkv, block_size, D] in the storage
format.  A slot names one token position in the pool:
slot = physical_block * block_size + offset.  A negative slot is padding and
writes nothing.

* append -- "vLLM + PagedAttention：打造高并发LLM推理引擎", "它是怎么工作的":
  each request's page table records which block its n-th token lives in,
  and a growing sequence only ever writes its new token's slot (old data is
  never copied).
* copy_blocks -- "PagedAttention 与 vLLM 推理加速" §3.2(3): a shared block is
  copied only when a writer is about to append into it (copy-on-write).
* swap_blocks -- "LLM Systems 24 ..." §3, conclusion: a preempted request's
  blocks are swapped out of the device pool and back in later; a block of
  one pool is copied whole into a block of another pool of the same shape.
"""
import numpy as np

from .storage import nan_fill


class RefCache:
    def __init__(self, num_blocks: int, Hkv: int, D: int, dtype: str, block_size: int = 16):
        self.dtype = dtype
        self.block_size = block_size
        shape = (num_blocks, Hkv, block_size, D)
        # every slot starts as NaN so a read of an unwritten slot shows up
        self.k = nan_fill(shape, dtype)
        self.v = nan_fill(shape, dtype)

    def append(self, k_new: np.ndarray, v_new: np.ndarray, slots: np.ndarray) -> None:
        """cache[slot // bs, :, slot % bs, :] = new[i] for every slot >= 0."""
        slots = np.asarray(slots, dtype=np.int64)
        for i, s in enumerate(slots):
            if s < 0:
                continue
            blk, off = divmod(int(s), self.block_size)
            self.k[blk, :, off, :] = k_new[i]
            self.v[blk, :, off, :] = v_new[i]

    def append_many(self, k_new: np.ndarray, v_new: np.ndarray, slots: np.ndarray) -> None:
        """The same writes as ``append`` done with one fancy-index store.

        Slots are distinct within a call, so the order of the writes does
        not matter.
        """
        slots = np.asarray(slots, dtype=np.int64)
        keep = slots >= 0
        blk = slots[keep] // self.block_size
        off = slots[keep] % self.block_size
        self.k[blk, :, off, :] = k_new[keep]
        self.v[blk, :, off, :] = v_new[keep]

    def append_fp8(self, k_new: np.ndarray, v_new: np.ndarray, slots: np.ndarray, src_dtype: str,
                   k_scale: float, v_scale: float) -> None:
        """An FP8 cache's append: each new K (V) element x (storage format
        ``src_dtype``) is stored as the E4M3 code of x / k_scale (v_scale),
        the division in float32 (``oracle.fp8.quantize``)."""
        from .fp8 import quantize
        from .storage import widen
        assert self.dtype == "e4m3"
        kq = quantize(widen(k_new, src_dtype).astype(np.float32), k_scale)
        vq = quantize(widen(v_new, src_dtype).astype(np.float32), v_scale)
        self.append(kq, vq, slots)

    def copy_rows_then_append(self, copies, k_new, v_new, slots) -> None:
        """The step's copy-on-write and append with the copies cut to the
        rows that hold tokens: for each (src, dst, rows), rows 0..rows-1 of
        dst receive src's, then the new tokens go to their slots.  Rows of
        dst at or past ``rows`` that no token is written into keep what they
        held (no token of the sequence lives there)."""
        for src, dst, rows in copies:
            self.k[int(dst), :, :int(rows)] = self.k[int(src), :, :int(rows)]
            self.v[int(dst), :, :int(rows)] = self.v[int(src), :, :int(rows)]
        self.append(k_new, v_new, slots)

    def copy_blocks(self, pairs) -> None:
        """cache[dst] = cache[src] for each (src, dst), K and V."""
        for src, dst in pairs:
            self.k[int(dst)] = self.k[int(src)]
            self.v[int(dst)] = self.v[int(src)]


def swap_blocks(dst: "RefCache", src: "RefCache", pairs) -> None:
    """dst[d] = src[s] for each (s, d), K and V (pools of the same shape)."""
    for s, d in pairs:
        dst.k[int(d)] = src.k[int(s)]
        dst.v[int(d)] = src.v[int(s)]
