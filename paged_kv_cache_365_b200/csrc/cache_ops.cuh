// Slot-mapped append of new tokens' K/V, copy-on-write block copy, and the
// block copy between the device pool and a host pool (swap).
//
// All are bit copies of 16-byte chunks: one thread moves one chunk, so a
// warp moves 512 contiguous bytes of a row (append) or of a block (copy),
// fully coalesced on both sides.
#pragma once

#include "common.cuh"

namespace pkv {

// "vLLM + PagedAttention：打造高并发LLM推理引擎", "它是怎么工作的": token t
// lands in slot s = block * 16 + offset of its sequence's page table; old
// tokens never move.  Chunks [0, total) are K, [total, 2 total) are V, where
// total = num_tokens * Hkv * row_chunks.
__global__ void __launch_bounds__(256)
    kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                     uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                     const int64_t* __restrict__ slots, long long total, int Hkv, int row_chunks,
                     int num_blocks) {
  pdl_enter();
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < 2 * total;
       i += stride) {
    const bool is_v = i >= total;
    const long long j = is_v ? i - total : i;
    const int c = static_cast<int>(j % row_chunks);
    const long long th = j / row_chunks;
    const int h = static_cast<int>(th % Hkv);
    const long long t = th / Hkv;
    const int64_t s = slots[t];
    if (s < 0) continue;  // padding
    const int64_t blk = s / kBlockSize;
    const int off = static_cast<int>(s % kBlockSize);
    if (blk >= num_blocks) {
      raise_error(PKV_ERR_SLOT_RANGE);
      continue;
    }
    const long long dst = ((blk * Hkv + h) * kBlockSize + off) * row_chunks + c;
    if (is_v)
      v_cache[dst] = v_new[j];
    else
      k_cache[dst] = k_new[j];
  }
}

// "PagedAttention 与 vLLM 推理加速" §3.2(3): copy a shared block before a
// writer appends into it.  grid = (chunk groups, pair, K|V).
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                       const int32_t* __restrict__ pairs, long long block_chunks, int num_blocks) {
  pdl_enter();
  constexpr int kUnroll = 4;
  const int p = blockIdx.y;
  const int src = pairs[2 * p];
  const int dst = pairs[2 * p + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_error(PKV_ERR_COPY_RANGE);
    return;
  }
  uint4* cache = blockIdx.z ? v_cache : k_cache;
  const uint4* from = cache + static_cast<size_t>(src) * block_chunks;
  uint4* to = cache + static_cast<size_t>(dst) * block_chunks;
  const long long step = static_cast<long long>(gridDim.x) * blockDim.x * kUnroll;
  for (long long base = static_cast<long long>(blockIdx.x) * blockDim.x * kUnroll + threadIdx.x;
       base < block_chunks; base += step) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long i = base + static_cast<long long>(u) * blockDim.x;
      if (i < block_chunks) v[u] = from[i];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long i = base + static_cast<long long>(u) * blockDim.x;
      if (i < block_chunks) to[i] = v[u];
    }
  }
}

// A decode step's copy-on-write and append in one launch, the copies cut to
// the rows that hold tokens: for each copy (src, dst, rows), rows 0..rows-1
// of dst receive src's (all kv-heads); every token with a slot gets its row.
// The caller gives each copy the first row a token of this call writes into
// dst, so copies and appends touch disjoint rows and need no ordering.
// Grid (x, n_copies + A, 2): z = K | V; y < n_copies: copy y, its
// Hkv * rows * row_chunks chunks over the x CTAs; the other A rows of y
// share the appends.
__global__ void __launch_bounds__(256)
    kv_append_copy_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                          uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                          const int64_t* __restrict__ slots, const int32_t* __restrict__ copies, int n_copies,
                          int n_tok, int Hkv, int row_chunks, int num_blocks) {
  pdl_enter();
  const bool is_v = blockIdx.z != 0;
  uint4* cache = is_v ? v_cache : k_cache;
  const long long per_block = static_cast<long long>(Hkv) * kBlockSize * row_chunks;
  if (static_cast<int>(blockIdx.y) < n_copies) {
    const int p = blockIdx.y;
    const int src = copies[3 * p], dst = copies[3 * p + 1], rows = copies[3 * p + 2];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks || rows < 0 || rows > kBlockSize) {
      if (threadIdx.x == 0 && blockIdx.x == 0 && !is_v) raise_error(PKV_ERR_COPY_RANGE);
      return;
    }
    const int per_head = rows * row_chunks;  // chunks of one head's first `rows` rows
    const int items = Hkv * per_head;
    const uint4* from = cache + static_cast<long long>(src) * per_block;
    uint4* to = cache + static_cast<long long>(dst) * per_block;
    // each thread moves several chunks, kUnroll loads in flight
    constexpr int kUnroll = 4;
    const int step = gridDim.x * blockDim.x;
    for (int t0 = blockIdx.x * blockDim.x + threadIdx.x; t0 < items; t0 += step * kUnroll) {
      uint4 v[kUnroll];
      int off[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int t = t0 + u * step;
        off[u] = -1;
        if (t < items) {
          const int h = t / per_head;
          off[u] = h * kBlockSize * row_chunks + (t - h * per_head);
          v[u] = from[off[u]];
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (off[u] >= 0) to[off[u]] = v[u];
    }
    return;
  }
  const long long items = static_cast<long long>(n_tok) * Hkv * row_chunks;
  const long long stride = static_cast<long long>(gridDim.y - n_copies) * gridDim.x * blockDim.x;
  for (long long j = (static_cast<long long>(blockIdx.y - n_copies) * gridDim.x + blockIdx.x) * blockDim.x +
                     threadIdx.x;
       j < items; j += stride) {
    const int c = static_cast<int>(j % row_chunks);
    const long long th = j / row_chunks;
    const int h = static_cast<int>(th % Hkv);
    const long long t = th / Hkv;
    const int64_t s = slots[t];
    if (s < 0) continue;
    const int64_t blk = s / kBlockSize;
    const int off = static_cast<int>(s % kBlockSize);
    if (blk >= num_blocks) {
      raise_error(PKV_ERR_SLOT_RANGE);
      continue;
    }
    cache[((blk * Hkv + h) * kBlockSize + off) * row_chunks + c] = (is_v ? v_new : k_new)[j];
  }
}

// "LLM Systems 24: Efficient LLM Inference with PagedAttention and vLLM" §3
// (conclusion): a request preempted for lack of KV blocks is swapped out
// and later swapped back in.  dst[d] = src[s] for each pair (s, d), K and V;
// either pool may be page-locked host memory mapped into the device's
// address space (the kernel then reads or writes it over the host link).
// The (pair, K|V, chunk) space is walked by a grid-stride loop with kUnroll
// independent loads in flight per thread before the stores, so a slow link
// still sees enough outstanding requests.
__global__ void __launch_bounds__(256)
    swap_blocks_kernel(uint4* __restrict__ dst_k, uint4* __restrict__ dst_v, const uint4* __restrict__ src_k,
                       const uint4* __restrict__ src_v, const int32_t* __restrict__ pairs, long long block_chunks,
                       long long total /* num_pairs * block_chunks */, int src_blocks, int dst_blocks) {
  pdl_enter();
  constexpr int kUnroll = 4;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long base = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; base < 2 * total;
       base += stride * kUnroll) {
    uint4 v[kUnroll];
    long long to[kUnroll];  // destination chunk; -1: nothing to store
    bool is_v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long i = base + u * stride;
      to[u] = -1;
      is_v[u] = i >= total;
      if (i >= 2 * total) continue;
      const long long j = is_v[u] ? i - total : i;
      const long long p = j / block_chunks;
      const long long c = j - p * block_chunks;
      const int s = pairs[2 * p];
      const int d = pairs[2 * p + 1];
      if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) {
        if (c == 0) raise_error(PKV_ERR_COPY_RANGE);
        continue;
      }
      v[u] = (is_v[u] ? src_v : src_k)[static_cast<long long>(s) * block_chunks + c];
      to[u] = static_cast<long long>(d) * block_chunks + c;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (to[u] >= 0) (is_v[u] ? dst_v : dst_k)[to[u]] = v[u];
    }
  }
}

}  // namespace pkv
