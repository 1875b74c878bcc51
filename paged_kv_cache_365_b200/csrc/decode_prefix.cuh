// Shared-prefix (cascade) decode: the merge of prefix and suffix partials.
//
// "PagedAttention 与 vLLM 推理加速" §3.2(3): requests with the same system
// prompt map the same physical blocks (stored once).  When the sequences of
// a batch start with the same prefix blocks, the cascade launch of the
// tensor-core kernel (decode_mma.cuh) reads each shared (block, kv-head)
// tile from HBM once: its prefix-role CTAs attend groups of 8 queries (of
// different sequences) to a chunk of the prefix, its sequence-role CTAs
// cover each sequence's own suffix.  This kernel combines the prefix
// chunks' and the suffix partitions' partial results with the same
// log-sum-exp rule as the split-K merge.  The result is the same attention
// (up to rounding); only the order of the work changes.
#pragma once

#include "decode_mma.cuh"

namespace pkv {

// Merge for the cascade: per (query head, sequence b = blockIdx.y), the
// prefix chunks (when the sequence starts with the prefix) then the suffix
// partitions, in order, rescaled to their common max.  HPC heads per CTA.
template <typename T, int D, int HPC>
__global__ void __launch_bounds__(kMergeWarps * 32) paged_decode_prefix_merge_kernel(const DecodeArgs a) {
  pdl_enter();
  const int hs = (threadIdx.x >> 5) / (kMergeWarps / HPC);
  const int h = blockIdx.x * HPC + hs;
  const int b = blockIdx.y;
  int ctx = a.context_lens[b];
  ctx = ctx < 0 ? 0 : (ctx > a.max_ctx ? a.max_ctx : ctx);
  const bool conforming = a.conform[b] != 0;
  const int tok_begin = conforming ? a.prefix_pages * kBlockSize : 0;
  const int n_suf = (ctx - tok_begin + a.partition - 1) / a.partition;
  const int n_pre = conforming ? a.num_chunks : 0;
  const bool skip = h >= a.num_q_heads;  // head slot past Hq (the barriers need every warp)
  const int hh = skip ? 0 : h;
  const size_t pre0 = (static_cast<size_t>(b) * a.num_q_heads + hh) * a.num_chunks;
  const size_t suf0 = (static_cast<size_t>(b) * a.num_q_heads + hh) * a.num_parts;
  __shared__ T sink[D];
  T* out = skip ? sink : reinterpret_cast<T*>(a.out) + (static_cast<size_t>(b) * a.num_q_heads + hh) * D;
  merge_partials<T, D, HPC>(
      skip ? 0 : n_pre + n_suf,
      [&](int p) { return p < n_pre ? a.wp_ml[pre0 + p] : a.ws_ml[suf0 + (p - n_pre)]; },
      [&](int p) { return p < n_pre ? a.wp_o + (pre0 + p) * D : a.ws_o + (suf0 + (p - n_pre)) * D; }, out, hs);
}

}  // namespace pkv
