// Host planning of a step, on top of the allocator's output: which rows a
// copy-on-write copy must move, and which leading blocks a batch shares
// (the prefix the cascade decode reads once).  Plain host code over host
// arrays; no CUDA call.
//
// Copy-on-write ("PagedAttention 与 vLLM 推理加速" §3.2(3); "LLM Systems 24:
// Efficient LLM Inference with PagedAttention and vLLM" §3): a shared block
// is copied before a sharer appends into it.  The block was partial (a full
// shared block is never copied), so only its first rows hold tokens; the
// first row the step writes into the new block is where the copy can stop.
//
// Shared prefix ("PagedAttention 与 vLLM 推理加速" §3.2(3)): requests with
// the same system prompt map the same physical blocks at the start of their
// block tables (§2.3).

#include <cstdint>
#include <vector>

#include "pkv.h"

extern "C" {

pkv_status pkv_cow_copy_rows(const int32_t* pairs, int num_pairs, const int64_t* slots, int num_slots,
                             int32_t* copies) {
  if (num_pairs < 0 || num_slots < 0 || (num_pairs > 0 && (pairs == nullptr || copies == nullptr)) ||
      (num_slots > 0 && slots == nullptr))
    return PKV_EINVAL;
  for (int i = 0; i < num_pairs; ++i)
    if (pairs[2 * i] < 0 || pairs[2 * i + 1] < 0) return PKV_EINVAL;
  for (int i = 0; i < num_pairs; ++i) {
    const int32_t src = pairs[2 * i], dst = pairs[2 * i + 1];
    int32_t rows = PKV_BLOCK_SIZE;
    for (int j = 0; j < num_slots; ++j) {
      const int64_t s = slots[j];
      if (s < 0 || s / PKV_BLOCK_SIZE != dst) continue;
      const int32_t r = static_cast<int32_t>(s % PKV_BLOCK_SIZE);
      if (r < rows) rows = r;
    }
    copies[3 * i] = src;
    copies[3 * i + 1] = dst;
    copies[3 * i + 2] = rows;
  }
  return PKV_OK;
}

pkv_status pkv_alloc_step_copies(pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* slots, int32_t* copies,
                                 int* n_copies) {
  if (a == nullptr || n < 0 || n_copies == nullptr || (n > 0 && copies == nullptr)) return PKV_EINVAL;
  std::vector<int32_t> pairs(2 * static_cast<size_t>(n > 0 ? n : 1));
  int nc = 0;
  const pkv_status st = pkv_alloc_step(a, seq_ids, n, slots, pairs.data(), &nc);
  if (st != PKV_OK) return st;
  *n_copies = nc;
  return pkv_cow_copy_rows(pairs.data(), nc, slots, n, copies);
}

pkv_status pkv_common_prefix_pages(const int32_t* block_tables, int num_seqs, int width,
                                   const int32_t* context_lens, int* prefix_pages) {
  if (prefix_pages == nullptr || num_seqs < 0 || width < 0 ||
      (num_seqs > 0 && (block_tables == nullptr || context_lens == nullptr)))
    return PKV_EINVAL;
  *prefix_pages = 0;
  if (num_seqs < 2) return PKV_OK;
  // pages every sequence fills completely
  int64_t full = width;
  for (int b = 0; b < num_seqs; ++b) {
    if (context_lens[b] < 0) return PKV_EINVAL;
    const int64_t f = context_lens[b] / PKV_BLOCK_SIZE;
    if (f < full) full = f;
  }
  int64_t p = 0;
  for (; p < full; ++p) {
    const int32_t blk = block_tables[p];
    bool same = true;
    for (int b = 1; b < num_seqs && same; ++b) same = block_tables[static_cast<int64_t>(b) * width + p] == blk;
    if (!same) break;
  }
  *prefix_pages = static_cast<int>(p);
  return PKV_OK;
}

pkv_status pkv_cascade_prefix_pages(const int32_t* block_tables, int num_seqs, int width,
                                    const int32_t* context_lens, pkv_dtype dtype, int* prefix_pages) {
  if (prefix_pages == nullptr) return PKV_EINVAL;
  int p = 0;
  const pkv_status st = pkv_common_prefix_pages(block_tables, num_seqs, width, context_lens, &p);
  if (st != PKV_OK) return st;
  const bool eligible = (dtype == PKV_F16 || dtype == PKV_BF16 || dtype == PKV_E4M3) && num_seqs >= PKV_CASCADE_MIN_SEQS &&
                        p >= PKV_CASCADE_MIN_PAGES;
  *prefix_pages = eligible ? p : 0;
  return PKV_OK;
}

}  // extern "C"
