// C ABI of libpkv: argument checks, dispatch to the kernel instantiations,
// launches.  Every host-checkable argument is checked before any CUDA call,
// so a rejected call has no side effect (and works without a GPU).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <unordered_set>

#include <cudaTypedefs.h>

#include "cache_ops.cuh"
#include "decode_fp8.cuh"
#include "decode_launch.cuh"
#include "multi_mma.cuh"
#include "multi_tc.cuh"
#include "pkv.h"

namespace pkv {
__device__ unsigned int g_error_snapshot = 0u;

__global__ void take_error_snapshot_kernel() { g_error_snapshot = atomicExch(&g_error_word, 0u); }

// The staged-copy wait of every kernel, on a barrier that nothing completes:
// it must give up after `limit` cycles and flag PKV_ERR_TIMEOUT.
__global__ void bounded_wait_selftest_kernel(long long limit) {
  __shared__ alignas(8) unsigned long long bar;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncwarp();
  const bool done = __all_sync(kFull, mbar_wait_bounded(b, 0u, limit));
  if (!done && threadIdx.x == 0) raise_error(PKV_ERR_TIMEOUT);
}
}  // namespace pkv

namespace {

// ---- several query tokens per sequence (tensor cores) -----------------------
// The multi-token merge: one CTA per (sequence, kv-head).
template <typename T, int D, int G>
pkv_status launch_multi_merge(const pkv::MultiArgs& a, cudaStream_t st) {
  return launch(pkv::paged_multi_merge_kernel<T, D, G>, dim3(a.num_seqs, a.num_kv_heads), dim3(pkv::kMergeWarps * 32),
                0, st, a);
}

template <typename T, int D, int G, int NT>
pkv_status launch_multi(const pkv::MultiArgs& a, const void* k_cache, const void* v_cache, int num_blocks,
                        cudaStream_t st) {
  constexpr int kStages = kMmaStages;
  using S = pkv::MmaShape<T, D, G, kMmaWarps, kStages>;
  CUtensorMap mk, mv;
  const long long rows = static_cast<long long>(num_blocks) * a.num_kv_heads * PKV_BLOCK_SIZE;
  if (!encode_cache_map(&mk, k_cache, pkv::Mma<T>::kTmaType, D, rows) ||
      !encode_cache_map(&mv, v_cache, pkv::Mma<T>::kTmaType, D, rows))
    return PKV_ECUDA;
  auto kfn = pkv::paged_multi_mma_kernel<T, D, G, NT, kMmaWarps, kStages>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmem)) !=
      cudaSuccess)
    return PKV_ECUDA;
  const dim3 grid(a.num_kv_heads, a.num_seqs * a.tiles, a.num_parts);
  if (launch(kfn, grid, dim3(kMmaWarps * 32), S::kSmem, st, a, mk, mv) != PKV_OK) return PKV_ECUDA;
  if (a.num_parts > 1) return launch_multi_merge<T, D, G>(a, st);
  return PKV_OK;
}

// Up to 16 rows per sequence (max_query_len * G): one tile of 8 NT rows,
// the warps splitting the pages.  Up to 32: one tile of 8 NW rows, one warp
// per 8 rows, the warps sharing the pages (paged_multi_rows_kernel).  More:
// tiles of 64 rows as the MMA's M dimension, 16 per warp
// (paged_multi_fa_kernel).
// Auto partition of the multi-token path: 2048 tokens, 1024 past 4096.
int resolve_multi_partition(int p, long long max_ctx) {
  return resolve_partition(p != 0 ? p : (max_ctx > 4096 ? 1024 : 2048), max_ctx);
}
// Auto partition of the tcgen05 multi-token kernel (more than 32 rows per
// kv-head, or an FP8 pool): PKV_TC_AUTO_PARTITION tokens.  Its items are
// claimed dynamically and listed longest first, so long partitions cost no
// tail, while each split adds partials and a merge.  Never more partitions
// than the multi-token rule above, so a workspace sized by it suffices.
int resolve_multi_tc_partition(int p, long long max_ctx) {
  return p != 0 ? resolve_partition(p, max_ctx) : PKV_TC_AUTO_PARTITION;
}
// Auto partition of the FP8 decode (a page is half the bytes of a 16-bit
// one): 768 tokens up to 4096 (1.5x the 16-bit rule: short batches keep
// enough, evenly sized CTAs for the last wave), 1024 up to 16384, 2048
// past it.  Never more partitions than the 16-bit rule, so its workspace
// suffices.
int resolve_fp8_partition(int p, long long max_ctx) {
  return resolve_partition(p != 0 ? p : (max_ctx > 16384 ? 2048 : max_ctx > 4096 ? 1024 : 768), max_ctx);
}
int multi_ntiles(long long rows) { return rows <= 8 ? 1 : 2; }
int multi_rows_warps(long long rows) { return rows <= 16 ? 0 : rows <= 24 ? 3 : 4; }
#ifndef PKV_FA_ABOVE_ROWS
#define PKV_FA_ABOVE_ROWS 32
#endif
constexpr int kFaAboveRows = PKV_FA_ABOVE_ROWS;  // rows per kv-head past which the M-dimension kernel runs
constexpr int kFaWarps = 4;  // 16 rows each
#ifndef PKV_FA_PAGES
#define PKV_FA_PAGES 2
#endif
constexpr int kFaPages = PKV_FA_PAGES;  // pages a warp takes in one step
constexpr int kFaCode = 100;  // dispatch code of paged_multi_fa_kernel
#ifndef PKV_ROWS_STAGES
#define PKV_ROWS_STAGES 2
#endif
#ifndef PKV_ROWS_PAGES
#define PKV_ROWS_PAGES 2
#endif
constexpr int kRowsStages = PKV_ROWS_STAGES;  // stages in the ring
constexpr int kRowsPages = PKV_ROWS_PAGES;    // pages per stage (taken in one step)

template <typename T, int D, int G, int NW>
pkv_status launch_multi_rows(const pkv::MultiArgs& a, const void* k_cache, const void* v_cache, int num_blocks,
                             cudaStream_t st) {
  using S = pkv::RowsShape<D, NW, kRowsStages, kRowsPages>;
  static_assert(kMaxPartition / PKV_BLOCK_SIZE <= S::kMaxPages, "the page table of a partition fits shared memory");
  CUtensorMap mk, mv;
  const long long rows = static_cast<long long>(num_blocks) * a.num_kv_heads * PKV_BLOCK_SIZE;
  if (!encode_cache_map(&mk, k_cache, pkv::Mma<T>::kTmaType, D, rows) ||
      !encode_cache_map(&mv, v_cache, pkv::Mma<T>::kTmaType, D, rows))
    return PKV_ECUDA;
  auto kfn = pkv::paged_multi_rows_kernel<T, D, G, NW, kRowsStages, kRowsPages>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmem)) !=
      cudaSuccess)
    return PKV_ECUDA;
  const dim3 grid(a.num_kv_heads, a.num_seqs * a.tiles, a.num_parts);
  if (launch(kfn, grid, dim3(NW * 32), S::kSmem, st, a, mk, mv) != PKV_OK) return PKV_ECUDA;
  if (a.num_parts > 1) return launch_multi_merge<T, D, G>(a, st);
  return PKV_OK;
}

template <typename T, int D, int G>
pkv_status launch_multi_fa(const pkv::MultiArgs& a, const void* k_cache, const void* v_cache, int num_blocks,
                           cudaStream_t st) {
  using S = pkv::RowsShape<D, kFaWarps, kRowsStages, kFaPages>;
  static_assert(kMaxPartition / PKV_BLOCK_SIZE <= S::kMaxPages, "the page table of a partition fits shared memory");
  CUtensorMap mk, mv;
  const long long rows = static_cast<long long>(num_blocks) * a.num_kv_heads * PKV_BLOCK_SIZE;
  if (!encode_cache_map(&mk, k_cache, pkv::Mma<T>::kTmaType, D, rows) ||
      !encode_cache_map(&mv, v_cache, pkv::Mma<T>::kTmaType, D, rows))
    return PKV_ECUDA;
  auto kfn = pkv::paged_multi_fa_kernel<T, D, G, kFaWarps, kRowsStages, kFaPages>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmem)) !=
      cudaSuccess)
    return PKV_ECUDA;
  const dim3 grid(a.num_kv_heads, a.num_seqs * a.tiles, a.num_parts);
  if (launch(kfn, grid, dim3(kFaWarps * 32), S::kSmem, st, a, mk, mv) != PKV_OK) return PKV_ECUDA;
  if (a.num_parts > 1) return launch_multi_merge<T, D, G>(a, st);
  return PKV_OK;
}

// More than kTcAboveRows rows per kv-head: tiles of 128 rows on the tcgen05
// tensor cores (paged_multi_tc_kernel), accumulators in tensor memory.
#ifndef PKV_TC_ABOVE_ROWS
#define PKV_TC_ABOVE_ROWS 32
#endif
constexpr int kTcAboveRows = PKV_TC_ABOVE_ROWS;
constexpr int kTcCode = 200;     // dispatch code of paged_multi_tc_kernel
constexpr int kTcFp8Code = 201;  // the same over an FP8 pool
constexpr int kTcKStages = PKV_TC_K_STAGES;
constexpr int kTcVStages = PKV_TC_V_STAGES;

bool encode_fp8_map(CUtensorMap* map, const void* base, int D, long long rows);

template <typename T, int D, int G, bool F8 = false>
pkv_status launch_multi_tc(const pkv::MultiArgs& a, const void* k_cache, const void* v_cache, int num_blocks,
                           cudaStream_t st) {
  using S = pkv::TcShape<D, kTcKStages, kTcVStages>;
  static_assert(kMaxPartition / PKV_BLOCK_SIZE <= S::kMaxPages && PKV_TC_AUTO_PARTITION / PKV_BLOCK_SIZE <= S::kMaxPages,
                "the page table of a partition fits shared memory");
  CUtensorMap mk, mv;
  const long long rows = static_cast<long long>(num_blocks) * a.num_kv_heads * PKV_BLOCK_SIZE;
  if (F8 ? !encode_fp8_map(&mk, k_cache, D, rows) || !encode_fp8_map(&mv, v_cache, D, rows)
         : !encode_cache_map(&mk, k_cache, pkv::Mma<T>::kTmaType, D, rows) ||
               !encode_cache_map(&mv, v_cache, pkv::Mma<T>::kTmaType, D, rows))
    return PKV_ECUDA;
  auto kfn = pkv::paged_multi_tc_kernel<T, D, G, kTcKStages, kTcVStages, F8>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmem)) !=
      cudaSuccess)
    return PKV_ECUDA;
  // the work list (one CTA), then a persistent grid of PKV_TC_MIN_CTAS CTAs
  // per SM claiming (list entry, kv-head) items until the list runs out
  if (launch(pkv::paged_multi_tc_plan_kernel<G>, dim3(1), dim3(1024), 0, st, a) != PKV_OK) return PKV_ECUDA;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long upper = static_cast<long long>(a.num_kv_heads) * a.num_seqs * a.tiles * a.num_parts;
  const long long ctas = std::min<long long>(static_cast<long long>(sms) * PKV_TC_MIN_CTAS, upper);
  if (launch(kfn, dim3(static_cast<unsigned>(ctas)), dim3(S::kThreads), S::kSmem, st, a, mk, mv) != PKV_OK)
    return PKV_ECUDA;
  if (a.num_parts > 1) return launch_multi_merge<T, D, G>(a, st);
  return PKV_OK;
}

template <typename T, int D, int G>
pkv_status dispatch_nt_multi(const pkv::MultiArgs& a, int NT, const void* k, const void* v, int nb,
                             cudaStream_t st) {
  // NT 1, 2: n-tiles per CTA (pages split over the warps); -3, -4: warps
  // splitting the rows; kFaCode: rows as the MMA's M dimension
  switch (NT) {
    case 1: return launch_multi<T, D, G, 1>(a, k, v, nb, st);
    case 2: return launch_multi<T, D, G, 2>(a, k, v, nb, st);
    case -3: return launch_multi_rows<T, D, G, 3>(a, k, v, nb, st);
    case -4: return launch_multi_rows<T, D, G, 4>(a, k, v, nb, st);
    case kFaCode: return launch_multi_fa<T, D, G>(a, k, v, nb, st);
    case kTcCode: return launch_multi_tc<T, D, G>(a, k, v, nb, st);
    case kTcFp8Code: return launch_multi_tc<T, D, G, true>(a, k, v, nb, st);
  }
  return PKV_EINVAL;
}

template <typename T, int D>
pkv_status dispatch_group_multi(const pkv::MultiArgs& a, int G, int NT, const void* k, const void* v, int nb,
                                cudaStream_t st) {
  switch (G) {
    case 1: return dispatch_nt_multi<T, D, 1>(a, NT, k, v, nb, st);
    case 2: return dispatch_nt_multi<T, D, 2>(a, NT, k, v, nb, st);
    case 4: return dispatch_nt_multi<T, D, 4>(a, NT, k, v, nb, st);
    case 8: return dispatch_nt_multi<T, D, 8>(a, NT, k, v, nb, st);
  }
  return PKV_EINVAL;
}

// ---- FP8 (E4M3) cache ---------------------------------------------------------
// The pool viewed as [num_blocks * Hkv * 16 rows, D bytes], one box per tile
// row span with the swizzle of that span (128 or 64 bytes).
bool encode_fp8_map(CUtensorMap* map, const void* base, int D, long long rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(D), 16};
  const cuuint32_t elem_strides[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

#ifndef PKV_FP8_STAGES
#define PKV_FP8_STAGES 3
#endif
constexpr int kFp8Stages = PKV_FP8_STAGES;  // pages in flight per warp (4 KB each at D = 128)

template <typename T, int D, int G>
pkv_status launch_decode_fp8(const pkv::DecodeArgs& a, float k_scale, float v_scale, cudaStream_t st) {
  using S = pkv::Fp8Shape<D, kMmaWarps, kFp8Stages>;
  CUtensorMap mk, mv;
  const long long rows = static_cast<long long>(a.num_blocks) * a.num_kv_heads * PKV_BLOCK_SIZE;
  if (!encode_fp8_map(&mk, a.k_cache, D, rows) || !encode_fp8_map(&mv, a.v_cache, D, rows)) return PKV_ECUDA;
  auto kfn = pkv::paged_decode_fp8_kernel<T, D, G, kMmaWarps, kFp8Stages>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmem)) !=
      cudaSuccess)
    return PKV_ECUDA;
  const dim3 grid(a.num_kv_heads, a.num_seqs, a.num_parts);
  if (launch(kfn, grid, dim3(kMmaWarps * 32), S::kSmem, st, a, mk, mv, v_scale, k_scale) != PKV_OK)
    return PKV_ECUDA;
  if (a.num_parts > 1) {
    if (launch_merge<T, D, ReduceK>(a, a.num_parts, st) != PKV_OK) return PKV_ECUDA;
  }
  return PKV_OK;
}

// Shared-prefix decode over an FP8 cache: (1) the prefix tiles as exact
// 16-bit code values in the workspace, (2) the cascade's prefix pass over
// them on the 16-bit tensor-core path (logits scaled by k_scale, partials by
// v_scale), (3) the suffix pass over the FP8 cache (beside the prefix pass;
// it makes a fused step's copies and append), (4) the cascade's merge.
template <typename T, int D, int G>
pkv_status launch_decode_prefix_fp8(const pkv::DecodeArgs& a0, void* mini_k, void* mini_v, float k_scale,
                                    float v_scale, cudaStream_t st) {
  const int row_chunks = D / 8;
  const long long total = static_cast<long long>(a0.prefix_pages) * a0.num_kv_heads * PKV_BLOCK_SIZE * row_chunks;
  long long nblk = (2 * total + 255) / 256;
  if (nblk > 148LL * 16) nblk = 148LL * 16;
  if (launch(pkv::dequant_prefix_kernel<T>, dim3(static_cast<unsigned>(nblk)), dim3(256), 0, st,
             reinterpret_cast<const uint2*>(a0.k_cache), reinterpret_cast<const uint2*>(a0.v_cache),
             static_cast<uint4*>(mini_k), static_cast<uint4*>(mini_v), a0.prefix_blocks, total, a0.num_kv_heads,
             row_chunks, a0.num_blocks) != PKV_OK)
    return PKV_ECUDA;
  {  // prefix pass
    using S = pkv::MmaShape<T, D, G, kMmaWarps, kMmaStages>;
    pkv::DecodeArgs ap = a0;
    ap.slots = nullptr;  // (the suffix pass makes the step's writes)
    ap.defer_wait = 0;
    ap.k_cache = static_cast<const unsigned char*>(mini_k);
    ap.v_cache = static_cast<const unsigned char*>(mini_v);
    ap.num_blocks = a0.prefix_pages;
    ap.prefix_ident = 1;
    ap.prefix_out_scale = v_scale;
    ap.y_offset = 0;
    CUtensorMap mk, mv;
    const long long rows = static_cast<long long>(a0.prefix_pages) * a0.num_kv_heads * PKV_BLOCK_SIZE;
    if (!encode_cache_map(&mk, mini_k, pkv::Mma<T>::kTmaType, D, rows) ||
        !encode_cache_map(&mv, mini_v, pkv::Mma<T>::kTmaType, D, rows))
      return PKV_ECUDA;
    auto kfn = pkv::paged_decode_mma_kernel<T, D, G, kMmaWarps, kMmaStages, true>;
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmem)) !=
        cudaSuccess)
      return PKV_ECUDA;
    const long long npre = static_cast<long long>(ap.num_qgroups) * ap.num_chunks;
    if (launch(kfn, dim3(ap.num_kv_heads, static_cast<unsigned>(npre), 1), dim3(kMmaWarps * 32), S::kSmem, st, ap,
               mk, mv) != PKV_OK)
      return PKV_ECUDA;
  }
  {  // suffix pass
    using S = pkv::Fp8Shape<D, kMmaWarps, kFp8Stages>;
    CUtensorMap mk, mv;
    const long long rows = static_cast<long long>(a0.num_blocks) * a0.num_kv_heads * PKV_BLOCK_SIZE;
    if (!encode_fp8_map(&mk, a0.k_cache, D, rows) || !encode_fp8_map(&mv, a0.v_cache, D, rows)) return PKV_ECUDA;
    auto kfn = pkv::paged_decode_fp8_kernel<T, D, G, kMmaWarps, kFp8Stages, true>;
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmem)) !=
        cudaSuccess)
      return PKV_ECUDA;
    pkv::DecodeArgs as = a0;
    as.defer_wait = 1;  // beside the prefix pass (see the kernel)
    if (launch(kfn, dim3(a0.num_kv_heads, a0.num_seqs, a0.num_parts), dim3(kMmaWarps * 32), S::kSmem, st, as, mk,
               mv, v_scale, k_scale) != PKV_OK)
      return PKV_ECUDA;
  }
  return launch_merge<T, D, PrefixMergeK>(a0, a0.num_chunks + a0.num_parts, st);
}

template <typename T, int D>
pkv_status dispatch_group_prefix_fp8(const pkv::DecodeArgs& a, int G, void* mk, void* mv, float k_scale, float v_scale,
                                     cudaStream_t st) {
  switch (G) {
    case 1: return launch_decode_prefix_fp8<T, D, 1>(a, mk, mv, k_scale, v_scale, st);
    case 2: return launch_decode_prefix_fp8<T, D, 2>(a, mk, mv, k_scale, v_scale, st);
    case 4: return launch_decode_prefix_fp8<T, D, 4>(a, mk, mv, k_scale, v_scale, st);
    case 8: return launch_decode_prefix_fp8<T, D, 8>(a, mk, mv, k_scale, v_scale, st);
  }
  return PKV_EINVAL;
}

// Prefix pages per prefix-role CTA of the FP8 cascade.  Its prefix pass is
// a launch of its own that the suffix pass runs beside; shorter chunks make
// more, shorter prefix CTAs, so the pass ends sooner and leaves the SMs to
// the suffix streaming.
#ifndef PKV_FP8_PREFIX_CHUNK
#define PKV_FP8_PREFIX_CHUNK 16
#endif
constexpr int kPrefixChunkPagesFp8 = PKV_FP8_PREFIX_CHUNK;
static_assert(kPrefixChunkPagesFp8 >= 1 && kPrefixChunkPagesFp8 <= 32, "one table entry per lane");

// The FP8 cascade's workspace: the 16-bit cascade's (with the FP8 chunk
// size), then (1024-aligned) the dequantised prefix tiles of K and of V,
// [prefix_pages][Hkv][16][D] each.
struct PrefixFp8Layout {
  PrefixLayout base;
  size_t off_k, off_v, total;
};
PrefixFp8Layout prefix_fp8_layout(long long B, long long Hq, long long Hkv, long long D, long long max_ctx,
                                  long long prefix_pages, long long part) {
  PrefixFp8Layout L;
  L.base = prefix_layout(B, Hq, D, max_ctx, prefix_pages, part, kPrefixChunkPagesFp8);
  const size_t tiles = static_cast<size_t>(prefix_pages * Hkv * PKV_BLOCK_SIZE * D * 2);
  L.off_k = (L.base.total + 1023) / 1024 * 1024;
  L.off_v = L.off_k + (tiles + 1023) / 1024 * 1024;
  L.total = L.off_v + tiles;
  return L;
}

template <typename T, int D>
pkv_status dispatch_group_fp8(const pkv::DecodeArgs& a, int G, float k_scale, float v_scale, cudaStream_t st) {
  switch (G) {
    case 1: return launch_decode_fp8<T, D, 1>(a, k_scale, v_scale, st);
    case 2: return launch_decode_fp8<T, D, 2>(a, k_scale, v_scale, st);
    case 4: return launch_decode_fp8<T, D, 4>(a, k_scale, v_scale, st);
    case 8: return launch_decode_fp8<T, D, 8>(a, k_scale, v_scale, st);
  }
  return PKV_EINVAL;
}

// Workspace of the multi-token path: partials [T][Hq][P][D] then (max, sum)
// [T][Hq][P]; nothing when every key fits one partition.
// Multi-token workspace: the partitions' partials (P > 1), then for the
// tcgen05 kernel its claim counter and work list (at most 2 T P entries:
// fewer than 2 T row tiles, each with at most P partitions).
size_t multi_partials_bytes(long long total_q, long long Hq, long long D, long long P) {
  if (P <= 1) return 0;
  const size_t o = static_cast<size_t>(total_q * Hq * P * D * 4);
  return (o + 15) / 16 * 16 + static_cast<size_t>(total_q * Hq * P * 8);
}
size_t multi_tc_list_offset(long long total_q, long long Hq, long long D, long long P) {
  return (multi_partials_bytes(total_q, Hq, D, P) + 15) / 16 * 16;
}
size_t multi_workspace_bytes(long long total_q, long long Hq, long long D, long long P) {
  return multi_tc_list_offset(total_q, Hq, D, P) + 16 + static_cast<size_t>(2 * total_q * (P > 1 ? P : 1)) * 8;
}

// Device address of caller memory the kernels may touch: device memory of
// the current device, managed memory, or page-locked host memory mapped
// into the device's address space.  Pageable host memory, another device's
// memory and unknown pointers are rejected.
bool device_view(const void* p, void** out) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  switch (at.type) {
    case cudaMemoryTypeDevice:
      if (at.device != dev) return false;
      *out = const_cast<void*>(p);
      return true;
    case cudaMemoryTypeManaged:
      *out = const_cast<void*>(p);
      return true;
    case cudaMemoryTypeHost:
      if (at.devicePointer == nullptr) return false;
      *out = at.devicePointer;
      return true;
    default:
      return false;
  }
}

}  // namespace

extern "C" {

const char* pkv_status_string(pkv_status s) {
  switch (s) {
    case PKV_OK: return "ok";
    case PKV_EINVAL: return "invalid argument";
    case PKV_ENOMEM: return "block pool exhausted";
    case PKV_ECUDA: return "CUDA error";
  }
  return "unknown status";
}

int pkv_abi_version(void) { return 1; }

pkv_status pkv_kv_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                         int num_blocks, pkv_dtype dtype, void* stream) {
  const int es = dtype_bytes(dtype);
  if (es == 0 || num_tokens < 0 || num_kv_heads <= 0 || !head_dim_ok(head_dim) || num_blocks <= 0)
    return PKV_EINVAL;
  if (num_tokens == 0) return PKV_OK;
  if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return PKV_EINVAL;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache)) return PKV_EINVAL;
  const int row_chunks = head_dim * es / 16;
  const long long total = static_cast<long long>(num_tokens) * num_kv_heads * row_chunks;
  const long long want = (2 * total + 255) / 256;
  const int blocks = static_cast<int>(want < 148 * 32 ? want : 148 * 32);
  return launch(pkv::kv_append_kernel, dim3(blocks), dim3(256), 0, static_cast<cudaStream_t>(stream),
                static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_cache),
                static_cast<uint4*>(v_cache), slot_mapping, total, num_kv_heads, row_chunks, num_blocks);
}

pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int num_pairs, int num_kv_heads,
                           int head_dim, int num_blocks, pkv_dtype dtype, void* stream) {
  const int es = dtype_bytes(dtype);
  if (es == 0 || num_pairs < 0 || num_pairs > 65535 || num_kv_heads <= 0 || !head_dim_ok(head_dim) ||
      num_blocks <= 0)
    return PKV_EINVAL;
  if (num_pairs == 0) return PKV_OK;
  if (!k_cache || !v_cache || !pairs || !aligned16(k_cache) || !aligned16(v_cache)) return PKV_EINVAL;
  const long long block_chunks = static_cast<long long>(num_kv_heads) * PKV_BLOCK_SIZE * head_dim * es / 16;
  const long long per_cta = 256 * 4;
  const int gx = static_cast<int>((block_chunks + per_cta - 1) / per_cta);
  const dim3 grid(gx, num_pairs, 2);
  return launch(pkv::copy_blocks_kernel, grid, dim3(256), 0, static_cast<cudaStream_t>(stream),
                static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), pairs, block_chunks, num_blocks);
}

pkv_status pkv_kv_append_copy(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                              const int64_t* slot_mapping, int num_tokens, const int32_t* copies, int num_copies,
                              int num_kv_heads, int head_dim, int num_blocks, pkv_dtype dtype, void* stream) {
  const int es = dtype_bytes(dtype);
  if (es == 0 || num_tokens < 0 || num_copies < 0 || num_kv_heads <= 0 || !head_dim_ok(head_dim) ||
      num_blocks <= 0)
    return PKV_EINVAL;
  if (num_tokens == 0 && num_copies == 0) return PKV_OK;
  if (!k_cache || !v_cache || !aligned16(k_cache) || !aligned16(v_cache)) return PKV_EINVAL;
  if (num_tokens > 0 && (!k_new || !v_new || !slot_mapping || !aligned16(k_new) || !aligned16(v_new)))
    return PKV_EINVAL;
  if (num_copies > 0 && !copies) return PKV_EINVAL;
  const int row_chunks = head_dim * es / 16;
  if (num_copies > 65535 - 1024) return PKV_EINVAL;  // copies are grid rows
  // x: CTAs per copy, each thread moving up to 8 chunks of a whole block;
  // the appends take A more rows of the grid
  const long long per_block = static_cast<long long>(num_kv_heads) * PKV_BLOCK_SIZE * row_chunks;
  const int gx = static_cast<int>((per_block + 256 * 8 - 1) / (256 * 8));
  const long long append_items = static_cast<long long>(num_tokens) * num_kv_heads * row_chunks;
  long long A = (append_items + static_cast<long long>(gx) * 256 - 1) / (static_cast<long long>(gx) * 256);
  if (A < 1) A = 1;
  if (A > 1024) A = 1024;
  const dim3 grid(gx, static_cast<unsigned>(num_copies + A), 2);
  return launch(pkv::kv_append_copy_kernel, grid, dim3(256), 0, static_cast<cudaStream_t>(stream),
                static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_cache),
                static_cast<uint4*>(v_cache), slot_mapping, copies, num_copies, num_tokens, num_kv_heads, row_chunks,
                num_blocks);
}

pkv_status pkv_copy_blocks_check(const int32_t* pairs_host, int num_pairs, int num_blocks) {
  if (num_pairs < 0 || num_blocks <= 0 || (num_pairs > 0 && pairs_host == nullptr)) return PKV_EINVAL;
  std::unordered_set<int32_t> dsts, srcs;
  for (int i = 0; i < num_pairs; ++i) {
    const int32_t s = pairs_host[2 * i], d = pairs_host[2 * i + 1];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) return PKV_EINVAL;
    if (!dsts.insert(d).second) return PKV_EINVAL;
    srcs.insert(s);
  }
  for (int32_t d : dsts)
    if (srcs.count(d)) return PKV_EINVAL;
  return PKV_OK;
}

pkv_status pkv_swap_blocks(void* dst_k, void* dst_v, int dst_blocks, const void* src_k, const void* src_v,
                           int src_blocks, const int32_t* pairs, int num_pairs, int num_kv_heads, int head_dim,
                           pkv_dtype dtype, void* stream) {
  const int es = dtype_bytes(dtype);
  if (es == 0 || num_pairs < 0 || num_kv_heads <= 0 || !head_dim_ok(head_dim) || dst_blocks <= 0 ||
      src_blocks <= 0)
    return PKV_EINVAL;
  if (num_pairs == 0) return PKV_OK;
  if (!dst_k || !dst_v || !src_k || !src_v || !pairs || !aligned16(dst_k) || !aligned16(dst_v) ||
      !aligned16(src_k) || !aligned16(src_v))
    return PKV_EINVAL;
  void *dk, *dv, *sk, *sv, *pp;
  if (!device_view(dst_k, &dk) || !device_view(dst_v, &dv) || !device_view(src_k, &sk) ||
      !device_view(src_v, &sv) || !device_view(pairs, &pp))
    return PKV_EINVAL;
  const long long block_chunks = static_cast<long long>(num_kv_heads) * PKV_BLOCK_SIZE * head_dim * es / 16;
  const long long total = block_chunks * num_pairs;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long per_cta = 256LL * 4;
  long long blocks = (2 * total + per_cta - 1) / per_cta;
  if (blocks > static_cast<long long>(sms) * 8) blocks = static_cast<long long>(sms) * 8;
  return launch(pkv::swap_blocks_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                static_cast<cudaStream_t>(stream), static_cast<uint4*>(dk), static_cast<uint4*>(dv),
                static_cast<const uint4*>(sk), static_cast<const uint4*>(sv), static_cast<const int32_t*>(pp),
                block_chunks, total, src_blocks, dst_blocks);
}

pkv_status pkv_swap_blocks_check(const int32_t* pairs_host, int num_pairs, int src_blocks, int dst_blocks) {
  if (num_pairs < 0 || src_blocks <= 0 || dst_blocks <= 0 || (num_pairs > 0 && pairs_host == nullptr))
    return PKV_EINVAL;
  std::unordered_set<int32_t> dsts;
  for (int i = 0; i < num_pairs; ++i) {
    const int32_t s = pairs_host[2 * i], d = pairs_host[2 * i + 1];
    if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) return PKV_EINVAL;
    if (!dsts.insert(d).second) return PKV_EINVAL;
  }
  return PKV_OK;
}

size_t pkv_decode_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                  int partition_tokens) {
  const int part = resolve_partition(partition_tokens, max_context_len);
  if (part < 0 || num_seqs < 0 || num_q_heads <= 0 || !head_dim_ok(head_dim) || max_context_len < 0) return 0;
  const long long P = (static_cast<long long>(max_context_len) + part - 1) / part;
  return workspace_bytes(num_seqs, num_q_heads, head_dim, P);
}

pkv_status pkv_paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* context_lens, int max_context_len, int num_seqs,
                                      int num_q_heads, int num_kv_heads, int head_dim, int num_blocks, float scale,
                                      int partition_tokens, pkv_dtype dtype, void* workspace,
                                      size_t workspace_bytes_given, void* stream) {
  pkv::DecodeArgs a{};
  long long P = 0;
  const pkv_status st0 = prepare_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                        max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                                        scale, partition_tokens, dtype, &a, &P);
  if (st0 != PKV_OK || num_seqs == 0) return st0;
  const size_t need = workspace_bytes(num_seqs, num_q_heads, head_dim, P);
  if (need > 0 && (workspace == nullptr || workspace_bytes_given < need || !aligned16(workspace)))
    return PKV_EINVAL;
  a.ws_o = static_cast<float*>(need ? workspace : nullptr);
  a.ws_ml = need ? reinterpret_cast<float2*>(static_cast<float*>(workspace) +
                                              static_cast<size_t>(num_seqs) * num_q_heads * P * head_dim)
                 : nullptr;

  const int G = num_q_heads / num_kv_heads;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (dtype) {
    case PKV_F32: return dispatch_dim<float>(a, head_dim, G, st);
    case PKV_F16: return dispatch_dim_mma<__half>(a, head_dim, G, st);
    case PKV_BF16: return dispatch_dim_mma<__nv_bfloat16>(a, head_dim, G, st);
    case PKV_E4M3: break;  // an FP8 cache decodes through pkv_paged_attention_decode_fp8
  }
  return PKV_EINVAL;
}

int pkv_partition_tokens(pkv_op op, int partition_tokens, int max_context_len, int extra) {
  if (max_context_len < 0) return -1;
  switch (op) {
    case PKV_OP_DECODE: return resolve_partition(partition_tokens, max_context_len);
    case PKV_OP_DECODE_FP8: return resolve_fp8_partition(partition_tokens, max_context_len);
    case PKV_OP_MULTI:
      if (extra > kTcAboveRows) return resolve_multi_tc_partition(partition_tokens, max_context_len);
      return resolve_multi_partition(partition_tokens, max_context_len);
    case PKV_OP_MULTI_FP8: return resolve_multi_tc_partition(partition_tokens, max_context_len);
    case PKV_OP_DECODE_PREFIX:
      if (extra <= 0) return -1;
      return resolve_prefix_partition(partition_tokens, max_context_len, extra);
  }
  return -1;
}

size_t pkv_decode_prefix_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                         int prefix_pages, int partition_tokens) {
  const int part = resolve_prefix_partition(partition_tokens, max_context_len, prefix_pages);
  if (part < 0 || num_seqs < 0 || num_q_heads <= 0 || !head_dim_ok(head_dim) || max_context_len < 0 ||
      prefix_pages <= 0)
    return 0;
  return prefix_layout(num_seqs, num_q_heads, head_dim, max_context_len, prefix_pages, part).total;
}

}  // extern "C"

namespace {
// The step's writes a fused decode makes (pkv_decode_step); all null when
// the decode stands alone.
struct StepWrites {
  const void* k_new = nullptr;
  const void* v_new = nullptr;
  const int64_t* slots = nullptr;
  const int32_t* copies = nullptr;
  int n_copies = 0;
  bool defer = false;  // the writes were launched just before the decode (see DecodeArgs::defer_wait)
};

void attach_step(pkv::DecodeArgs* a, const StepWrites& w) {
  a->k_new = static_cast<const unsigned char*>(w.k_new);
  a->v_new = static_cast<const unsigned char*>(w.v_new);
  a->slots = w.slots;
  a->copies = w.copies;
  a->n_copies = w.n_copies;
  a->defer_wait = w.defer ? 1 : 0;
}

constexpr int kValidateOnly = -2;  // decode_prefix_impl's phase: check the arguments, launch nothing

pkv_status decode_prefix_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                                             const int32_t* block_tables, int max_blocks_per_seq,
                                             const int32_t* context_lens, int max_context_len,
                                             const int32_t* prefix_blocks, int prefix_pages, int num_seqs,
                                             int num_q_heads, int num_kv_heads, int head_dim, int num_blocks,
                                             float scale, int partition_tokens, pkv_dtype dtype, void* workspace,
                                             size_t workspace_bytes_given, int phase, void* stream,
                                             const StepWrites& step = StepWrites{}) {
  if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_EINVAL;  // tensor-core path only
  if (prefix_pages <= 0 || prefix_pages > max_blocks_per_seq) return PKV_EINVAL;
  pkv::DecodeArgs a{};
  long long P = 0;
  const int part = resolve_prefix_partition(partition_tokens, max_context_len, prefix_pages);
  if (part < 0) return PKV_EINVAL;
  const pkv_status st0 = prepare_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                        max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                                        scale, part, dtype, &a, &P);
  if (st0 != PKV_OK || num_seqs == 0) return st0;
  if (prefix_blocks == nullptr) return PKV_EINVAL;
  const PrefixLayout L = prefix_layout(num_seqs, num_q_heads, head_dim, max_context_len, prefix_pages, a.partition);
  if (workspace == nullptr || workspace_bytes_given < L.total || !aligned16(workspace)) return PKV_EINVAL;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  a.num_parts = static_cast<int>(L.parts);
  a.ws_o = reinterpret_cast<float*>(ws + L.off_so);
  a.ws_ml = reinterpret_cast<float2*>(ws + L.off_sml);
  a.wp_o = reinterpret_cast<float*>(ws + L.off_po);
  a.wp_ml = reinterpret_cast<float2*>(ws + L.off_pml);
  a.conform = reinterpret_cast<int*>(ws + L.off_conform);
  a.prefix_blocks = prefix_blocks;
  attach_step(&a, step);
  a.prefix_pages = prefix_pages;
  a.chunk_pages = kPrefixChunkPages;
  a.num_chunks = static_cast<int>(L.chunks);
  a.num_qgroups = (num_seqs * (num_q_heads / num_kv_heads) + kMmaWarps * 16 - 1) / (kMmaWarps * 16);  // 16 queries per prefix warp
  // suffix partitions in flight per sequence: enough for the longest suffix
  // of a sequence that shares the prefix; a sequence that does not share it
  // loops over its extra partitions
  const long long span_max = static_cast<long long>(max_context_len) - static_cast<long long>(prefix_pages) * PKV_BLOCK_SIZE;
  a.suffix_z = span_max > 0 ? static_cast<int>((span_max + a.partition - 1) / a.partition) : 1;
  if (static_cast<long long>(a.num_qgroups) * a.num_chunks + static_cast<long long>(num_seqs) * a.suffix_z > 65535)
    return PKV_EINVAL;

  if (phase == kValidateOnly) return PKV_OK;
  const int G = num_q_heads / num_kv_heads;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == PKV_F16) return dispatch_dim_prefix<__half>(a, head_dim, G, phase, st);
  return dispatch_dim_prefix<__nv_bfloat16>(a, head_dim, G, phase, st);
}
}  // namespace

extern "C" {

pkv_status pkv_paged_attention_decode_prefix(void* out, const void* q, const void* k_cache, const void* v_cache,
                                             const int32_t* block_tables, int max_blocks_per_seq,
                                             const int32_t* context_lens, int max_context_len,
                                             const int32_t* prefix_blocks, int prefix_pages, int num_seqs,
                                             int num_q_heads, int num_kv_heads, int head_dim, int num_blocks,
                                             float scale, int partition_tokens, pkv_dtype dtype, void* workspace,
                                             size_t workspace_bytes_given, void* stream) {
  return decode_prefix_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                            max_context_len, prefix_blocks, prefix_pages, num_seqs, num_q_heads, num_kv_heads,
                            head_dim, num_blocks, scale, partition_tokens, dtype, workspace, workspace_bytes_given, -1,
                            stream);
}

pkv_status pkv_paged_attention_decode_prefix_phase(void* out, const void* q, const void* k_cache,
                                                   const void* v_cache, const int32_t* block_tables,
                                                   int max_blocks_per_seq, const int32_t* context_lens,
                                                   int max_context_len, const int32_t* prefix_blocks,
                                                   int prefix_pages, int num_seqs, int num_q_heads,
                                                   int num_kv_heads, int head_dim, int num_blocks, float scale,
                                                   int partition_tokens, pkv_dtype dtype, void* workspace,
                                                   size_t workspace_bytes_given, int phase, void* stream) {
  if (phase < 0 || phase > 2) return PKV_EINVAL;
  return decode_prefix_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                            max_context_len, prefix_blocks, prefix_pages, num_seqs, num_q_heads, num_kv_heads,
                            head_dim, num_blocks, scale, partition_tokens, dtype, workspace, workspace_bytes_given,
                            phase, stream);
}


pkv_status pkv_decode_step(void* out, const void* q, void* k_cache, void* v_cache, const void* k_new,
                           const void* v_new, const int64_t* slot_mapping, const int32_t* copies, int num_copies,
                           const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                           int max_context_len, const int32_t* prefix_blocks, int prefix_pages, int num_seqs,
                           int num_q_heads, int num_kv_heads, int head_dim, int num_blocks, float scale,
                           int partition_tokens, pkv_dtype dtype, void* workspace, size_t workspace_bytes_given,
                           void* stream) {
  if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_EINVAL;  // tensor-core path only
  if (num_copies < 0 || num_copies > num_seqs || prefix_pages < 0) return PKV_EINVAL;
  if (num_seqs > 0 && (!k_new || !v_new || !slot_mapping || !aligned16(k_new) || !aligned16(v_new)))
    return PKV_EINVAL;
  if (num_copies > 0 && copies == nullptr) return PKV_EINVAL;
  StepWrites w;
  w.k_new = k_new;
  w.v_new = v_new;
  w.slots = slot_mapping;
  w.copies = copies;
  w.n_copies = num_copies;
  if (prefix_pages > 0) {
    // the cascade: the copies and the append in their own launch, which
    // the cascade does not wait for except where it reads what they write
    // (each sequence's last page): its CTAs stream the prefix and the other
    // pages meanwhile
    const pkv_status sv = decode_prefix_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                             context_lens, max_context_len, prefix_blocks, prefix_pages, num_seqs,
                                             num_q_heads, num_kv_heads, head_dim, num_blocks, scale,
                                             partition_tokens, dtype, workspace, workspace_bytes_given,
                                             kValidateOnly, stream);
    if (sv != PKV_OK || num_seqs == 0) return sv;
    const pkv_status sc = pkv_kv_append_copy(k_new, v_new, k_cache, v_cache, slot_mapping, num_seqs, copies,
                                             num_copies, num_kv_heads, head_dim, num_blocks, dtype, stream);
    if (sc != PKV_OK) return sc;
    StepWrites after;
    after.defer = true;
    return decode_prefix_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                              max_context_len, prefix_blocks, prefix_pages, num_seqs, num_q_heads, num_kv_heads,
                              head_dim, num_blocks, scale, partition_tokens, dtype, workspace, workspace_bytes_given,
                              -1, stream, after);
  }
  pkv::DecodeArgs a{};
  long long P = 0;
  const pkv_status st0 = prepare_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                        max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                                        scale, partition_tokens, dtype, &a, &P);
  if (st0 != PKV_OK || num_seqs == 0) return st0;
  const size_t need = workspace_bytes(num_seqs, num_q_heads, head_dim, P);
  if (need > 0 && (workspace == nullptr || workspace_bytes_given < need || !aligned16(workspace)))
    return PKV_EINVAL;
  a.ws_o = static_cast<float*>(need ? workspace : nullptr);
  a.ws_ml = need ? reinterpret_cast<float2*>(static_cast<float*>(workspace) +
                                              static_cast<size_t>(num_seqs) * num_q_heads * P * head_dim)
                 : nullptr;
  attach_step(&a, w);
  const int G = num_q_heads / num_kv_heads;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == PKV_F16) return dispatch_dim_mma<__half>(a, head_dim, G, st);
  return dispatch_dim_mma<__nv_bfloat16>(a, head_dim, G, st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without caller-provided scratch: the split-K workspace lives in a
// fixed device array owned by the library (see pkv.h for who needs this).
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_static_workspace[PKV_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_ws_mutex;
// per device: the id of the context the address was looked up in, and the
// address
struct StaticWsEntry {
  unsigned long long ctx_id;
  void* addr;
};
StaticWsEntry g_static_ws[kMaxDevices] = {};

// Unique id of the calling thread's current context (0 when none is bound).
// Ids are never reused within a process, unlike context handles.  Driver
// API calls reached through the runtime's entry-point query, so the library
// links only the runtime.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = reinterpret_cast<GetCurrent>(driver_entry_point("cuCtxGetCurrent"));
  static GetId get_id = reinterpret_cast<GetId>(driver_entry_point("cuCtxGetId"));
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&c) != CUDA_SUCCESS || c == nullptr ||
      get_id(c, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_static_workspace on the current device.  In host code
// the array's name only stands in for it, so the address is looked up with
// the device current and kept, keyed by the device and the id of its current
// context: when the caller has destroyed and re-created the device's context
// (for example after cudaDeviceReset), the module is loaded anew and the
// address is looked up again.
pkv_status static_workspace_address(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ECUDA;
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  StaticWsEntry& e = g_static_ws[dev];
  unsigned long long id = current_context_id();
  if (e.addr == nullptr || id == 0 || e.ctx_id != id) {
    // (a thread with no context bound yet gets the device's primary context
    // from this runtime call; its id is read after it)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) return PKV_ECUDA;
    id = current_context_id();
    if (id == 0) return PKV_ECUDA;
    e.ctx_id = id;
    e.addr = p;
  }
  *addr = e.addr;
  return PKV_OK;
}

}  // namespace

extern "C" {

pkv_status pkv_paged_attention_decode_static_ws(void* out, const void* q, const void* k_cache,
                                                const void* v_cache, const int32_t* block_tables,
                                                int max_blocks_per_seq, const int32_t* context_lens,
                                                int max_context_len, int num_seqs, int num_q_heads,
                                                int num_kv_heads, int head_dim, int num_blocks, float scale,
                                                int partition_tokens, pkv_dtype dtype, void* stream) {
  // the size this call needs; larger than the fixed area -> rejected up front
  const size_t need =
      pkv_decode_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len, partition_tokens);
  if (need > static_cast<size_t>(PKV_STATIC_WORKSPACE_BYTES)) return PKV_EINVAL;
  void* ws = nullptr;
  const pkv_status st = static_workspace_address(&ws);
  if (st != PKV_OK) return st;
  return pkv_paged_attention_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                    max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                                    scale, partition_tokens, dtype, ws, PKV_STATIC_WORKSPACE_BYTES, stream);
}


pkv_status pkv_selftest_bounded_wait(long long limit_cycles, void* stream) {
  if (limit_cycles <= 0 || limit_cycles > (1ll << 32)) return PKV_EINVAL;
  pkv::bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

pkv_status pkv_get_error(uint32_t* flags, void* stream) {
  if (flags == nullptr) return PKV_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  pkv::take_error_snapshot_kernel<<<1, 1, 0, st>>>();
  if (cudaGetLastError() != cudaSuccess) return PKV_ECUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, pkv::g_error_snapshot, sizeof(v), 0, cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return PKV_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PKV_ECUDA;
  *flags = v;
  return PKV_OK;
}

size_t pkv_multi_workspace_bytes(int total_query_tokens, int num_q_heads, int head_dim, int max_context_len,
                                 int partition_tokens) {
  const int part = resolve_multi_partition(partition_tokens, max_context_len);
  if (part < 0 || total_query_tokens < 0 || num_q_heads <= 0 || !head_dim_ok(head_dim) || max_context_len < 0)
    return 0;
  const long long P = (static_cast<long long>(max_context_len) + part - 1) / part;
  return multi_workspace_bytes(total_query_tokens, num_q_heads, head_dim, P);
}

}  // extern "C"

namespace {
// Both multi-token entry points: a 16-bit pool (fp8 false; every kernel by
// rows per kv-head) or an FP8 pool (the tcgen05 kernel for every shape).
pkv_status multi_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                      int max_context_len, const int32_t* query_start, int max_query_len, int total_query_tokens,
                      int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int num_blocks, float scale,
                      int partition_tokens, pkv_dtype dtype, void* workspace, size_t workspace_bytes_given,
                      void* stream, bool fp8, float k_scale, float v_scale) {
  if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_EINVAL;  // tensor-core path only
  if (fp8 && (!std::isfinite(k_scale) || !std::isfinite(v_scale) || !(k_scale > 0.f) || !(v_scale > 0.f)))
    return PKV_EINVAL;
  int part = resolve_multi_partition(partition_tokens, max_context_len);
  if (part < 0 || num_seqs < 0 || num_kv_heads <= 0 || num_kv_heads > 65535 || num_q_heads <= 0 ||
      num_q_heads % num_kv_heads != 0 || !group_ok(num_q_heads / num_kv_heads) || !head_dim_ok(head_dim) ||
      num_blocks <= 0 || max_context_len < 0 || max_blocks_per_seq <= 0 || max_query_len < 0 ||
      total_query_tokens < 0 || num_q_heads > 65535 ||
      static_cast<long long>(max_context_len) > static_cast<long long>(max_blocks_per_seq) * PKV_BLOCK_SIZE ||
      !std::isfinite(scale))
    return PKV_EINVAL;
  if (num_seqs == 0 || total_query_tokens == 0 || max_query_len == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start) return PKV_EINVAL;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PKV_EINVAL;
  if (static_cast<long long>(num_blocks) * num_kv_heads * PKV_BLOCK_SIZE > 0x7fffffffLL) return PKV_EINVAL;
  const int G = num_q_heads / num_kv_heads;
  const long long rows_max = static_cast<long long>(max_query_len) * G;
  const bool tc = fp8 || rows_max > kTcAboveRows;
  const bool fa = !tc && rows_max > kFaAboveRows;
  const int NW = (fa || tc) ? 0 : multi_rows_warps(rows_max);
  const int NT = tc ? (fp8 ? kTcFp8Code : kTcCode) : fa ? kFaCode : NW ? -NW : multi_ntiles(rows_max);
  if (tc) part = resolve_multi_tc_partition(partition_tokens, max_context_len);
  const int tile_rows = tc ? 128 : fa ? 16 * kFaWarps : 8 * (NW ? NW : NT);
  const long long tiles = (rows_max + tile_rows - 1) / tile_rows;
  const long long P = (static_cast<long long>(max_context_len) + part - 1) / part;
  if (P > 65535) return PKV_EINVAL;
  if (tc) {
    // the persistent kernel's work list: a tile index fits 15 bits, the
    // (entry, kv-head) items an int
    if (tiles > 32767 || 2LL * total_query_tokens * P * num_kv_heads >= (1LL << 31)) return PKV_EINVAL;
  } else if (tiles * num_seqs > 65535) {
    return PKV_EINVAL;
  }
  const size_t need = tc ? multi_workspace_bytes(total_query_tokens, num_q_heads, head_dim, P)
                        : multi_partials_bytes(total_query_tokens, num_q_heads, head_dim, P);
  if (need > 0 && (workspace == nullptr || workspace_bytes_given < need || !aligned16(workspace)))
    return PKV_EINVAL;
  pkv::MultiArgs a{};
  a.out = out;
  a.q = q;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start = query_start;
  if (P > 1) {
    a.ws_o = static_cast<float*>(workspace);
    const size_t o = static_cast<size_t>(total_query_tokens) * num_q_heads * P * head_dim * 4;
    a.ws_ml = reinterpret_cast<float2*>(static_cast<unsigned char*>(workspace) + (o + 15) / 16 * 16);
  }
  if (tc) {
    unsigned char* l = static_cast<unsigned char*>(workspace) +
                       multi_tc_list_offset(total_query_tokens, num_q_heads, head_dim, P);
    a.tc_ctr = reinterpret_cast<int*>(l);
    a.tc_items = reinterpret_cast<int2*>(l + 16);
  }
  a.bt_stride = max_blocks_per_seq;
  a.max_ctx = max_context_len;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.partition = part;
  a.num_parts = P > 1 ? static_cast<int>(P) : 1;
  a.tiles = static_cast<int>(tiles);
  a.max_q = max_query_len;
  a.total_q = total_query_tokens;
  a.qk_scale = scale * kLog2e * (fp8 ? k_scale : 1.f);
  a.v_scale = fp8 ? v_scale : 1.f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto run = [&](auto tag) -> pkv_status {
    using T = decltype(tag);
    if (head_dim == 64) return dispatch_group_multi<T, 64>(a, G, NT, k_cache, v_cache, num_blocks, st);
    return dispatch_group_multi<T, 128>(a, G, NT, k_cache, v_cache, num_blocks, st);
  };
  if (dtype == PKV_F16) return run(__half{});
  return run(__nv_bfloat16{});
}
}  // namespace

extern "C" {

pkv_status pkv_paged_attention_multi(void* out, const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, int max_blocks_per_seq,
                                     const int32_t* context_lens, int max_context_len,
                                     const int32_t* query_start, int max_query_len, int total_query_tokens,
                                     int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int num_blocks,
                                     float scale, int partition_tokens, pkv_dtype dtype, void* workspace,
                                     size_t workspace_bytes_given, void* stream) {
  return multi_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, max_context_len,
                    query_start, max_query_len, total_query_tokens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                    num_blocks, scale, partition_tokens, dtype, workspace, workspace_bytes_given, stream, false, 1.f,
                    1.f);
}

pkv_status pkv_paged_attention_multi_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_tables, int max_blocks_per_seq,
                                         const int32_t* context_lens, int max_context_len,
                                         const int32_t* query_start, int max_query_len, int total_query_tokens,
                                         int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                         int num_blocks, float scale, float k_scale, float v_scale,
                                         int partition_tokens, pkv_dtype q_dtype, void* workspace,
                                         size_t workspace_bytes_given, void* stream) {
  return multi_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, max_context_len,
                    query_start, max_query_len, total_query_tokens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                    num_blocks, scale, partition_tokens, q_dtype, workspace, workspace_bytes_given, stream, true,
                    k_scale, v_scale);
}

size_t pkv_decode_prefix_fp8_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                             int max_context_len, int prefix_pages, int partition_tokens) {
  const int part = resolve_prefix_partition(partition_tokens, max_context_len, prefix_pages);
  if (part < 0 || num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || !head_dim_ok(head_dim) ||
      max_context_len < 0 || prefix_pages <= 0)
    return 0;
  return prefix_fp8_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, prefix_pages, part).total;
}

}  // extern "C"

namespace {
pkv_status decode_prefix_fp8_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                                  int max_context_len, const int32_t* prefix_blocks, int prefix_pages, int num_seqs,
                                  int num_q_heads, int num_kv_heads, int head_dim, int num_blocks, float scale,
                                  float k_scale, float v_scale, int partition_tokens, pkv_dtype q_dtype,
                                  void* workspace, size_t workspace_bytes_given, void* stream,
                                  const StepWrites& w = StepWrites{}) {
  if (q_dtype != PKV_F16 && q_dtype != PKV_BF16) return PKV_EINVAL;
  if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || !(k_scale > 0.f) || !(v_scale > 0.f))
    return PKV_EINVAL;
  if (prefix_pages <= 0 || prefix_pages > max_blocks_per_seq) return PKV_EINVAL;
  const int part = resolve_prefix_partition(partition_tokens, max_context_len, prefix_pages);
  if (part < 0) return PKV_EINVAL;
  pkv::DecodeArgs a{};
  long long P = 0;
  const pkv_status st0 = prepare_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                        max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                                        scale, part, q_dtype, &a, &P);
  if (st0 != PKV_OK || num_seqs == 0) return st0;
  if (prefix_blocks == nullptr) return PKV_EINVAL;
  if (static_cast<long long>(prefix_pages) * num_kv_heads * PKV_BLOCK_SIZE > 0x7fffffffLL) return PKV_EINVAL;
  const PrefixFp8Layout L =
      prefix_fp8_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, prefix_pages, a.partition);
  if (workspace == nullptr || workspace_bytes_given < L.total || !aligned16(workspace)) return PKV_EINVAL;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  a.num_parts = static_cast<int>(L.base.parts);
  a.ws_o = reinterpret_cast<float*>(ws + L.base.off_so);
  a.ws_ml = reinterpret_cast<float2*>(ws + L.base.off_sml);
  a.wp_o = reinterpret_cast<float*>(ws + L.base.off_po);
  a.wp_ml = reinterpret_cast<float2*>(ws + L.base.off_pml);
  a.conform = reinterpret_cast<int*>(ws + L.base.off_conform);
  a.prefix_blocks = prefix_blocks;
  a.prefix_pages = prefix_pages;
  a.chunk_pages = kPrefixChunkPagesFp8;
  a.num_chunks = static_cast<int>(L.base.chunks);
  a.num_qgroups = (num_seqs * (num_q_heads / num_kv_heads) + kMmaWarps * 16 - 1) / (kMmaWarps * 16);
  if (static_cast<long long>(a.num_qgroups) * a.num_chunks > 65535 || a.num_parts > 65535) return PKV_EINVAL;
  a.qk_scale *= k_scale;
  attach_step(&a, w);
  const int G = num_q_heads / num_kv_heads;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* mk = ws + L.off_k;
  void* mv = ws + L.off_v;
  auto run = [&](auto tag) -> pkv_status {
    using T = decltype(tag);
    if (head_dim == 64) return dispatch_group_prefix_fp8<T, 64>(a, G, mk, mv, k_scale, v_scale, st);
    return dispatch_group_prefix_fp8<T, 128>(a, G, mk, mv, k_scale, v_scale, st);
  };
  if (q_dtype == PKV_F16) return run(__half{});
  return run(__nv_bfloat16{});
}
}  // namespace

extern "C" {

pkv_status pkv_paged_attention_decode_prefix_fp8(void* out, const void* q, const void* k_cache,
                                                 const void* v_cache, const int32_t* block_tables,
                                                 int max_blocks_per_seq, const int32_t* context_lens,
                                                 int max_context_len, const int32_t* prefix_blocks,
                                                 int prefix_pages, int num_seqs, int num_q_heads, int num_kv_heads,
                                                 int head_dim, int num_blocks, float scale, float k_scale,
                                                 float v_scale, int partition_tokens, pkv_dtype q_dtype,
                                                 void* workspace, size_t workspace_bytes_given, void* stream) {
  return decode_prefix_fp8_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                max_context_len, prefix_blocks, prefix_pages, num_seqs, num_q_heads, num_kv_heads,
                                head_dim, num_blocks, scale, k_scale, v_scale, partition_tokens, q_dtype, workspace,
                                workspace_bytes_given, stream);
}

pkv_status pkv_kv_append_fp8(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                             int num_blocks, pkv_dtype src_dtype, float k_scale, float v_scale, void* stream) {
  if ((src_dtype != PKV_F16 && src_dtype != PKV_BF16) || num_tokens < 0 || num_kv_heads <= 0 ||
      !head_dim_ok(head_dim) || num_blocks <= 0 || !std::isfinite(k_scale) || !std::isfinite(v_scale) ||
      !(k_scale > 0.f) || !(v_scale > 0.f))
    return PKV_EINVAL;
  if (num_tokens == 0) return PKV_OK;
  if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping || !aligned16(k_new) || !aligned16(v_new) ||
      !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_EINVAL;
  const int row_chunks = head_dim / 8;  // 8 elements: 16 bytes in, 8 bytes out
  const long long total = static_cast<long long>(num_tokens) * num_kv_heads * row_chunks;
  long long blocks = (2 * total + 255) / 256;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto run = [&](auto kernel) {
    return launch(kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, static_cast<const uint4*>(k_new),
                  static_cast<const uint4*>(v_new), static_cast<uint2*>(k_cache), static_cast<uint2*>(v_cache),
                  slot_mapping, total, num_kv_heads, row_chunks, num_blocks, k_scale, v_scale);
  };
  if (src_dtype == PKV_F16) return run(pkv::kv_append_fp8_kernel<__half>);
  return run(pkv::kv_append_fp8_kernel<__nv_bfloat16>);
}

}  // extern "C"

namespace {
pkv_status decode_fp8_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                           int max_context_len, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                           int num_blocks, float scale, float k_scale, float v_scale, int partition_tokens,
                           pkv_dtype q_dtype, void* workspace, size_t workspace_bytes_given, void* stream,
                           const StepWrites& w = StepWrites{}) {
  if (q_dtype != PKV_F16 && q_dtype != PKV_BF16) return PKV_EINVAL;
  if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || !(k_scale > 0.f) || !(v_scale > 0.f))
    return PKV_EINVAL;
  pkv::DecodeArgs a{};
  long long P = 0;
  partition_tokens = resolve_fp8_partition(partition_tokens, max_context_len);
  if (partition_tokens < 0) return PKV_EINVAL;
  const pkv_status st0 = prepare_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                        max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                                        scale, partition_tokens, q_dtype, &a, &P);
  if (st0 != PKV_OK || num_seqs == 0) return st0;
  const size_t need = workspace_bytes(num_seqs, num_q_heads, head_dim, P);
  if (need > 0 && (workspace == nullptr || workspace_bytes_given < need || !aligned16(workspace)))
    return PKV_EINVAL;
  a.ws_o = static_cast<float*>(need ? workspace : nullptr);
  a.ws_ml = need ? reinterpret_cast<float2*>(static_cast<float*>(workspace) +
                                              static_cast<size_t>(num_seqs) * num_q_heads * P * head_dim)
                 : nullptr;
  a.qk_scale *= k_scale;
  attach_step(&a, w);
  const int G = num_q_heads / num_kv_heads;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto run = [&](auto tag) -> pkv_status {
    using T = decltype(tag);
    if (head_dim == 64) return dispatch_group_fp8<T, 64>(a, G, k_scale, v_scale, st);
    return dispatch_group_fp8<T, 128>(a, G, k_scale, v_scale, st);
  };
  if (q_dtype == PKV_F16) return run(__half{});
  return run(__nv_bfloat16{});
}
}  // namespace

extern "C" {

pkv_status pkv_paged_attention_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                                          const int32_t* block_tables, int max_blocks_per_seq,
                                          const int32_t* context_lens, int max_context_len, int num_seqs,
                                          int num_q_heads, int num_kv_heads, int head_dim, int num_blocks,
                                          float scale, float k_scale, float v_scale, int partition_tokens,
                                          pkv_dtype q_dtype, void* workspace, size_t workspace_bytes_given,
                                          void* stream) {
  return decode_fp8_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, max_context_len,
                         num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks, scale, k_scale, v_scale,
                         partition_tokens, q_dtype, workspace, workspace_bytes_given, stream);
}

pkv_status pkv_decode_step_fp8(void* out, const void* q, void* k_cache, void* v_cache, const void* k_new,
                               const void* v_new, const int64_t* slot_mapping, const int32_t* copies, int num_copies,
                               const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                               int max_context_len, const int32_t* prefix_blocks, int prefix_pages, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int num_blocks, float scale,
                               float k_scale, float v_scale, int partition_tokens, pkv_dtype q_dtype, void* workspace,
                               size_t workspace_bytes_given, void* stream) {
  if (num_copies < 0 || num_copies > num_seqs || prefix_pages < 0) return PKV_EINVAL;
  if (num_seqs > 0 && (!k_new || !v_new || !slot_mapping || !aligned16(k_new) || !aligned16(v_new)))
    return PKV_EINVAL;
  if (num_copies > 0 && copies == nullptr) return PKV_EINVAL;
  StepWrites w;
  w.k_new = k_new;
  w.v_new = v_new;
  w.slots = slot_mapping;
  w.copies = copies;
  w.n_copies = num_copies;
  if (prefix_pages > 0)  // the cascade: its suffix pass makes the writes
    return decode_prefix_fp8_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                  max_context_len, prefix_blocks, prefix_pages, num_seqs, num_q_heads, num_kv_heads,
                                  head_dim, num_blocks, scale, k_scale, v_scale, partition_tokens, q_dtype, workspace,
                                  workspace_bytes_given, stream, w);
  return decode_fp8_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, max_context_len,
                         num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks, scale, k_scale, v_scale,
                         partition_tokens, q_dtype, workspace, workspace_bytes_given, stream, w);
}

}  // extern "C"
