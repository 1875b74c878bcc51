// Launch side of the decode kernels: launch configuration (warps, stages,
// partitions), tensor maps of the pool, grids, merge launches, and the
// argument checks shared by the decode entry points.  Included once, by
// pkv_api.cu (one translation unit, so the device error word is shared).
#pragma once

#include <cmath>
#include <cstdint>

#include <cudaTypedefs.h>

#include "decode.cuh"
#include "decode_mma.cuh"
#include "decode_prefix.cuh"
#include "pkv.h"

namespace {

constexpr int kWarps = 4;  // CUDA-core (fp32) kernel
// tensor-core kernel: warps per CTA and staged pages per warp
#ifndef PKV_MMA_WARPS
#define PKV_MMA_WARPS 2
#endif
#ifndef PKV_MMA_STAGES
#define PKV_MMA_STAGES 2
#endif
constexpr int kMmaWarps = PKV_MMA_WARPS;
constexpr int kMmaStages = PKV_MMA_STAGES;
// tokens per work unit: the fp32 kernel's warps hold one table entry per
// lane, the tensor-core kernel's warps as many as a partition needs
constexpr int kMaxPartition = 2048;
static_assert(kMaxPartition <= kWarps * 32 * PKV_BLOCK_SIZE, "fp32 kernel: one table entry per lane");
static_assert(kMaxPartition <= 128 * PKV_BLOCK_SIZE, "tensor-core kernel: its warps hold a partition's table entries");
constexpr float kLog2e = 1.4426950408889634f;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int dtype_bytes(pkv_dtype dt) {
  switch (dt) {
    case PKV_F32: return 4;
    case PKV_F16: return 2;
    case PKV_BF16: return 2;
    case PKV_E4M3: return 1;
  }
  return 0;
}

// Tokens per split-K partition.  Auto (0): 512, or 1024 when the longest
// context exceeds 4096 tokens (long contexts: half the partials to merge and
// half the per-CTA fixed cost, still thousands of CTAs).
int resolve_partition(int p, long long max_ctx) {
  if (p == 0) return max_ctx > 4096 ? 2 * PKV_DEFAULT_PARTITION : PKV_DEFAULT_PARTITION;
  if (p < PKV_BLOCK_SIZE || p > kMaxPartition || p % PKV_BLOCK_SIZE != 0) return -1;
  return p;
}

bool head_dim_ok(int d) { return d == 64 || d == 128; }
bool group_ok(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

// Stages per warp: keep roughly 24 KB of K+V in flight per warp.
constexpr int stages_for(int stage_bytes) {
  return stage_bytes >= 16384 ? 2 : (24576 / stage_bytes > 8 ? 8 : 24576 / stage_bytes);
}


// Launch with programmatic stream serialization (see pdl_wait in common.cuh).
template <typename... KArgs, typename... Args>
pkv_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

// Merge launches: heads per CTA from the number of partials per head
// (8 warps on one head when there are many, one warp per head when few).
template <typename T, int D, template <typename, int, int> class K>
pkv_status launch_merge(const pkv::DecodeArgs& a, int partials_per_head, cudaStream_t st) {
  const dim3 block(pkv::kMergeWarps * 32);
  if (partials_per_head >= 32)
    return launch(K<T, D, 1>::fn, dim3(a.num_q_heads, a.num_seqs), block, 0, st, a);
  if (partials_per_head >= 8)
    return launch(K<T, D, 4>::fn, dim3((a.num_q_heads + 3) / 4, a.num_seqs), block, 0, st, a);
  return launch(K<T, D, 8>::fn, dim3((a.num_q_heads + 7) / 8, a.num_seqs), block, 0, st, a);
}
template <typename T, int D, int HPC>
struct ReduceK {
  static constexpr auto fn = pkv::paged_decode_reduce_kernel<T, D, HPC>;
};
template <typename T, int D, int HPC>
struct PrefixMergeK {
  static constexpr auto fn = pkv::paged_decode_prefix_merge_kernel<T, D, HPC>;
};

template <typename T, int D, int G>
pkv_status launch_decode(const pkv::DecodeArgs& a, cudaStream_t st) {
  constexpr int kStages = stages_for(2 * PKV_BLOCK_SIZE * D * static_cast<int>(sizeof(T)));
  using S = pkv::DecodeShape<T, D, G, kWarps, kStages>;
  auto kfn = pkv::paged_decode_partition_kernel<T, D, G, kWarps, kStages>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmem)) !=
      cudaSuccess)
    return PKV_ECUDA;
  const dim3 grid(a.num_kv_heads, a.num_seqs, a.num_parts);
  if (launch(kfn, grid, dim3(kWarps * 32), S::kSmem, st, a) != PKV_OK) return PKV_ECUDA;
  if (a.num_parts > 1) {
    if (launch_merge<T, D, ReduceK>(a, a.num_parts, st) != PKV_OK) return PKV_ECUDA;
  }
  return PKV_OK;
}

// A driver API function, reached through the runtime (nullptr when absent).
void* driver_entry_point(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}

// ---- tensor-core path (fp16 / bf16): tensor-map TMA + mma.sync ----------
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn =
      reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(driver_entry_point("cuTensorMapEncodeTiled"));
  return fn;
}

// The pool viewed as a 2-D tensor [num_blocks * Hkv * 16 rows, D columns],
// loaded in 16 x 64 boxes with the 128-byte swizzle.
bool encode_cache_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int D, long long rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {64, 16};
  const cuuint32_t elem_strides[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int D, int G>
pkv_status launch_decode_mma(const pkv::DecodeArgs& a, cudaStream_t st) {
  constexpr int kStages = kMmaStages;
  using S = pkv::MmaShape<T, D, G, kMmaWarps, kStages>;
  CUtensorMap mk, mv;
  const long long rows = static_cast<long long>(a.num_blocks) * a.num_kv_heads * PKV_BLOCK_SIZE;
  if (!encode_cache_map(&mk, a.k_cache, pkv::Mma<T>::kTmaType, D, rows) ||
      !encode_cache_map(&mv, a.v_cache, pkv::Mma<T>::kTmaType, D, rows))
    return PKV_ECUDA;
  auto kfn = pkv::paged_decode_mma_kernel<T, D, G, kMmaWarps, kStages, false>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmem)) !=
      cudaSuccess)
    return PKV_ECUDA;
  const dim3 grid(a.num_kv_heads, a.num_seqs, a.num_parts);
  if (launch(kfn, dim3(grid), dim3(kMmaWarps * 32), S::kSmem, st, a, mk, mv) != PKV_OK) return PKV_ECUDA;
  if (a.num_parts > 1) {
    if (launch_merge<T, D, ReduceK>(a, a.num_parts, st) != PKV_OK) return PKV_ECUDA;
  }
  return PKV_OK;
}

template <typename T, int D>
pkv_status dispatch_group_mma(const pkv::DecodeArgs& a, int G, cudaStream_t st) {
  switch (G) {
    case 1: return launch_decode_mma<T, D, 1>(a, st);
    case 2: return launch_decode_mma<T, D, 2>(a, st);
    case 4: return launch_decode_mma<T, D, 4>(a, st);
    case 8: return launch_decode_mma<T, D, 8>(a, st);
  }
  return PKV_EINVAL;
}

template <typename T>
pkv_status dispatch_dim_mma(const pkv::DecodeArgs& a, int D, int G, cudaStream_t st) {
  if (D == 64) return dispatch_group_mma<T, 64>(a, G, st);
  if (D == 128) return dispatch_group_mma<T, 128>(a, G, st);
  return PKV_EINVAL;
}

// ---- shared-prefix (cascade) path ------------------------------------------
constexpr int kPrefixChunkPages = 32;  // prefix pages per prefix-role CTA (one table entry per lane)

// Partition of the cascade's suffix pass.  Auto (0): the longest suffix
// (context past the prefix) rounded up to whole pages, kept in [512, 2048],
// so that a batch of short suffixes needs one partition per sequence.
int resolve_prefix_partition(int partition_tokens, int max_context_len, int prefix_pages) {
  if (partition_tokens != 0) return resolve_partition(partition_tokens, max_context_len);
  const long long span = static_cast<long long>(max_context_len) - static_cast<long long>(prefix_pages) * 16;
  long long p = (span + 15) / 16 * 16;
  if (p < PKV_DEFAULT_PARTITION) p = PKV_DEFAULT_PARTITION;
  if (p > kMaxPartition) p = kMaxPartition;
  return static_cast<int>(p);
}

struct PrefixLayout {
  long long parts, chunks;
  size_t off_so, off_sml, off_po, off_pml, off_conform, total;
};

// Workspace of the cascade: suffix partials [B][Hq][P][D] + (max, sum)
// [B][Hq][P], prefix partials [B][Hq][C][D] + [B][Hq][C], flags [B].
PrefixLayout prefix_layout(long long B, long long Hq, long long D, long long max_ctx, long long prefix_pages,
                           long long part, long long chunk_pages = kPrefixChunkPages) {
  auto up16 = [](size_t x) { return (x + 15) / 16 * 16; };
  PrefixLayout L;
  L.parts = (max_ctx + part - 1) / part;
  if (L.parts < 1) L.parts = 1;
  L.chunks = (prefix_pages + chunk_pages - 1) / chunk_pages;
  L.off_so = 0;
  L.off_sml = up16(L.off_so + static_cast<size_t>(B * Hq * L.parts * D * 4));
  L.off_po = up16(L.off_sml + static_cast<size_t>(B * Hq * L.parts * 8));
  L.off_pml = up16(L.off_po + static_cast<size_t>(B * Hq * L.chunks * D * 4));
  L.off_conform = up16(L.off_pml + static_cast<size_t>(B * Hq * L.chunks * 8));
  L.total = up16(L.off_conform + static_cast<size_t>(B * 4));
  return L;
}

// Cascade launch.  phase -1: the whole cascade (one launch of both roles,
// prefix-role CTAs first, then the merge); 0: the prefix-role CTAs only; 1:
// the suffix-role CTAs only; 2: the merge only.  Split into phases, the
// prefix pass (which reads only q and the shared, full prefix blocks) can
// run beside the step's copies and append on another stream.
template <typename T, int D, int G>
pkv_status launch_decode_prefix(const pkv::DecodeArgs& a0, int phase, cudaStream_t st) {
  constexpr int kStages = kMmaStages;
  using S = pkv::MmaShape<T, D, G, kMmaWarps, kStages>;
  pkv::DecodeArgs a = a0;
  const long long npre = static_cast<long long>(a.num_qgroups) * a.num_chunks;
  const long long nsuf = static_cast<long long>(a.num_seqs) * a.suffix_z;
  if (npre + nsuf > 65535) return PKV_EINVAL;
  if (phase != 2) {
    CUtensorMap mk, mv;
    const long long rows = static_cast<long long>(a.num_blocks) * a.num_kv_heads * PKV_BLOCK_SIZE;
    if (!encode_cache_map(&mk, a.k_cache, pkv::Mma<T>::kTmaType, D, rows) ||
        !encode_cache_map(&mv, a.v_cache, pkv::Mma<T>::kTmaType, D, rows))
      return PKV_ECUDA;
    auto kfn = pkv::paged_decode_mma_kernel<T, D, G, kMmaWarps, kStages, true>;
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmem)) !=
        cudaSuccess)
      return PKV_ECUDA;
    const long long ygrid = phase == 0 ? npre : phase == 1 ? nsuf : npre + nsuf;
    a.y_offset = phase == 1 ? static_cast<int>(npre) : 0;
    if (ygrid > 0 && launch(kfn, dim3(a.num_kv_heads, static_cast<unsigned>(ygrid), 1), dim3(kMmaWarps * 32),
                            S::kSmem, st, a, mk, mv) != PKV_OK)
      return PKV_ECUDA;
    if (phase >= 0) return PKV_OK;
  }
  // merge prefix chunks and suffix partitions
  return launch_merge<T, D, PrefixMergeK>(a, a.num_chunks + a.num_parts, st);
}

template <typename T, int D>
pkv_status dispatch_group_prefix(const pkv::DecodeArgs& a, int G, int phase, cudaStream_t st) {
  switch (G) {
    case 1: return launch_decode_prefix<T, D, 1>(a, phase, st);
    case 2: return launch_decode_prefix<T, D, 2>(a, phase, st);
    case 4: return launch_decode_prefix<T, D, 4>(a, phase, st);
    case 8: return launch_decode_prefix<T, D, 8>(a, phase, st);
  }
  return PKV_EINVAL;
}

template <typename T>
pkv_status dispatch_dim_prefix(const pkv::DecodeArgs& a, int D, int G, int phase, cudaStream_t st) {
  if (D == 64) return dispatch_group_prefix<T, 64>(a, G, phase, st);
  if (D == 128) return dispatch_group_prefix<T, 128>(a, G, phase, st);
  return PKV_EINVAL;
}

// Checks shared by the decode entry points; fills `a` (everything but the
// workspace) and the partition count.  No CUDA call.
pkv_status prepare_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                          int max_context_len, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                          int num_blocks, float scale, int partition_tokens, pkv_dtype dtype, pkv::DecodeArgs* a,
                          long long* P_out) {
  const int part = resolve_partition(partition_tokens, max_context_len);
  if (dtype_bytes(dtype) == 0 || part < 0 || num_seqs < 0 || num_seqs > 65535 || num_kv_heads <= 0 ||
      num_kv_heads > 65535 || num_q_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
      !group_ok(num_q_heads / num_kv_heads) || !head_dim_ok(head_dim) || num_blocks <= 0 ||
      max_context_len < 0 || max_blocks_per_seq <= 0 ||
      static_cast<long long>(max_context_len) > static_cast<long long>(max_blocks_per_seq) * PKV_BLOCK_SIZE ||
      !std::isfinite(scale))
    return PKV_EINVAL;
  if (num_seqs == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_EINVAL;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PKV_EINVAL;
  const long long P = (static_cast<long long>(max_context_len) + part - 1) / part;
  if (P > 65535) return PKV_EINVAL;
  // tile row coordinates of the 2-D cache view are 32-bit
  if (static_cast<long long>(num_blocks) * num_kv_heads * PKV_BLOCK_SIZE > 0x7fffffffLL) return PKV_EINVAL;
  a->out = out;
  a->q = q;
  a->k_cache = static_cast<const unsigned char*>(k_cache);
  a->v_cache = static_cast<const unsigned char*>(v_cache);
  a->block_tables = block_tables;
  a->context_lens = context_lens;
  a->bt_stride = max_blocks_per_seq;
  a->max_ctx = max_context_len;
  a->num_seqs = num_seqs;
  a->num_q_heads = num_q_heads;
  a->num_kv_heads = num_kv_heads;
  a->num_blocks = num_blocks;
  a->partition = part;
  a->num_parts = P > 1 ? static_cast<int>(P) : 1;
  a->qk_scale = scale * kLog2e;
  a->prefix_out_scale = 1.f;
  *P_out = P;
  return PKV_OK;
}

template <typename T, int D>
pkv_status dispatch_group(const pkv::DecodeArgs& a, int G, cudaStream_t st) {
  switch (G) {
    case 1: return launch_decode<T, D, 1>(a, st);
    case 2: return launch_decode<T, D, 2>(a, st);
    case 4: return launch_decode<T, D, 4>(a, st);
    case 8: return launch_decode<T, D, 8>(a, st);
  }
  return PKV_EINVAL;
}

template <typename T>
pkv_status dispatch_dim(const pkv::DecodeArgs& a, int D, int G, cudaStream_t st) {
  if (D == 64) return dispatch_group<T, 64>(a, G, st);
  if (D == 128) return dispatch_group<T, 128>(a, G, st);
  return PKV_EINVAL;
}

size_t workspace_bytes(long long B, long long Hq, long long D, long long P) {
  if (P <= 1) return 0;
  return static_cast<size_t>(B * Hq * P * (D + 2) * 4);
}

}  // namespace
