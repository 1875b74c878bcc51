// Multi-token paged attention on the 5th-generation tensor cores (tcgen05),
// for prefill chunks and long verification runs: many query rows per
// (sequence, kv-head).
//
// "LLM Systems 24: Efficient LLM Inference with PagedAttention and vLLM"
// §2.2.1.3 (batches that mix prefill chunks with decode steps) and
// "PagedAttention 与 vLLM 推理加速" §6 (the large model checks a run of
// guessed tokens in one pass): each new token attends causally over its
// sequence's paged K/V, read through the block table (§2.3).  The result is
// the one paged_multi_fa_kernel computes (multi_mma.cuh); what changes is
// where the contraction runs and where its accumulators live.
//
// Work items are (sequence, row tile of 128, key partition, kv-head); a
// row is a (token, head) pair of the kv-head, as in the other multi-token
// kernels.  A plan kernel (one CTA) lists the (sequence, tile, partition)
// entries that have keys to attend, longest first; a persistent grid of two
// CTAs per SM claims items from an atomic counter until the list runs out.
// Six warps with fixed jobs, walking the same items in the same order:
//   warp 0      claims the next item, writes its page table and bounds into
//               a two-slot ring in shared memory, and issues the TMA copies
//               of its pages (a box per lane), four per key block (64 keys), into
//               a K ring and a V ring; a K stage is free again once its
//               block's scores are formed, a V stage once its P.V is done,
//               so the K loads run ahead of the S-buffer turnaround; over an
//               FP8 pool it also widens each K block's codes to fp16 in
//               place once they have landed;
//   warp 1      owns the tensor memory and issues the MMAs from one thread:
//                 S_j  = Q . K_j^T      (M 128, N 64, A and B from shared
//                                        memory, K-major, 128-byte swizzle)
//                 O   += P_j . V_j      (A = P from tensor memory, B = V
//                                        from shared memory, MN-major)
//               S is double-buffered, so the scores of block j+1 are formed
//               while block j's softmax runs; over an FP8 pool the whole
//               warp widens each V block while the block's softmax runs;
//   warps 2-5   softmax and epilogue, one thread per row (its tensor-memory
//               lane): the row's 64 scores of a block come in with
//               tcgen05.ld, the causal mask and the running max need no
//               shuffles, and P goes back into the S buffer as hi + lo
//               16-bit parts (two MMAs, ~2^-16 relative error, as in the
//               other kernels).  The running max is moved only when a block
//               raises it by more than 2^8 (then O is rescaled in tensor
//               memory), so most blocks need no O traffic at all.  At an
//               item's end they load the next item's Q while its last P.V
//               runs, then read O out and release it.
// Tensor memory: O in columns [0, D), S/P buffers at columns 128 and 192
// (256 columns a CTA, two CTAs an SM).  Invalid V rows of a block (past the
// context, or pages the table does not name) are zeroed in shared memory
// before the block's P.V, so a NaN in an unused slot never meets a zero
// weight; their keys are masked in the softmax.
//
// Every wait is bounded (PKV_ERR_TIMEOUT, then a bounded drain of the
// copies and the MMAs in flight); the tensor memory is released on every
// path.
#pragma once

#include "decode_fp8.cuh"
#include "multi_mma.cuh"

namespace pkv {

// ----------------------------------------------------------------------------
// tcgen05 primitives (inline PTX, cta_group::1)
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive on `bar` once every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// D (tensor memory) = A . B (+ D when acc != 0); A and B in shared memory.
__device__ __forceinline__ void tc_mma_ss(uint32_t d, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "}" ::"r"(d),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc)
      : "memory");
}

// D = A . B (+ D); A in tensor memory, B in shared memory.
__device__ __forceinline__ void tc_mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "}" ::"r"(d),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc)
      : "memory");
}

// 32 consecutive 32-bit columns of this thread's lane (warp-collective; the
// warp's lane quadrant is in taddr), waited for inside the same statement so
// that no use of the registers can be scheduled ahead of the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// 64 consecutive 32-bit columns of this thread's lane in one load, waited
// for inside the same statement.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, "
      "%36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, "
      "%57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]),
        "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]),
        "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
        "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),
        "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

// max of three (one instruction)
__device__ __forceinline__ float fmax3(float x, float y, float z) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(x), "f"(y), "f"(z));
  return d;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (Blackwell form): 128-byte swizzle, start
// address, leading / stride byte offsets (all in 16-byte units).
//   K-major operand: rows 128 bytes apart, 8-row groups `sbo` apart; the
//     leading offset is unused by the swizzled form (1).
//   MN-major operand: 64 MN-elements of a K-row contiguous, K-rows 128
//     bytes apart, 8-row K groups `sbo` apart, the next 64 MN-elements
//     `lbo` further on.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) /* descriptor version */ |
         (2ull << 61) /* 128-byte swizzle */;
}

template <typename T>
struct TcFmt;
template <>
struct TcFmt<__half> {
  static constexpr uint32_t kCode = 0;
};
template <>
struct TcFmt<__nv_bfloat16> {
  static constexpr uint32_t kCode = 1;
};

// Instruction descriptor of kind::f16 with fp32 accumulation: A and B of
// type T, A K-major, B K-major or MN-major, M x N.
template <typename T>
__host__ __device__ constexpr uint32_t tc_idesc(int M, int N, bool b_mn_major) {
  return (1u << 4) /* D fp32 */ | (TcFmt<T>::kCode << 7) | (TcFmt<T>::kCode << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ----------------------------------------------------------------------------
// the kernel
// ----------------------------------------------------------------------------
// Tokens of the kernel's auto key partition (its page table in shared
// memory holds that many pages).
#ifndef PKV_TC_AUTO_PARTITION
#define PKV_TC_AUTO_PARTITION 8192
#endif

template <int D, int NSK, int NSV>
struct TcShape {
  static constexpr int kRows = 128;                 // query rows of a tile (the MMA's M, one per TMEM lane)
  static constexpr int kPages = 4;                  // pages per key block
  static constexpr int kKeys = kPages * kBlockSize;  // keys per block (the S MMA's N)
  static constexpr int kPanels = D / 64;            // 128-byte column panels of a row
  static constexpr int kQPanel = kRows * 128;       // bytes of one Q panel
  static constexpr int kKVPanel = kKeys * 128;      // bytes of one K (or V) panel of a block
  static constexpr int kKV = kPanels * kKVPanel;    // K (or V) of one block: one stage of a ring
  static constexpr size_t kOffK = size_t(kPanels) * kQPanel;         // K ring: NSK stages
  static constexpr size_t kOffV = kOffK + size_t(NSK) * kKV;        // V ring: NSV stages
  static constexpr size_t kOffBars = kOffV + size_t(NSV) * kKV;
  // barriers: kfull[NSK], kempty[NSK], vfull[NSV], vempty[NSV], sfull[2],
  // pfull[2], pvdone, final, qfull, qempty, oempty, itemfull[2],
  // itemempty[2], drain, kready[NSK] (FP8: the K block widened)
  static constexpr int kBars = 3 * NSK + 2 * NSV + 14;
  static constexpr size_t kOffTab = kOffBars + size_t(kBars) * 8;
  // pages of the longest partition (the auto one, or 2048 tokens)
  static constexpr int kMaxPages = PKV_TC_AUTO_PARTITION / kBlockSize > 128 ? PKV_TC_AUTO_PARTITION / kBlockSize : 128;
  // two work-item slots: their page tables, then their descriptions
  static constexpr size_t kOffItem = kOffTab + 2 * size_t(kMaxPages) * 4;
  static constexpr size_t kOffSlot = kOffItem + 2 * 64;
  static constexpr size_t kSmem = 1024 /* alignment slack */ + kOffSlot + 16;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kColO = 0;
  static constexpr uint32_t kColS = 128;  // S/P buffer b at kColS + 64 b
  static constexpr int kThreads = 192;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(kKV % 1024 == 0 && kQPanel % 1024 == 0, "swizzled panels need 1024-byte alignment");
};

// FP8 pools: a block's 64 x D E4M3 codes land (TMA, the pool's per-page
// swizzle of decode_fp8.cuh) in the upper half of a 16-bit stage and are
// widened in place into the stage's 16-bit layout by one warp (K by the
// producer, V by the MMA warp); keys not in
// `valid` (bit r: key r of the block) become zeros.  Outputs below the codes
// are written while the codes are read; the rest only after the whole warp
// has read its codes (__syncwarp), since they overwrite them.
template <int D, int NSK, int NSV>
__device__ __forceinline__ void tc_widen_fp8(unsigned char* stage, uint64_t valid, int lane) {
  using S = TcShape<D, NSK, NSV>;
  constexpr int kH = S::kKV / 2;  // byte offset of the codes
  constexpr int kPer = D / 16;    // 16-code pieces per lane in each half
  // piece k of half h of this lane: key r, codes 16 u .. 16 u + 15 (16-byte
  // chunk u of the key's row of codes)
  auto piece = [&](int h, int k, int& r, int& u) {
    const int i = lane + 32 * k;
    if constexpr (D == 128) {
      r = i >> 2;
      u = (i & 3) + 4 * h;  // half 0: columns 0..63 (panel 0), half 1: panel 1
    } else {
      r = (i >> 2) + 32 * h;  // half 0: keys 0..31, half 1: keys 32..63
      u = i & 3;
    }
  };
  auto src = [&](int r, int u) { return reinterpret_cast<const uint4*>(stage + kH + swz8<D>(r, u)); };
  // the two 16-bit chunks (8 elements each) of codes 16 u .. 16 u + 15
  auto put = [&](int r, int u, uint4 w) {
    uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
    if ((valid >> r) & 1ull) {
      e4m3x4_to_f16(w.x, lo.x, lo.y);
      e4m3x4_to_f16(w.y, lo.z, lo.w);
      e4m3x4_to_f16(w.z, hi.x, hi.y);
      e4m3x4_to_f16(w.w, hi.z, hi.w);
    }
    unsigned char* row = stage + (u >> 2) * S::kKVPanel + r * 128;
    const int c = (2 * u) & 7;
    *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = lo;
    *reinterpret_cast<uint4*>(row + (((c + 1) ^ (r & 7)) << 4)) = hi;
  };
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    int r, u;
    piece(0, k, r, u);
    put(r, u, *src(r, u));
  }
  uint4 w[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    int r, u;
    piece(1, k, r, u);
    w[k] = *src(r, u);
  }
  __syncwarp();
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    int r, u;
    piece(1, k, r, u);
    put(r, u, w[k]);
  }
}

// One work item of the persistent kernel: a (sequence, kv-head, row tile,
// key partition), described by the producer warp for the other warps.
struct TcItem {
  int nb;  // key blocks of 64; < 0: no more work
  int b, kvh, z, r0, R, q0, base, tok0, tok1, nblk, direct;
};
static_assert(sizeof(TcItem) <= 64, "an item slot is 64 bytes");

// Key partitions of row tile t of a sequence that the kernel visits: the
// partitions up to the tile's last position (a sequence held by one
// partition: that one, also when it has nothing to attend, so its rows are
// written as zeros).
__host__ __device__ inline int tc_tile_parts(int ctx, int nq, int G, int t, int partition) {
  if (ctx <= partition) return 1;
  const int R = nq * G;
  const int p_hi = ctx - nq + (min(R, t * 128 + 128) - 1) / G;
  const int lim = min(ctx, p_hi + 1);
  return lim > 0 ? (lim + partition - 1) / partition : 0;
}

// Key blocks (64 keys) of partition z of row tile t.
__device__ __forceinline__ int tc_item_blocks(int ctx, int nq, int G, int t, int z, int partition) {
  const int R = nq * G;
  const int p_hi = ctx - nq + (min(R, t * 128 + 128) - 1) / G;
  const int tok0 = z * partition;
  const int tok1 = min(min(ctx, tok0 + partition), p_hi + 1);
  return tok1 > tok0 ? (tok1 - tok0 + 63) / 64 : 0;
}

// The work list: one entry (b, tile << 16 | partition) per visited
// (sequence, row tile, partition), longest first (a counting sort on the
// number of key blocks, at most a partition's pages / 4), so the
// items left at the end of the kernel are the short ones; its length; the
// claim counter zeroed.  One CTA of 1024 threads.
template <int G>
__global__ void __launch_bounds__(1024) paged_multi_tc_plan_kernel(const MultiArgs a) {
  pdl_enter();
  constexpr int kMaxNb = TcShape<128, 2, 2>::kMaxPages / 4;  // key blocks of the longest partition
  __shared__ int cnt[kMaxNb + 1], at[kMaxNb + 1];
  const int tid = threadIdx.x;
  if (tid <= kMaxNb) cnt[tid] = 0;
  __syncthreads();
  for (int pass = 0; pass < 2; ++pass) {
    for (int b = tid; b < a.num_seqs; b += 1024) {
      int ctx, q0, nq;
      if (!multi_seq(a, b, ctx, q0, nq, pass == 0)) continue;
      const int nt = (nq * G + 127) / 128;
      for (int t = 0; t < nt; ++t) {
        const int nz = tc_tile_parts(ctx, nq, G, t, a.partition);
        for (int z = 0; z < nz; ++z) {
          const int nb = min(tc_item_blocks(ctx, nq, G, t, z, a.partition), kMaxNb);
          if (pass == 0)
            atomicAdd(&cnt[nb], 1);
          else
            a.tc_items[atomicAdd(&at[nb], 1)] = make_int2(b, (t << 16) | z);
        }
      }
    }
    __syncthreads();
    if (pass == 0 && tid == 0) {
      int o = 0;
      for (int nb = kMaxNb; nb >= 0; --nb) {
        at[nb] = o;
        o += cnt[nb];
      }
      a.tc_ctr[0] = 0;
      a.tc_ctr[1] = o;
    }
    __syncthreads();
  }
}

#ifndef PKV_TC_K_STAGES
#define PKV_TC_K_STAGES 2
#endif
#ifndef PKV_TC_V_STAGES
#define PKV_TC_V_STAGES 2
#endif
#ifndef PKV_TC_MIN_CTAS
#define PKV_TC_MIN_CTAS 2
#endif

template <typename T, int D, int G, int NSK, int NSV, bool F8 = false>
__global__ void __launch_bounds__(TcShape<D, NSK, NSV>::kThreads, PKV_TC_MIN_CTAS)
    paged_multi_tc_kernel(const MultiArgs a, const __grid_constant__ CUtensorMap tmap_k,
                          const __grid_constant__ CUtensorMap tmap_v) {
  if (threadIdx.x == 0) {
    // the descriptors are kernel parameters: fetch them while the previous
    // kernel drains
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_k) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_v) : "memory");
  }
  pdl_enter();
  using S = TcShape<D, NSK, NSV>;
  // the MMAs' element type: T, or fp16 over an FP8 pool (every E4M3 value
  // is an fp16 value; bf16 queries are rescaled into fp16 per row)
  using TM = typename std::conditional<F8, __half, T>::type;
  using M = Mma<TM>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  unsigned char* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sq = smem_addr(smem);
  const uint32_t sk = sq + static_cast<uint32_t>(S::kOffK);
  const uint32_t sv = sq + static_cast<uint32_t>(S::kOffV);
  const uint32_t bars = sq + static_cast<uint32_t>(S::kOffBars);
  const uint32_t bar_kfull = bars, bar_kempty = bar_kfull + 8 * NSK;
  const uint32_t bar_vfull = bar_kempty + 8 * NSK, bar_vempty = bar_vfull + 8 * NSV;
  const uint32_t bar_sfull = bar_vempty + 8 * NSV;
  const uint32_t bar_pfull = bar_sfull + 16, bar_pvdone = bar_pfull + 16, bar_final = bar_pvdone + 8;
  const uint32_t bar_qfull = bar_final + 8, bar_qempty = bar_qfull + 8, bar_oempty = bar_qempty + 8;
  const uint32_t bar_itemfull = bar_oempty + 8, bar_itemempty = bar_itemfull + 16, bar_drain = bar_itemempty + 16;
  const uint32_t bar_kready = bar_drain + 8;
  int* tables = reinterpret_cast<int*>(smem + S::kOffTab);
  TcItem* items = reinterpret_cast<TcItem*>(smem + S::kOffItem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kOffSlot);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSK; ++s) {
      mbar_init(bar_kfull + 8 * s, 1);
      mbar_init(bar_kempty + 8 * s, 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(bar_vfull + 8 * s, 1);
      mbar_init(bar_vempty + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_sfull + 8 * i, 1);
      mbar_init(bar_pfull + 8 * i, 4);      // one arrival per softmax warp
      mbar_init(bar_itemfull + 8 * i, 1);   // the producer
      mbar_init(bar_itemempty + 8 * i, 5);  // the MMA warp and the softmax warps
    }
    mbar_init(bar_pvdone, 1);
    mbar_init(bar_final, 1);
    mbar_init(bar_qfull, 4);
    mbar_init(bar_qempty, 1);
    mbar_init(bar_oempty, 4);
    mbar_init(bar_drain, 1);
    for (int s = 0; s < NSK; ++s) mbar_init(bar_kready + 8 * s, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = a.tc_ctr[1] * a.num_kv_heads;  // written by the plan kernel

  bool bad = false;
  int issued_k = 0, issued_v = 0;  // producer: key blocks whose K (V) copies it issued, over all items
  auto wait_all = [&](uint32_t bar, uint32_t parity) { return __all_sync(kFull, mbar_wait_bounded(bar, parity)); };
  // every warp walks the same items in the same order; item `it` sits in
  // slot it & 1, its key blocks are numbered on from those of the items
  // before it (g0 + j), which fixes their ring stages and barrier phases
  auto loaded_in = [&](const TcItem& item, const int* tab, int i) { return i < item.nblk && tab[i] >= 0; };

  if (warp == 0) {
    // ---- producer (the whole warp): claims items, describes them, and
    // issues their K and V copies (one TMA box per lane) -----------------------
    // A K stage is released as soon as the block's S = Q.K^T MMAs are done,
    // a V stage once its P.V MMAs are done, so K runs up to NSK blocks
    // ahead of the scores and V up to NSV blocks ahead of the P.V products;
    // one loop polls both rings, so a V stage that frees late never holds
    // back the next K copy, and the next item's copies start as soon as the
    // rings have room.
    for (int it = 0; !bad; ++it) {
      const int slot = it & 1;
      if (it >= 2 && !wait_all(bar_itemempty + 8 * slot, ((it >> 1) - 1) & 1)) {
        bad = true;
        break;
      }
      int w = 0;
      if (lane == 0) w = atomicAdd(a.tc_ctr, 1);
      w = __shfl_sync(kFull, w, 0);
      TcItem& item = items[slot];
      int* tab = tables + slot * S::kMaxPages;
      if (w >= n_items) {
        if (lane == 0) {
          item.nb = -1;
          mbar_arrive(bar_itemfull + 8 * slot);
        }
        break;
      }
      const int2 e = a.tc_items[w / a.num_kv_heads];
      TcItem d;
      d.kvh = w % a.num_kv_heads;
      d.b = e.x;
      d.z = e.y & 0xffff;
      const int tile = e.y >> 16;
      int ctx, q0, nq;
      multi_seq(a, d.b, ctx, q0, nq, false);  // the plan kernel listed valid sequences only
      d.q0 = q0;
      d.R = nq * G;
      d.r0 = tile * S::kRows;
      d.base = ctx - nq;
      const int p_hi = d.base + (min(d.R, d.r0 + S::kRows) - 1) / G;
      d.direct = ctx <= a.partition;
      d.tok0 = d.z * a.partition;
      d.tok1 = min(min(ctx, d.tok0 + a.partition), p_hi + 1);
      d.nblk = d.tok1 > d.tok0 ? (d.tok1 - d.tok0 + kBlockSize - 1) / kBlockSize : 0;  // <= kMaxPages
      d.nb = (d.nblk + S::kPages - 1) / S::kPages;
      const int pg0 = d.tok0 / kBlockSize;
      for (int j = lane; j < d.nblk; j += 32) {
        const int t = a.block_tables[static_cast<long long>(d.b) * a.bt_stride + pg0 + j];
        const bool in = t >= 0 && t < a.num_blocks;
        if (!in) raise_error(PKV_ERR_BLOCK_RANGE);
        tab[j] = in ? t : -1;
      }
      __threadfence_block();
      __syncwarp();
      if (lane == 0) {
        item = d;
        mbar_arrive(bar_itemfull + 8 * slot);  // release: the table and the description
      }
      // a block's copies, one TMA box per lane (page p, 64-column panel):
      // lane 0 first arms the stage's barrier with the block's bytes
      auto issue = [&](bool is_v, int c) {
        const int g = (is_v ? issued_v : issued_k);
        const int s = g % (is_v ? NSV : NSK);
        constexpr uint32_t kPageBytes = F8 ? kBlockSize * D : kBlockSize * D * 2;
        constexpr int kBoxes = F8 ? 1 : S::kPanels;  // boxes a page
        uint32_t bytes = 0;
#pragma unroll
        for (int p = 0; p < S::kPages; ++p)
          if (loaded_in(d, tab, c * S::kPages + p)) bytes += kPageBytes;
        const uint32_t bar = (is_v ? bar_vfull : bar_kfull) + 8 * s;
        if (lane == 0) {
          if (bytes == 0)
            mbar_arrive(bar);
          else
            mbar_arrive_expect_tx(bar, bytes);
        }
        __syncwarp();
        if (bytes == 0 || lane >= S::kPages * kBoxes) return;
        const int p = lane / kBoxes, bx = lane % kBoxes;
        const int i = c * S::kPages + p;
        if (!loaded_in(d, tab, i)) return;
        const uint32_t st = (is_v ? sv : sk) + s * S::kKV;
        const CUtensorMap* map = is_v ? &tmap_v : &tmap_k;
        const int y = (tab[i] * a.num_kv_heads + d.kvh) * kBlockSize;
        if constexpr (F8)
          tma_load_2d(st + S::kKV / 2 + p * kPageBytes, map, 0, y, bar);  // one box of 16 rows x D codes
        else
          tma_load_2d(st + bx * S::kKVPanel + p * 2048, map, bx * 64, y, bar);
      };
      // the whole warp runs the loop (each decision taken by lane 0 and
      // shared); over an FP8 pool it also widens each K block once its codes
      // have landed, so the MMA warp widens only V
      int ck = 0, cv = 0, cw = 0;  // this item's blocks issued (K, V), K blocks widened
      long long t0 = clock64();
      while (ck < d.nb || cv < d.nb || (F8 && cw < d.nb)) {
        bool moved = false;
        const bool k_go = __shfl_sync(kFull, ck < d.nb && (issued_k < NSK || mbar_test(bar_kempty + 8 * (issued_k % NSK),
                                                                                         ((issued_k / NSK) - 1) & 1)), 0);
        if (k_go) {
          issue(false, ck);
          ++ck;
          ++issued_k;
          moved = true;
        }
        const bool v_go = __shfl_sync(kFull, cv < d.nb && (issued_v < NSV || mbar_test(bar_vempty + 8 * (issued_v % NSV),
                                                                                         ((issued_v / NSV) - 1) & 1)), 0);
        if (v_go) {
          issue(true, cv);
          ++cv;
          ++issued_v;
          moved = true;
        }
        if constexpr (F8) {
          const int gw = issued_k - ck + cw;  // the K block to widen next
          const bool w_go = __shfl_sync(kFull, cw < ck && mbar_test(bar_kfull + 8 * (gw % NSK), (gw / NSK) & 1), 0);
          if (w_go) {
            // the keys of block cw that are there
            const int lim = d.tok1 - (d.tok0 + cw * S::kKeys);
            uint64_t m = lim >= S::kKeys ? ~0ull : (lim > 0 ? (1ull << lim) - 1ull : 0ull);
#pragma unroll
            for (int p = 0; p < S::kPages; ++p)
              if (!loaded_in(d, tab, cw * S::kPages + p)) m &= ~(0xFFFFull << (16 * p));
            tc_widen_fp8<D, NSK, NSV>(smem + S::kOffK + (gw % NSK) * S::kKV, m, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_kready + 8 * (gw % NSK));
            ++cw;
            moved = true;
          }
        }
        if (moved) {
          t0 = clock64();
        } else if (__shfl_sync(kFull, clock64() - t0 > (1ll << 32), 0)) {
          if (lane == 0) raise_error(PKV_ERR_TIMEOUT);
          bad = true;
          break;
        } else {
          __nanosleep(32);
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (lane 0); V-row zeroing, or the widening of FP8 V codes,
    // by the whole warp ---------------------------------------------------
    constexpr uint32_t kIdQK = tc_idesc<TM>(128, S::kKeys, false);
    constexpr uint32_t kIdPV = tc_idesc<TM>(128, D, true);
    int g0 = 0;  // key blocks of the items before this one
    for (int it = 0; !bad; ++it) {
      const int slot = it & 1;
      if (!wait_all(bar_itemfull + 8 * slot, (it >> 1) & 1)) {
        bad = true;
        break;
      }
      const TcItem& d = items[slot];
      if (d.nb < 0) break;
      const int* tab = tables + slot * S::kMaxPages;
      // keys of block c that are there (inside the partition and the
      // context, on pages the table names): bit r for key r
      auto valid_keys = [&](int c) -> uint64_t {
        const int lim = d.tok1 - (d.tok0 + c * S::kKeys);
        uint64_t m = lim >= S::kKeys ? ~0ull : (lim > 0 ? (1ull << lim) - 1ull : 0ull);
#pragma unroll
        for (int p = 0; p < S::kPages; ++p)
          if (!loaded_in(d, tab, c * S::kPages + p)) m &= ~(0xFFFFull << (16 * p));
        return m;
      };
      // O still holds the previous item's result until its epilogue has read
      // it: the first P.V of this item (or the end of an item without keys)
      // waits for that
      bool o_free = it == 0;
      auto free_o = [&]() -> bool {
        if (o_free) return true;
        o_free = true;
        return wait_all(bar_oempty, (it - 1) & 1);
      };
      auto pv = [&](int j) -> bool {
        const int g = g0 + j;
        const int s = g % NSV;
        if constexpr (F8) {
          // the block's V codes widened while its softmax runs
          if (!wait_all(bar_vfull + 8 * s, (g / NSV) & 1)) return false;
          tc_widen_fp8<D, NSK, NSV>(smem + S::kOffV + s * S::kKV, valid_keys(j), lane);
          fence_proxy_async_smem();
          if (!wait_all(bar_pfull + 8 * (g & 1), (g >> 1) & 1)) return false;
        } else {
          if (!wait_all(bar_pfull + 8 * (g & 1), (g >> 1) & 1)) return false;
          if (!wait_all(bar_vfull + 8 * s, (g / NSV) & 1)) return false;
          // zero the V rows of keys that are not there (past the context or
          // on pages the table does not name): a zero weight must not meet
          // a NaN
          const uint32_t vst_off = static_cast<uint32_t>(S::kOffV) + s * S::kKV;
          bool zeroed = false;
#pragma unroll
          for (int p = 0; p < S::kPages; ++p) {
            const int i = j * S::kPages + p;
            const int page_tok = d.tok0 + i * kBlockSize;
            const int first = loaded_in(d, tab, i) ? max(0, min(kBlockSize, d.tok1 - page_tok)) : 0;
            if (first >= kBlockSize) continue;
            zeroed = true;
            const int n = (kBlockSize - first) * S::kPanels * 8;  // 16-byte chunks
            for (int e = lane; e < n; e += 32) {
              const int row = first + e / (S::kPanels * 8);
              const int pn = (e / 8) % S::kPanels;
              *reinterpret_cast<uint4*>(smem + vst_off + pn * S::kKVPanel + (p * kBlockSize + row) * 128 +
                                        (e & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
          }
          if (zeroed) fence_proxy_async_smem();
        }
        if (j == 0 && !free_o()) return false;
        __syncwarp();
        tc_fence_after();
        if (lane == 0) {
          const uint32_t vst = sv + s * S::kKV;
          const uint32_t pcol = tmem + S::kColS + 64 * (g & 1);
#pragma unroll
          for (int kk = 0; kk < S::kKeys / 16; ++kk) {
            const uint64_t vd = sw128_desc(vst + kk * 2048, S::kKVPanel, 1024);
            tc_mma_ts(tmem + S::kColO, pcol + 8 * kk, vd, kIdPV, (j > 0 || kk > 0) ? 1u : 0u);  // P hi
#ifndef PKV_TC_NO_LO
            tc_mma_ts(tmem + S::kColO, pcol + 32 + 8 * kk, vd, kIdPV, 1u);                       // P lo
#endif
          }
          tc_commit(bar_vempty + 8 * s);  // the block's V may be overwritten
          tc_commit(bar_pvdone);
        }
        __syncwarp();
        return true;
      };
      if (!wait_all(bar_qfull, it & 1)) {
        bad = true;
        break;
      }
      for (int c = 0; c < d.nb && !bad; ++c) {
        const int g = g0 + c;
        const int s = g % NSK;
        // (over an FP8 pool: the block's K codes landed and widened by the
        // producer warp)
        if (!wait_all((F8 ? bar_kready : bar_kfull) + 8 * s, (g / NSK) & 1)) {
          bad = true;
          break;
        }
        // S buffer g & 1 was last read (as P) by the P.V of block g - 2.
        // Inside an item that is the latest P.V issued; at an item's first
        // block the previous item's last P.V (g - 1) is issued too, so that
        // one is waited for (a phase wait must name the newest phase that
        // can have completed)
        const int last_pv = c == 0 ? g - 1 : g - 2;
        if (last_pv >= 0 && !wait_all(bar_pvdone, last_pv & 1)) {
          bad = true;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t kst = sk + s * S::kKV;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t qd = sw128_desc(sq + (ks >> 2) * S::kQPanel + (ks & 3) * 32, 16, 1024);
            const uint64_t kd = sw128_desc(kst + (ks >> 2) * S::kKVPanel + (ks & 3) * 32, 16, 1024);
            tc_mma_ss(tmem + S::kColS + 64 * (g & 1), qd, kd, kIdQK, ks > 0 ? 1u : 0u);
          }
          tc_commit(bar_kempty + 8 * s);  // the block's K may be overwritten
          tc_commit(bar_sfull + 8 * (g & 1));
          if (c == d.nb - 1) tc_commit(bar_qempty);  // the item's Q tile is no longer read
        }
        __syncwarp();
        if (c >= 1 && !pv(c - 1)) {
          bad = true;
          break;
        }
      }
      if (bad) break;
      if (d.nb > 0) {
        if (!pv(d.nb - 1)) {
          bad = true;
          break;
        }
      } else {
        if (lane == 0) tc_commit(bar_qempty);
        if (!free_o()) {
          bad = true;
          break;
        }
      }
      // the item's result is complete once its last P.V is (one phase per
      // item, so no parity ambiguity)
      g0 += d.nb;  // (read before the slot is released)
      __syncwarp();
      if (lane == 0) {
        tc_commit(bar_final);
        mbar_arrive(bar_itemempty + 8 * slot);
      }
      __syncwarp();
    }
    if (bad && lane == 0) raise_error(PKV_ERR_TIMEOUT);
    // every MMA this thread issued completes before the tensor memory goes
    if (lane == 0) tc_commit(bar_drain);
    __syncwarp();
    mbar_wait_bounded(bar_drain, 0);
  } else {
    // ---- softmax (one thread per row) and epilogue ----------------------------
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    // this thread's row of the item's Q into the 128-byte-swizzled K-major
    // tile (rows past the item's are zeros); returns the row's logit
    // multiplier (log2 units; over an FP8 pool it carries the K scale and,
    // for bf16 queries, the row's power-of-two rescale)
    auto load_q = [&](const TcItem& d) -> float {
      float qmul = a.qk_scale;
      const int tr = d.r0 + r;
      const uint4* src =
          tr < d.R ? reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(a.q) +
                                                    (static_cast<size_t>(d.q0 + tr / G) * a.num_q_heads +
                                                     d.kvh * G + tr % G) * D)
                   : nullptr;
      // (8 chunks of 16 bytes at a time: the row is live next to the
      // current item's softmax state)
      float sc = 1.f;
      if constexpr (F8 && !std::is_same<T, __half>::value) {
        // bf16 row -> fp16 times 2^kq, kq putting the row's largest
        // magnitude just under 2^15 (exact unless an element falls below
        // fp16's normal range); the logits take 2^-kq back
        float mx = 0.f;
        if (src) {
#pragma unroll 4
          for (int c = 0; c < D / 8; ++c) {
            const uint4 u = src[c];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = Mma<T>::unpack(w[e]);
              mx = fmax3(mx, fabsf(f.x), fabsf(f.y));
            }
          }
        }
        const int ex = static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu) - 127;
        const int kq = mx > 0.f ? min(max(14 - ex, -126), 126) : 0;
        sc = __uint_as_float(static_cast<uint32_t>(kq + 127) << 23);
        qmul *= __uint_as_float(static_cast<uint32_t>(127 - kq) << 23);
      }
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        uint4 qv[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) qv[c] = src ? src[8 * h + c] : make_uint4(0u, 0u, 0u, 0u);
        if constexpr (F8 && !std::is_same<T, __half>::value) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t w[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = Mma<T>::unpack(w[e]);
              w[e] = Mma<__half>::pack(f.x * sc, f.y * sc);
            }
            qv[c] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(smem + h * S::kQPanel + r * 128 + ((c ^ (r & 7)) << 4)) = qv[c];
      }
      fence_proxy_async_smem();  // the tensor core reads the tile through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_qfull);
      return qmul;
    };

    int g0 = 0;  // key blocks of the items before this one
    if (!wait_all(bar_itemfull, 0)) bad = true;  // item 0 sits in slot 0
    float qmul = 0.f;
    if (!bad && items[0].nb >= 0) qmul = load_q(items[0]);
    // the item descriptions are read in shared memory, where they stay
    // until this warp releases the slot
    for (int it = 0; !bad && items[it & 1].nb >= 0; ++it) {
      const int slot = it & 1;
      const TcItem& d = items[slot];
      const int* tab = tables + slot * S::kMaxPages;
      const int tr = d.r0 + r;
      const bool valid = tr < d.R;
      const int pos = valid ? d.base + tr / G : -1;
      float m_ref = -INFINITY, l = 0.f;
      // a warp whose 32 rows are all padding (a tile of <= 96 rows) keeps
      // step with the others but computes nothing: its rows of P and O are
      // never read back
      const bool warp_pad = d.r0 + 32 * (warp & 3) >= d.R;
      for (int j = 0; j < d.nb; ++j) {
        const int g = g0 + j;
        // the block's key limits need no scores: keys kb0 + e with e <= lim
        // are causal for this row and inside the partition and the context
        const int kb0 = d.tok0 + j * S::kKeys;
        uint32_t pages_ok = 0;
#pragma unroll
        for (int p = 0; p < S::kPages; ++p) pages_ok |= loaded_in(d, tab, j * S::kPages + p) ? (1u << p) : 0u;
        const int lim = min(pos, d.tok1 - 1) - kb0;
        // plain block: every key in, and a positive scale, so the max can be
        // taken on the raw scores and the scale folded into the exponent
        const bool plain = __all_sync(kFull, lim >= S::kKeys - 1 && pages_ok == 0xFu && qmul > 0.f);
        if (!wait_all(bar_sfull + 8 * (g & 1), (g >> 1) & 1)) {
          bad = true;
          break;
        }
        tc_fence_after();
        if (warp_pad) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_pfull + 8 * (g & 1));
          continue;
        }
        const uint32_t scol = tmem + lane_off + S::kColS + 64 * (g & 1);
        uint32_t v[S::kKeys];
        tmem_ld64(scol, v);
        float x[S::kKeys];
        float mul = qmul;  // x * mul is the score in log2 units
        if (plain) {
#pragma unroll
          for (int k = 0; k < S::kKeys; ++k) x[k] = __uint_as_float(v[k]);
        } else {
          // masked keys to -inf, the scale applied here
#pragma unroll
          for (int k = 0; k < S::kKeys; ++k) {
            const bool ok = k <= lim && ((pages_ok >> (k >> 4)) & 1u);
            x[k] = ok ? __uint_as_float(v[k]) * qmul : -INFINITY;
          }
          mul = 1.f;
        }
        // block max: a tree of three-input maxima
        float t[S::kKeys / 4];
#pragma unroll
        for (int k = 0; k < S::kKeys / 4; ++k) t[k] = fmax3(x[4 * k], x[4 * k + 1], fmaxf(x[4 * k + 2], x[4 * k + 3]));
#pragma unroll
        for (int w = S::kKeys / 4; w > 1; w /= 2)
#pragma unroll
          for (int k = 0; k < w / 2; ++k) t[k] = fmaxf(t[k], t[k + w / 2]);
        const float bm = t[0] * mul;
        // move the reference max only when this block exceeds it by 2^8
        float alpha = 1.f;
        bool rescale = false;
        if (bm > m_ref + 8.f) {
          alpha = exp2_sfu(m_ref - bm);  // 0 while no key was seen
          rescale = m_ref != -INFINITY && j > 0;
          l *= alpha;
          m_ref = bm;
        }
        // 2^(x mul - m) as one FFMA leaves the residual of the rounded max
        // product, up to half an ulp of m: harmless while |m| < 2^20 (under
        // 2^-4); past that the scores are rounded to their products first,
        // so the maximal one gives exactly 2^0
        if (__any_sync(kFull, fabsf(m_ref) >= 1048576.f && mul != 1.f)) {
#pragma unroll
          for (int k = 0; k < S::kKeys; ++k) x[k] *= mul;
          mul = 1.f;
        }
        const float nmr = m_ref == -INFINITY ? 0.f : -m_ref;
        uint32_t ph[S::kKeys / 2], pl[S::kKeys / 2];
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
        for (int k = 0; k < S::kKeys; k += 2) {
          const float p0 = exp2_sfu(fmaf(x[k], mul, nmr)), p1 = exp2_sfu(fmaf(x[k + 1], mul, nmr));
          acc[(k / 2) & 7] += p0 + p1;
          ph[k / 2] = M::pack(p0, p1);
          const float2 hv = M::unpack(ph[k / 2]);
          pl[k / 2] = M::pack(p0 - hv.x, p1 - hv.y);
        }
        const float sum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
        l += sum;
        if (__any_sync(kFull, rescale)) {
          // O holds the P.V of blocks < j: wait for the last of them, then
          // rescale this thread's row in tensor memory
          if (!wait_all(bar_pvdone, (g - 1) & 1)) {
            bad = true;
            break;
          }
          tc_fence_after();
          const float f = rescale ? alpha : 1.f;
#pragma unroll
          for (int h = 0; h < D / 32; ++h) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + S::kColO + 32 * h, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(tmem + lane_off + S::kColO + 32 * h, o);
          }
        }
        tmem_st32(scol, ph);
        tmem_st32(scol + 32, pl);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_pfull + 8 * (g & 1));
      }
      if (bad) break;
      // the next item's Q goes in while this item's last P.V runs
      const int nslot = (it + 1) & 1;
      if (!wait_all(bar_itemfull + 8 * nslot, ((it + 1) >> 1) & 1)) {
        bad = true;
        break;
      }
      const TcItem& nd = items[nslot];
      float nqmul = 0.f;
      if (nd.nb >= 0) {
        if (!wait_all(bar_qempty, it & 1)) {
          bad = true;
          break;
        }
        nqmul = load_q(nd);
      }
      // epilogue: the item's MMAs done (its final commit follows its last
      // P.V), then each row out of tensor memory
      if (!wait_all(bar_final, it & 1)) {
        bad = true;
        break;
      }
      if (!warp_pad) {
        tc_fence_after();
        const bool has = valid && pos >= d.tok0;
        const size_t row = valid ? static_cast<size_t>(d.q0 + tr / G) * a.num_q_heads + d.kvh * G + tr % G : 0;
        // over an FP8 pool the V scale multiplies the output (or the
        // partial: the merge is linear in it)
        const float osc = F8 ? a.v_scale : 1.f;
        const float inv = has ? osc / l : 0.f;
#pragma unroll
        for (int h = 0; h < D / 32; ++h) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + S::kColO + 32 * h, o);
          if (!valid) continue;
          if (d.direct) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<T*>(a.out) + row * D + 32 * h);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                w[e] = has ? Mma<T>::pack(__uint_as_float(o[8 * q + 2 * e]) * inv,
                                          __uint_as_float(o[8 * q + 2 * e + 1]) * inv)
                           : 0u;
              dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else if (has) {
            float4* dst = reinterpret_cast<float4*>(a.ws_o + (row * a.num_parts + d.z) * D + 32 * h);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(__uint_as_float(o[4 * q]) * osc, __uint_as_float(o[4 * q + 1]) * osc,
                                   __uint_as_float(o[4 * q + 2]) * osc, __uint_as_float(o[4 * q + 3]) * osc);
          }
        }
        if (has && !d.direct) a.ws_ml[row * a.num_parts + d.z] = make_float2(m_ref, l);
      }
      g0 += d.nb;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar_oempty);                 // O may be overwritten
        mbar_arrive(bar_itemempty + 8 * slot);  // the slot may be refilled
      }
      qmul = nqmul;
    }
    if (bad && lane == 0) raise_error(PKV_ERR_TIMEOUT);
  }

  // ---- teardown ---------------------------------------------------------------
  tc_fence_before();
  const bool any_bad = __syncthreads_or(bad);
  tc_fence_after();
  if (any_bad && warp == 0 && lane == 0) {
    // the last block the producer issued into each stage lands before the
    // CTA exits
    for (int c = max(0, issued_k - NSK); c < issued_k; ++c)
      mbar_wait_bounded(bar_kfull + 8 * (c % NSK), (c / NSK) & 1);
    for (int c = max(0, issued_v - NSV); c < issued_v; ++c)
      mbar_wait_bounded(bar_vfull + 8 * (c % NSV), (c / NSV) & 1);
  }
  if (warp == 1) tmem_dealloc(tmem, S::kTmemCols);
}

}  // namespace pkv
