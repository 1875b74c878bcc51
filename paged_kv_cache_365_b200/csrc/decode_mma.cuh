// Paged decode attention on the tensor cores (fp16 / bf16 caches).
//
// Same computation and work split as paged_decode_partition_kernel
// (decode.cuh): one CTA per (kv-head, sequence, partition), warp w walks
// pages w, w+NWARPS, ... with its own ring of staged tiles, per-warp online
// softmax, fixed-order merge, direct output or split-K workspace.  What
// changes is how a 16-token page is consumed:
//
//  * Staging: each (block, kv-head) tile is loaded with tensor-map TMA
//    (cp.async.bulk.tensor.2d) in boxes of 16 rows x 64 elements with the
//    128-byte swizzle, so that the 8-row ldmatrix reads below hit eight
//    different bank groups.  The cache is viewed as a 2-D tensor
//    [num_blocks * Hkv * 16 rows, D columns]; a tile is rows
//    (block * Hkv + kv_head) * 16 .. +15.
//  * Q.K: S^T[16 tokens x 8 heads] = K[16 x D] . Q^T[D x 8] with
//    mma.sync m16n8k16 (fp32 accumulate): A = K from shared memory via
//    ldmatrix, B = the group's queries held in registers (heads >= G are
//    zero).  The GQA group is the MMA's N dimension, so the cost of a page
//    does not grow with G (G <= 8).
//  * Softmax on the accumulator fragment: a lane holds two tokens of two
//    heads; per-head max over the page takes three shuffles.
//  * P.V: O^T[D x 8] += V^T[D x 16] . P^T[16 x 8]: A = V^T via
//    ldmatrix.trans, B = P^T, obtained from the score fragment by
//    movmatrix.trans.  P is fed as hi + lo 16-bit parts (two MMAs), so its
//    rounding error is ~2^-16 relative instead of 2^-8 (bf16) / 2^-11 (fp16).
//  * Tail rows of the last page (tokens past the context) are masked in
//    registers: their logits become -inf and their V fragment halves are
//    zeroed, so a NaN in an unused slot never meets a zero weight.
#pragma once

#include <cuda.h>
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "decode.cuh"

namespace pkv {

// ----------------------------------------------------------------------------
// tensor-core and TMA primitives (inline PTX)
// ----------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

template <typename T>
struct Mma;

template <>
struct Mma<__nv_bfloat16> {
  __device__ __forceinline__ static void run(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  // (x -> low half, y -> high half), round to nearest even
  __device__ __forceinline__ static uint32_t pack(float x, float y) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  __device__ __forceinline__ static float2 unpack(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
  static constexpr CUtensorMapDataType kTmaType = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
};

template <>
struct Mma<__half> {
  __device__ __forceinline__ static void run(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  __device__ __forceinline__ static uint32_t pack(float x, float y) {
    const __half2 h = __floats2half2_rn(x, y);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  __device__ __forceinline__ static float2 unpack(uint32_t u) {
    return __half22float2(*reinterpret_cast<const __half2*>(&u));
  }
  static constexpr CUtensorMapDataType kTmaType = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
};

// 2-D tensor-map load of one box into shared memory, completing on `bar`.
// x (the inner coordinate) is a multiple of 64 elements, so the copy starts
// on a 128-byte boundary.  No multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Byte offset of 16-byte chunk `chunk` (0..D/8-1) of row `row` (0..15) in a
// tile stored as D/64 boxes of [16 rows][128 B] with the 128-byte swizzle
// (chunk index XOR row mod 8 within each 128-byte row).
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>((chunk >> 3) * 2048 + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}


template <typename T, int D, int G, int NWARPS, int NSTAGE>
struct MmaShape {
  static constexpr int kTile = kBlockSize * D * 2;   // bytes of a (block, kv-head) tile
  static constexpr int kStage = 2 * kTile;           // K + V
  static constexpr int kBoxes = D / 64;              // 16 x 64 boxes per tile
  static constexpr int kKSteps = D / 16;             // QK k-steps; also PV m-tiles
  static constexpr int kWarpStageBytes = NSTAGE * kStage;
  static constexpr size_t kSmemStages = size_t(NWARPS) * kWarpStageBytes;
  static constexpr size_t kSmemBars = size_t(NWARPS) * NSTAGE * 8;
  static constexpr size_t kSmem = 1024 /* alignment slack */ + kSmemStages + kSmemBars;
  // warp record: o[8][D], m[8], l[8] (8 query columns, the MMA's N)
  static constexpr int kRecM = 8 * D, kRecL = 8 * D + 8;
  // block-table entries a lane holds: a warp's pages of a 2048-token partition
  static constexpr int kTab = (128 + 32 * NWARPS - 1) / (32 * NWARPS);
  static_assert(D % 64 == 0, "a tile row is a whole number of 128-byte boxes");
  static_assert(G >= 1 && G <= 8, "the group is the MMA's N = 8 dimension");
  static_assert(size_t(8) * (D + 2) * sizeof(float) <= size_t(kWarpStageBytes),
                "a warp's merge record must fit in its own stages");
  static_assert(kStage % 1024 == 0, "swizzled boxes need 1024-byte alignment");
};

// Prefix role, one warp: 16 queries of kv-head kvh (query i = sequence i / G,
// head i % G) over pages [pg0, pg0 + nblk) of the shared prefix, queries as
// the MMA's M dimension:
//   S[16 q x 16 tok] = Q[16 x D] . K^T     (A = Q in registers, B = K via ldmatrix)
//   O[16 q x D]     += P[16 x 16] . V      (A = P straight from the S fragments,
//                                           B = V via ldmatrix.trans; hi + lo P)
// Every warp of the CTA walks all pages with its own stages (the tiles come
// from L2 after the first warp's read) and writes its queries' partial
// results directly: warps have disjoint queries, nothing to merge.
template <typename T, int D, int G, int NSTAGE>
__device__ __forceinline__ bool prefix_warp(const DecodeArgs& a, const CUtensorMap* tmap_k,
                                            const CUtensorMap* tmap_v, int kvh, int q0, int chunk, int pg0,
                                            int nblk, uint32_t stage0, uint32_t bar0, uint32_t& phase_bits,
                                            int lane) {
  using M = Mma<T>;
  constexpr int kTile = kBlockSize * D * 2, kStage = 2 * kTile, kKSteps = D / 16, kNTiles = D / 8;
  const int g8 = lane >> 2, t4 = lane & 3, lm = lane >> 3, lr = lane & 7;
  const int nq = a.num_seqs * G;
  // lane j: block of page pg0 + j (nblk <= 32)
  int my_phys = -1;
  if (lane < nblk) {
    const int e = a.prefix_ident ? pg0 + lane : a.prefix_blocks[pg0 + lane];
    if (e >= 0 && e < a.num_blocks)
      my_phys = e;
    else
      raise_error(PKV_ERR_BLOCK_RANGE);
  }
  auto issue = [&](int i) {
    const int phys = __shfl_sync(kFull, my_phys, i & 31);
    if (lane == 0 && i < nblk) {
      const uint32_t bar = bar0 + 8 * (i % NSTAGE);
      if (phys >= 0) {
        const uint32_t dst = stage0 + (i % NSTAGE) * kStage;
        const int y = (phys * a.num_kv_heads + kvh) * kBlockSize;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, kStage);
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_2d(dst + bx * 2048, tmap_k, bx * 64, y, bar);
          tma_load_2d(dst + kTile + bx * 2048, tmap_v, bx * 64, y, bar);
        }
      } else {
        mbar_arrive(bar);
      }
    }
  };
#pragma unroll
  for (int i = 0; i < NSTAGE; ++i) issue(i);

  // A fragments of the 16 queries (rows past the batch are zero)
  uint32_t qa[kKSteps][4];
  {
    const int ra = q0 + g8, rb = q0 + g8 + 8;
    const T* pa = ra < nq ? reinterpret_cast<const T*>(a.q) +
                                (static_cast<size_t>(ra / G) * a.num_q_heads + kvh * G + ra % G) * D
                          : nullptr;
    const T* pb = rb < nq ? reinterpret_cast<const T*>(a.q) +
                                (static_cast<size_t>(rb / G) * a.num_q_heads + kvh * G + rb % G) * D
                          : nullptr;
#pragma unroll
    for (int ks = 0; ks < kKSteps; ++ks) {
      const int d = ks * 16 + 2 * t4;
      qa[ks][0] = pa ? *reinterpret_cast<const uint32_t*>(pa + d) : 0u;
      qa[ks][1] = pb ? *reinterpret_cast<const uint32_t*>(pb + d) : 0u;
      qa[ks][2] = pa ? *reinterpret_cast<const uint32_t*>(pa + d + 8) : 0u;
      qa[ks][3] = pb ? *reinterpret_cast<const uint32_t*>(pb + d + 8) : 0u;
    }
  }
  float o[kNTiles][4];
#pragma unroll
  for (int j = 0; j < kNTiles; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float mA = -INFINITY, mB = -INFINITY;  // rows g8, g8 + 8
  float lA = 0.f, lB = 0.f;

  int consumed = 0;
  bool ok = true;
  for (int i = 0; i < nblk; ++i) {
    const int s = i % NSTAGE;
    ok = mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
    ok = __all_sync(kFull, ok);
    if (!ok) {
      if (lane == 0) raise_error(PKV_ERR_TIMEOUT);
      break;
    }
    phase_bits ^= 1u << s;  // (a stage that timed out keeps its parity: the drain waits on it again)
    consumed = i + 1;
    if (__shfl_sync(kFull, my_phys, i) >= 0) {
      const uint32_t kt = stage0 + s * kStage;
      const uint32_t vt = kt + kTile;
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int row = lr + ((lm >> 1) << 3);  // token
#pragma unroll
        for (int ks = 0; ks < kKSteps; ++ks) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kt + swz(row, 2 * ks + (lm & 1)), b0, b1, b2, b3);
          M::run(sc[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
          M::run(sc[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
        }
      }
      float x[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) x[nt][e] = sc[nt][e] * a.qk_scale;
      float mxA = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
      float mxB = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
      // the reference max moves only when a score passes it by more than
      // 2^8 (one vote a page otherwise; see the sequence role)
      if (__any_sync(kFull, mxA > mA + 8.f || mxB > mB + 8.f)) {
#pragma unroll
        for (int msk = 1; msk <= 2; msk <<= 1) {
          mxA = fmaxf(mxA, __shfl_xor_sync(kFull, mxA, msk));
          mxB = fmaxf(mxB, __shfl_xor_sync(kFull, mxB, msk));
        }
        const float nA = fmaxf(mA, mxA), nB = fmaxf(mB, mxB);
        const float alA = exp2_sfu(mA - nA), alB = exp2_sfu(mB - nB);
        mA = nA;
        mB = nB;
        lA *= alA;
        lB *= alB;
#pragma unroll
        for (int j = 0; j < kNTiles; ++j) {
          o[j][0] *= alA;
          o[j][1] *= alA;
          o[j][2] *= alB;
          o[j][3] *= alB;
        }
      }
      float p[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        p[nt][0] = exp2_sfu(x[nt][0] - mA);
        p[nt][1] = exp2_sfu(x[nt][1] - mA);
        p[nt][2] = exp2_sfu(x[nt][2] - mB);
        p[nt][3] = exp2_sfu(x[nt][3] - mB);
      }
      lA += p[0][0] + p[0][1] + p[1][0] + p[1][1];
      lB += p[0][2] + p[0][3] + p[1][2] + p[1][3];
      uint32_t ph[4], pl[4];
      {
        const float v[4][2] = {{p[0][0], p[0][1]}, {p[0][2], p[0][3]}, {p[1][0], p[1][1]}, {p[1][2], p[1][3]}};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          ph[r] = M::pack(v[r][0], v[r][1]);
          const float2 hv = M::unpack(ph[r]);
          pl[r] = M::pack(v[r][0] - hv.x, v[r][1] - hv.y);
        }
      }
      {
        const int row = lr + ((lm & 1) << 3);  // token
#pragma unroll
        for (int j = 0; j < kNTiles; j += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vt + swz(row, j + (lm >> 1)), b0, b1, b2, b3);
          M::run(o[j], ph[0], ph[1], ph[2], ph[3], b0, b1);
          M::run(o[j], pl[0], pl[1], pl[2], pl[3], b0, b1);
          M::run(o[j + 1], ph[0], ph[1], ph[2], ph[3], b2, b3);
          M::run(o[j + 1], pl[0], pl[1], pl[2], pl[3], b2, b3);
        }
      }
    }
    __syncwarp();
    issue(i + NSTAGE);
  }
  if (consumed < nblk) {  // after a give-up: wait (bounded) for copies in flight
    const int last = min(nblk, consumed + NSTAGE);
    for (int i = consumed; i < last; ++i) {
      const int s = i % NSTAGE;
      mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
      phase_bits ^= 1u << s;
    }
    return false;
  }
#pragma unroll
  for (int msk = 1; msk <= 2; msk <<= 1) {
    lA += __shfl_xor_sync(kFull, lA, msk);
    lB += __shfl_xor_sync(kFull, lB, msk);
  }
  const int rows[2] = {q0 + g8, q0 + g8 + 8};
  const float ms[2] = {mA, mB}, ls[2] = {lA, lB};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qi = rows[r];
    if (qi >= nq) continue;
    const size_t slot = (static_cast<size_t>(qi / G) * a.num_q_heads + kvh * G + qi % G) * a.num_chunks + chunk;
    float* dst = a.wp_o + slot * D;
#pragma unroll
    for (int j = 0; j < kNTiles; ++j)
      *reinterpret_cast<float2*>(dst + 8 * j + 2 * t4) =
          make_float2(o[j][2 * r] * a.prefix_out_scale, o[j][2 * r + 1] * a.prefix_out_scale);
    if (t4 == 0) a.wp_ml[slot] = make_float2(ms[r], ls[r]);
  }
  return true;
}

// The step's writes for sequence b and kv-head kvh ("PagedAttention 与 vLLM
// 推理加速" §3.2(3): the shared partial block is copied before the writer
// appends; "vLLM + PagedAttention：打造高并发LLM推理引擎", "它是怎么工作的": the
// new token goes into its slot), made by the one warp that later stages the
// sequence's last page: rows 0 .. rows-1 of the copy whose destination is
// the slot's block, then the token.  The stores are issued here and fenced
// for the async proxy just before that warp's TMA load of the page (see
// the issue step of the kernel), so their latency hides behind the pages
// streamed before it.
template <typename T, int D>
__device__ __forceinline__ void fused_step_append(const DecodeArgs& a, int b, int kvh, int lane) {
  constexpr int kRowChunks = D * static_cast<int>(sizeof(T)) / 16;  // 16-byte chunks of a row
  const int64_t s = a.slots[b];
  const int64_t blk = s >= 0 ? s / kBlockSize : -1;
  const bool ok = s >= 0 && blk < a.num_blocks;
  if (s >= 0 && !ok && lane == 0) raise_error(PKV_ERR_SLOT_RANGE);
  if (!ok) return;
  // the copy into this block, if any: every lane scans its share of the
  // list with independent loads (one round trip), the first match wins
  int first = 0x7fffffff;
  for (int i = lane; i < a.n_copies; i += 32)
    if (a.copies[3 * i + 1] == static_cast<int>(blk)) first = min(first, i);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) first = min(first, __shfl_xor_sync(kFull, first, m));
  int src = -1, rows = 0;
  if (first != 0x7fffffff) {
    src = a.copies[3 * first];
    rows = a.copies[3 * first + 2];
  }
  if (src >= 0 && (src >= a.num_blocks || rows < 0 || rows > kBlockSize)) {
    if (lane == 0) raise_error(PKV_ERR_COPY_RANGE);
    src = -1;
  }
  const size_t head = static_cast<size_t>(kBlockSize) * kRowChunks;  // chunks of one (block, kv-head) tile
  uint4* kc = reinterpret_cast<uint4*>(const_cast<unsigned char*>(a.k_cache));
  uint4* vc = reinterpret_cast<uint4*>(const_cast<unsigned char*>(a.v_cache));
  if (src >= 0) {
    const size_t from = (static_cast<size_t>(src) * a.num_kv_heads + kvh) * head;
    const size_t to = (static_cast<size_t>(blk) * a.num_kv_heads + kvh) * head;
    for (int e = lane; e < 2 * rows * kRowChunks; e += 32) {
      uint4* c = e < rows * kRowChunks ? kc : vc;
      const int k = e < rows * kRowChunks ? e : e - rows * kRowChunks;
      c[to + k] = c[from + k];
    }
  }
  __syncwarp();  // (the token's row may lie inside the copied rows)
  const size_t dst = (static_cast<size_t>(blk) * a.num_kv_heads + kvh) * head +
                     static_cast<size_t>(s % kBlockSize) * kRowChunks;
  const size_t in = (static_cast<size_t>(b) * a.num_kv_heads + kvh) * kRowChunks;
  for (int e = lane; e < 2 * kRowChunks; e += 32) {
    if (e < kRowChunks)
      kc[dst + e] = reinterpret_cast<const uint4*>(a.k_new)[in + e];
    else
      vc[dst + e - kRowChunks] = reinterpret_cast<const uint4*>(a.v_new)[in + e - kRowChunks];
  }
}

// One CTA of 4 warps does one of two jobs:
//  * sequence role: the G query heads of (sequence b, kv-head) over the
//    partitions part, part + Z, ... of the sequence's context (in a cascade
//    launch: of its suffix, when its table starts with the shared prefix);
//  * prefix role (cascade launch only): 16 queries per warp, 64 per CTA, of
//    one kv-head, taken from consecutive sequences (query i = sequence
//    i / G, head i % G), over one chunk of the shared prefix pages
//    (prefix_warp).  The prefix tiles are read from L2 by every query
//    group; HBM sees them once.
// Grid: plain (Hkv, B, Z); cascade (Hkv, QG * NC + B * Z) with the prefix
// CTAs first, so they start early and overlap the suffix streaming.
template <typename T, int D, int G, int NWARPS, int NSTAGE, bool kCascade>
__global__ void __launch_bounds__(NWARPS * 32)
    paged_decode_mma_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v) {
  // a deferred wait lets the dependents launch at once, but the
  // prerequisite launch is still waited for: by the warps that stage the
  // pages it writes, and by every CTA before it exits (below)
  if (a.defer_wait)
    pdl_trigger();
  else
    pdl_enter();
  using S = MmaShape<T, D, G, NWARPS, NSTAGE>;
  using M = Mma<T>;
  constexpr float kLazyMax = 8.f;  // the reference max moves only past 2^kLazyMax (see the softmax)
  // kPack (G <= 4): the spare query columns [G, 2G) repeat queries [0, G)
  // (identical scores, max and sum) and carry P's lo part where columns
  // [0, G) carry its hi part; the two columns of O^T are added at the end,
  // so P.V takes one MMA per m-tile instead of two
  constexpr bool kPack = G <= 4;
  const int kvh = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g8 = lane >> 2;  // fragment row group (also: this lane's query column)
  const int t4 = lane & 3;   // thread in group
  constexpr bool cascade = kCascade;  // launched by the shared-prefix entry point

  // ---- role, work range, query columns ------------------------------------
  bool prefix_role = false;
  int b = 0, part = 0, stride = gridDim.z, chunk = 0, qg = 0;
  if (cascade) {
    const int npre = a.num_qgroups * a.num_chunks;
    const int yy = static_cast<int>(blockIdx.y) + a.y_offset;  // a split launch covers part of the roles
    if (yy < npre) {
      prefix_role = true;
      qg = yy / a.num_chunks;
      chunk = yy % a.num_chunks;
    } else {
      const int y = yy - npre;
      b = y % a.num_seqs;
      part = y / a.num_seqs;
    }
    stride = a.suffix_z;
  } else {
    b = blockIdx.y;
    part = blockIdx.z;
  }

  int ctx = 0, tok_begin = 0, nparts = 0, span = 0;
  if (!prefix_role) {
    // A sequence whose table starts with the prefix blocks covers only its
    // suffix (the prefix role covers the rest); one that does not covers
    // its whole context.  The check's loads go out with the length's.
    int same = 1;
    if (cascade)
      for (int j = threadIdx.x; j < a.prefix_pages; j += NWARPS * 32)
        if (a.block_tables[static_cast<long long>(b) * a.bt_stride + j] != a.prefix_blocks[j]) same = 0;
    ctx = a.context_lens[b];
    if (ctx < 0 || ctx > a.max_ctx) {
      if (threadIdx.x == 0 && kvh == 0 && part == 0) raise_error(PKV_ERR_CONTEXT_RANGE);
      ctx = ctx < 0 ? 0 : a.max_ctx;
    }
    if (cascade) {
      const bool conforming = __syncthreads_and(same) && ctx >= a.prefix_pages * kBlockSize;
      if (conforming) tok_begin = a.prefix_pages * kBlockSize;
      if (threadIdx.x == 0 && kvh == 0 && part == 0) a.conform[b] = conforming ? 1 : 0;
    }
    span = ctx - tok_begin;
    nparts = (span + a.partition - 1) / a.partition;
    if (part >= (nparts > 0 ? nparts : 1)) {
      if (a.defer_wait && threadIdx.x == 0) pdl_wait();
      return;
    }
    if (span == 0) {
      if (tok_begin == 0) {  // nothing to attend to at all
        T* out = reinterpret_cast<T*>(a.out) + (static_cast<size_t>(b) * a.num_q_heads + kvh * G) * D;
        for (int i = threadIdx.x; i < G * D; i += NWARPS * 32) out[i] = Fmt<T>::from_f32(0.f);
      }
      if (a.defer_wait && threadIdx.x == 0) pdl_wait();
      return;
    }
  } else {
    nparts = 1;
  }
  // query columns of this CTA: the G heads of sequence b
  const int ncol = G;
  auto col_valid = [&](int n) { return n < ncol; };
  auto col_row = [&](int n) -> size_t {  // row of q / out for query column n
    return static_cast<size_t>(b) * a.num_q_heads + kvh * G + n;
  };

  extern __shared__ unsigned char smem_raw[];
  // swizzled boxes want 1024-byte aligned destinations
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  unsigned char* smem = smem_raw + pad;
  unsigned char* my_stages = smem + static_cast<size_t>(warp) * S::kWarpStageBytes;
  const uint32_t stage0 = smem_addr(my_stages);
  const uint32_t bar0 = smem_addr(smem + S::kSmemStages) + warp * NSTAGE * 8;
  if (lane == 0) {
    for (int s = 0; s < NSTAGE; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_barrier_init();
  }
  __syncwarp();

  uint32_t phase_bits = 0;  // barrier phase parity per stage (carries across partitions)
  if (cascade && prefix_role) {
    // warp w: queries (qg * NWARPS + w) * 16 .. + 15 over the chunk's pages
    const int pg0 = chunk * a.chunk_pages;
    const int nblk = min(a.prefix_pages - pg0, a.chunk_pages);
    prefix_warp<T, D, G, NSTAGE>(a, &tmap_k, &tmap_v, kvh, (qg * NWARPS + warp) * 16, chunk, pg0, nblk, stage0,
                                 bar0, phase_bits, lane);
    if (a.defer_wait && threadIdx.x == 0) pdl_wait();
    return;
  }

  // B fragments of Q^T (k = d, n = query column g8), zero past the columns
  // (with kPack the columns [G, 2G) repeat queries [0, G))
  uint32_t qb[S::kKSteps][2];
  {
    const bool ok = kPack ? g8 < 2 * ncol : col_valid(g8);
    const T* qp = reinterpret_cast<const T*>(a.q) + (ok ? col_row(g8 & (G - 1)) : 0) * D;
#pragma unroll
    for (int ks = 0; ks < S::kKSteps; ++ks) {
      qb[ks][0] = ok ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 2 * t4) : 0u;
      qb[ks][1] = ok ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 8 + 2 * t4) : 0u;
    }
  }
  // per-lane ldmatrix row/chunk selectors
  const int lm = lane >> 3;  // which 8x8 matrix this lane addresses
  const int lr = lane & 7;   // row within it
  bool timed_out = false;

  for (int pidx = part; pidx < nparts; pidx += stride) {
    // pages of this work item: a partition of the sequence, or a prefix chunk
    const int tok0 = tok_begin + pidx * a.partition;
    const int tok1 = min(ctx, tok0 + a.partition);
    const int pg0 = tok0 / kBlockSize;
    const int nblk = (tok1 - tok0 + kBlockSize - 1) / kBlockSize;
    const int my_n = warp < nblk ? (nblk - warp + NWARPS - 1) / NWARPS : 0;  // <= 32 * S::kTab
    // a fused step: the warp that stages the sequence's last page (page
    // nblk - 1 of the last partition, its page `last_i`) writes the new
    // token and its copy-on-write copy first, and fences them before that
    // page's TMA load
    int last_i = -1;
    if (!prefix_role && (a.slots != nullptr || a.defer_wait) && pidx == nparts - 1 && warp == (nblk - 1) % NWARPS)
      last_i = (nblk - 1) / NWARPS;

    // lane j: physical blocks of this warp's pages j, j + 32, ... (page
    // warp + j*NWARPS of the partition, and so on)
    int my_phys[S::kTab];
#pragma unroll
    for (int h = 0; h < S::kTab; ++h) {
      my_phys[h] = -1;
      const int j = lane + 32 * h;
      if (j < my_n) {
        const int pg = pg0 + warp + j * NWARPS;
        const int e = a.block_tables[static_cast<long long>(b) * a.bt_stride + pg];
        if (e >= 0 && e < a.num_blocks)
          my_phys[h] = e;
        else
          raise_error(PKV_ERR_BLOCK_RANGE);
      }
    }
    auto phys_of = [&](int i) {  // block of this warp's page i (all lanes)
      int r = -1;
#pragma unroll
      for (int h = 0; h < S::kTab; ++h) {
        const int v = __shfl_sync(kFull, my_phys[h], i & 31);
        if ((i >> 5) == h) r = v;
      }
      return r;
    };

    auto issue = [&](int i) {
      const int phys = phys_of(i);
      if (i == last_i) {  // the step's writes into this page (made below, or by the
                          // preceding launch), visible to the TMA read
        if (a.defer_wait) pdl_wait();
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncwarp();
      }
      if (lane == 0 && i < my_n) {
        const uint32_t bar = bar0 + 8 * (i % NSTAGE);
        if (phys >= 0) {
          const uint32_t dst = stage0 + (i % NSTAGE) * S::kStage;
          const int y = (phys * a.num_kv_heads + kvh) * kBlockSize;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(bar, S::kStage);
#pragma unroll
          for (int bx = 0; bx < S::kBoxes; ++bx) {
            tma_load_2d(dst + bx * 2048, &tmap_k, bx * 64, y, bar);
            tma_load_2d(dst + S::kTile + bx * 2048, &tmap_v, bx * 64, y, bar);
          }
        } else {
          mbar_arrive(bar);
        }
      }
    };
    if (last_i >= 0) {
      // the warp's first pages go out before the step's writes, so that
      // the writes' latency overlaps them; the last page waits for them
#pragma unroll
      for (int i = 0; i < NSTAGE; ++i)
        if (i != last_i) issue(i);
      if (a.slots != nullptr) fused_step_append<T, D>(a, b, kvh, lane);
      if (last_i < NSTAGE) issue(last_i);
    } else {
#pragma unroll
      for (int i = 0; i < NSTAGE; ++i) issue(i);
    }

    // O^T accumulator fragments: o[i] = rows d = 16 i + g8 (+8), columns 2 t4 (+1)
    float o[S::kKSteps][4];
#pragma unroll
    for (int i = 0; i < S::kKSteps; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY;  // running max of columns 2 t4, 2 t4 + 1 (log2 units)
    float l0 = 0.f, l1 = 0.f;              // this lane's share of their running sums
    int consumed = 0;

    for (int i = 0; i < my_n; ++i) {
      const int s = i % NSTAGE;
      bool ok = mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
      ok = __all_sync(kFull, ok);
      if (!ok) {
        if (lane == 0) raise_error(PKV_ERR_TIMEOUT);
        timed_out = true;
        break;
      }
      phase_bits ^= 1u << s;  // (a stage that timed out keeps its parity: the drain waits on it again)
      consumed = i + 1;
      const int phys = phys_of(i);
      if (phys >= 0) {
        const int page_tok = tok0 + (warp + i * NWARPS) * kBlockSize;
        const int nvalid = min(kBlockSize, tok1 - page_tok);
        const uint32_t kt = stage0 + s * S::kStage;
        const uint32_t vt = kt + S::kTile;

        // (1) S^T = K . Q^T
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        {
          const int row = lr + ((lm & 1) << 3);
#pragma unroll
          for (int ks = 0; ks < S::kKSteps; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(kt + swz(row, 2 * ks + (lm >> 1)), a0, a1, a2, a3);
            M::run(sc, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
          }
        }
        // (2) scale, mask the tail, online softmax per query column
        const bool v_lo = g8 < nvalid, v_hi = g8 + 8 < nvalid;
        const float x0 = v_lo ? sc[0] * a.qk_scale : -INFINITY;  // token g8,   column 2 t4
        const float x1 = v_lo ? sc[1] * a.qk_scale : -INFINITY;  // token g8,   column 2 t4 + 1
        const float x2 = v_hi ? sc[2] * a.qk_scale : -INFINITY;  // token g8+8, column 2 t4
        const float x3 = v_hi ? sc[3] * a.qk_scale : -INFINITY;  // token g8+8, column 2 t4 + 1
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
        // The reference max of a column moves only when one of the page's
        // scores passes it by more than 2^8 (so p <= 2^8): most pages then
        // need one vote, no reduction and no rescale.  Any reference is
        // exact once the same one scales l and O.
        if (__any_sync(kFull, mx0 > m0 + kLazyMax || mx1 > m1 + kLazyMax)) {
#pragma unroll
          for (int msk = 4; msk <= 16; msk <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, msk));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, msk));
          }
          const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
          const float al0 = exp2_sfu(m0 - n0), al1 = exp2_sfu(m1 - n1);
          m0 = n0;
          m1 = n1;
          l0 *= al0;
          l1 *= al1;
#pragma unroll
          for (int mt = 0; mt < S::kKSteps; ++mt) {
            o[mt][0] *= al0;
            o[mt][1] *= al1;
            o[mt][2] *= al0;
            o[mt][3] *= al1;
          }
        }
        const float p0 = exp2_sfu(x0 - m0), p1 = exp2_sfu(x1 - m1), p2 = exp2_sfu(x2 - m0), p3 = exp2_sfu(x3 - m1);
        l0 += p0 + p2;
        l1 += p1 + p3;
        // (3) P^T as B fragments, split into hi + lo 16-bit parts (kPack:
        // one fragment, hi in columns [0, G), lo in [G, 2G))
        const uint32_t top_hi = M::pack(p0, p1), bot_hi = M::pack(p2, p3);
        const float2 th = M::unpack(top_hi), bh = M::unpack(bot_hi);
        uint32_t top_lo, bot_lo;
        if constexpr (kPack) {
          const bool h0 = 2 * t4 < G, h1 = 2 * t4 + 1 < G;
          top_lo = M::pack(h0 ? th.x : p0 - th.x, h1 ? th.y : p1 - th.y);
          bot_lo = M::pack(h0 ? bh.x : p2 - bh.x, h1 ? bh.y : p3 - bh.y);
        } else {
          top_lo = M::pack(p0 - th.x, p1 - th.y);
          bot_lo = M::pack(p2 - bh.x, p3 - bh.y);
        }
        const uint32_t pl0 = movm_t(top_lo), pl1 = movm_t(bot_lo);
        const uint32_t pb0 = kPack ? 0u : movm_t(top_hi), pb1 = kPack ? 0u : movm_t(bot_hi);
        // V^T fragment halves of tokens past the context are zeroed
        uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
        if (nvalid < kBlockSize) {
          keep_lo = (2 * t4 < nvalid ? 0x0000ffffu : 0u) | (2 * t4 + 1 < nvalid ? 0xffff0000u : 0u);
          keep_hi = (2 * t4 + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * t4 + 9 < nvalid ? 0xffff0000u : 0u);
        }
        // (4) O^T += V^T . P^T (the masks only on a partial last page)
        auto pv = [&](auto masked) {
          const int row = lr + ((lm >> 1) << 3);
#pragma unroll
          for (int mt = 0; mt < S::kKSteps; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(vt + swz(row, 2 * mt + (lm & 1)), a0, a1, a2, a3);
            if constexpr (decltype(masked)::value) {
              a0 &= keep_lo;
              a1 &= keep_lo;
              a2 &= keep_hi;
              a3 &= keep_hi;
            }
            if constexpr (!kPack) M::run(o[mt], a0, a1, a2, a3, pb0, pb1);
            M::run(o[mt], a0, a1, a2, a3, pl0, pl1);
          }
        };
        if (nvalid < kBlockSize)
          pv(std::true_type{});
        else
          pv(std::false_type{});
      }
      __syncwarp();
      issue(i + NSTAGE);
    }

    // after a give-up, wait (bounded) for the copies still in flight
    if (consumed < my_n) {
      const int last = min(my_n, consumed + NSTAGE);
      for (int i = consumed; i < last; ++i) {
        const int s = i % NSTAGE;
        mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
        phase_bits ^= 1u << s;
      }
    }

    // running sums over the lanes of each column (same t4)
#pragma unroll
    for (int msk = 4; msk <= 16; msk <<= 1) {
      l0 += __shfl_xor_sync(kFull, l0, msk);
      l1 += __shfl_xor_sync(kFull, l1, msk);
    }

    if constexpr (kPack) {  // query n: column n (hi) + column n + G (lo)
#pragma unroll
      for (int mt = 0; mt < S::kKSteps; ++mt) {
        if constexpr (G == 1) {
          o[mt][0] += o[mt][1];
          o[mt][2] += o[mt][3];
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) o[mt][e] += __shfl_xor_sync(kFull, o[mt][e], G / 2);
        }
      }
    }
    // warp record [o: 8 x D][m: 8][l: 8] in the warp's own (drained) stages
    float* rec = reinterpret_cast<float*>(my_stages);
    const int ha = 2 * t4, hb = 2 * t4 + 1;
    const bool va = ha < ncol, vb = hb < ncol;
#pragma unroll
    for (int mt = 0; mt < S::kKSteps; ++mt) {
      const int d0 = 16 * mt + g8;
      if (va) {
        rec[ha * D + d0] = o[mt][0];
        rec[ha * D + d0 + 8] = o[mt][2];
      }
      if (vb) {
        rec[hb * D + d0] = o[mt][1];
        rec[hb * D + d0 + 8] = o[mt][3];
      }
    }
    if (g8 == 0) {
      if (va) {
        rec[S::kRecM + ha] = m0;
        rec[S::kRecL + ha] = l0;
      }
      if (vb) {
        rec[S::kRecM + hb] = m1;
        rec[S::kRecL + hb] = l1;
      }
    }
    __syncthreads();

    // merge the warps in a fixed order
    for (int idx = threadIdx.x; idx < ncol * D; idx += NWARPS * 32) {
      const int g = idx / D;
      const int d = idx % D;
      if (!col_valid(g)) continue;
      float Mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < NWARPS; ++w)
        Mx = fmaxf(Mx, reinterpret_cast<const float*>(smem + w * S::kWarpStageBytes)[S::kRecM + g]);
      float num = 0.f, den = 0.f;
#pragma unroll
      for (int w = 0; w < NWARPS; ++w) {
        const float* r = reinterpret_cast<const float*>(smem + w * S::kWarpStageBytes);
        const float sc = exp2f(r[S::kRecM + g] - Mx);
        num = fmaf(sc, r[g * D + d], num);
        den = fmaf(sc, r[S::kRecL + g], den);
      }
      const size_t row = col_row(g);
      if (nparts == 1 && !cascade) {
        reinterpret_cast<T*>(a.out)[row * D + d] = Fmt<T>::from_f32(num / den);
      } else {
        const size_t wrow = row * a.num_parts + pidx;
        a.ws_o[wrow * D + d] = num;
        if (d == 0) a.ws_ml[wrow] = make_float2(Mx, den);
      }
    }
    // the records must be read before the next partition's copies land
    __syncthreads();
    if (__syncthreads_or(timed_out)) break;
  }
  // with a deferred wait the launch still ends after the one it follows
  if (a.defer_wait && threadIdx.x == 0) pdl_wait();
}

}  // namespace pkv
