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
  static_assert(D % 64 == 0, "a tile row is a whole number of 128-byte boxes");
  static_assert(G >= 1 && G <= 8, "the group is the MMA's N = 8 dimension");
  static_assert(size_t(G) * (D + 2) * sizeof(float) <= size_t(kWarpStageBytes),
                "a warp's merge record must fit in its own stages");
  static_assert(kStage % 1024 == 0, "swizzled boxes need 1024-byte alignment");
};

template <typename T, int D, int G, int NWARPS, int NSTAGE>
__global__ void __launch_bounds__(NWARPS * 32)
    paged_decode_mma_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v) {
  using S = MmaShape<T, D, G, NWARPS, NSTAGE>;
  using M = Mma<T>;
  const int kvh = blockIdx.x;
  const int b = blockIdx.y;
  const int part = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g8 = lane >> 2;  // fragment row group
  const int t4 = lane & 3;   // thread in group

  int ctx = a.context_lens[b];
  if (ctx < 0 || ctx > a.max_ctx) {
    if (threadIdx.x == 0 && kvh == 0 && part == 0) raise_error(PKV_ERR_CONTEXT_RANGE);
    ctx = ctx < 0 ? 0 : a.max_ctx;
  }
  // shared-prefix mode: a sequence that starts with the prefix blocks only
  // covers its suffix here (the prefix pass covered the rest); one that
  // does not covers its whole context
  const bool cascade = a.prefix_blocks != nullptr;
  int tok_begin = 0;
  if (cascade) {
    int same = 1;
    for (int j = threadIdx.x; j < a.prefix_pages; j += NWARPS * 32)
      if (a.block_tables[static_cast<long long>(b) * a.bt_stride + j] != a.prefix_blocks[j]) same = 0;
    const bool conforming = __syncthreads_and(same) && ctx >= a.prefix_pages * kBlockSize;
    if (conforming) tok_begin = a.prefix_pages * kBlockSize;
    if (threadIdx.x == 0 && kvh == 0 && part == 0) a.conform[b] = conforming ? 1 : 0;
  }
  const int span = ctx - tok_begin;
  const int nparts = (span + a.partition - 1) / a.partition;
  if (part >= (nparts > 0 ? nparts : 1)) return;

  const int h0 = kvh * G;
  T* out = reinterpret_cast<T*>(a.out) + (static_cast<size_t>(b) * a.num_q_heads + h0) * D;
  if (span == 0) {
    if (tok_begin == 0)  // nothing to attend to at all
      for (int i = threadIdx.x; i < G * D; i += NWARPS * 32) out[i] = Fmt<T>::from_f32(0.f);
    return;
  }

  const int tok0 = tok_begin + part * a.partition;
  const int tok1 = min(ctx, tok0 + a.partition);
  const int pg0 = tok0 / kBlockSize;
  const int nblk = (tok1 - tok0 + kBlockSize - 1) / kBlockSize;
  const int my_n = warp < nblk ? (nblk - warp + NWARPS - 1) / NWARPS : 0;

  extern __shared__ unsigned char smem_raw[];
  // swizzled boxes want 1024-byte aligned destinations
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  unsigned char* smem = smem_raw + pad;
  unsigned char* my_stages = smem + static_cast<size_t>(warp) * S::kWarpStageBytes;
  const uint32_t stage0 = smem_addr(my_stages);
  const uint32_t bar0 = smem_addr(smem + S::kSmemStages) + warp * NSTAGE * 8;

  // lane j: physical block of this warp's j-th page (page warp + j*NWARPS)
  int my_phys = -1;
  if (lane < my_n) {
    const int e = a.block_tables[static_cast<long long>(b) * a.bt_stride + pg0 + warp + lane * NWARPS];
    if (e >= 0 && e < a.num_blocks)
      my_phys = e;
    else
      raise_error(PKV_ERR_BLOCK_RANGE);
  }
  if (lane == 0) {
    for (int s = 0; s < NSTAGE; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_barrier_init();
  }
  __syncwarp();

  auto issue = [&](int i) {
    const int phys = __shfl_sync(kFull, my_phys, i & 31);
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
#pragma unroll
  for (int i = 0; i < NSTAGE; ++i) issue(i);

  // B fragments of Q^T (k = d, n = head): head g8 of the group, zero past G
  uint32_t qb[S::kKSteps][2];
  {
    const T* qp = reinterpret_cast<const T*>(a.q) + (static_cast<size_t>(b) * a.num_q_heads + h0 + g8) * D;
#pragma unroll
    for (int ks = 0; ks < S::kKSteps; ++ks) {
      qb[ks][0] = g8 < G ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 2 * t4) : 0u;
      qb[ks][1] = g8 < G ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 8 + 2 * t4) : 0u;
    }
  }

  // O^T accumulator fragments: o[i] = rows d = 16 i + g8 (+8), heads 2 t4 (+1)
  float o[S::kKSteps][4];
#pragma unroll
  for (int i = 0; i < S::kKSteps; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY;  // running max of heads 2 t4, 2 t4 + 1 (log2 units)
  float l0 = 0.f, l1 = 0.f;              // this lane's share of their running sums
  uint32_t phase_bits = 0;
  int consumed = 0;

  // per-lane ldmatrix row/chunk selectors
  const int lm = lane >> 3;   // which 8x8 matrix this lane addresses
  const int lr = lane & 7;    // row within it

  for (int i = 0; i < my_n; ++i) {
    const int s = i % NSTAGE;
    bool ok = mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
    phase_bits ^= 1u << s;
    ok = __all_sync(kFull, ok);
    if (!ok) {
      if (lane == 0) raise_error(PKV_ERR_TIMEOUT);
      break;
    }
    consumed = i + 1;
    const int phys = __shfl_sync(kFull, my_phys, i);
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
      // (2) scale, mask the tail, online softmax per head
      const bool v_lo = g8 < nvalid, v_hi = g8 + 8 < nvalid;
      const float x0 = v_lo ? sc[0] * a.qk_scale : -INFINITY;  // token g8,   head 2 t4
      const float x1 = v_lo ? sc[1] * a.qk_scale : -INFINITY;  // token g8,   head 2 t4 + 1
      const float x2 = v_hi ? sc[2] * a.qk_scale : -INFINITY;  // token g8+8, head 2 t4
      const float x3 = v_hi ? sc[3] * a.qk_scale : -INFINITY;  // token g8+8, head 2 t4 + 1
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
      for (int msk = 4; msk <= 16; msk <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, msk));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, msk));
      }
      const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
      const float al0 = exp2f(m0 - n0), al1 = exp2f(m1 - n1);
      m0 = n0;
      m1 = n1;
      const float p0 = exp2f(x0 - n0), p1 = exp2f(x1 - n1), p2 = exp2f(x2 - n0), p3 = exp2f(x3 - n1);
      l0 = fmaf(l0, al0, p0 + p2);
      l1 = fmaf(l1, al1, p1 + p3);
#pragma unroll
      for (int mt = 0; mt < S::kKSteps; ++mt) {
        o[mt][0] *= al0;
        o[mt][1] *= al1;
        o[mt][2] *= al0;
        o[mt][3] *= al1;
      }
      // (3) P^T as B fragments, split into hi + lo 16-bit parts
      const uint32_t top_hi = M::pack(p0, p1), bot_hi = M::pack(p2, p3);
      const float2 th = M::unpack(top_hi), bh = M::unpack(bot_hi);
      const uint32_t top_lo = M::pack(p0 - th.x, p1 - th.y), bot_lo = M::pack(p2 - bh.x, p3 - bh.y);
      const uint32_t pb0 = movm_t(top_hi), pb1 = movm_t(bot_hi);
      const uint32_t pl0 = movm_t(top_lo), pl1 = movm_t(bot_lo);
      // V^T fragment halves of tokens past the context are zeroed
      uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
      if (nvalid < kBlockSize) {
        keep_lo = (2 * t4 < nvalid ? 0x0000ffffu : 0u) | (2 * t4 + 1 < nvalid ? 0xffff0000u : 0u);
        keep_hi = (2 * t4 + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * t4 + 9 < nvalid ? 0xffff0000u : 0u);
      }
      // (4) O^T += V^T . P^T
      {
        const int row = lr + ((lm >> 1) << 3);
#pragma unroll
        for (int mt = 0; mt < S::kKSteps; ++mt) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(vt + swz(row, 2 * mt + (lm & 1)), a0, a1, a2, a3);
          a0 &= keep_lo;
          a1 &= keep_lo;
          a2 &= keep_hi;
          a3 &= keep_hi;
          M::run(o[mt], a0, a1, a2, a3, pb0, pb1);
          M::run(o[mt], a0, a1, a2, a3, pl0, pl1);
        }
      }
    }
    __syncwarp();
    issue(i + NSTAGE);
  }

  // after a give-up, wait (bounded) for the copies still in flight
  if (consumed < my_n) {
    const int last = min(my_n, consumed + NSTAGE);
    for (int i = consumed + 1; i < last; ++i) {
      const int s = i % NSTAGE;
      mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
      phase_bits ^= 1u << s;
    }
  }

  // running sums over the lanes of each head (same t4)
#pragma unroll
  for (int msk = 4; msk <= 16; msk <<= 1) {
    l0 += __shfl_xor_sync(kFull, l0, msk);
    l1 += __shfl_xor_sync(kFull, l1, msk);
  }

  // warp record [o: G x D][m: G][l: G] in the warp's own (drained) stages
  float* rec = reinterpret_cast<float*>(my_stages);
  const int ha = 2 * t4, hb = 2 * t4 + 1;
#pragma unroll
  for (int mt = 0; mt < S::kKSteps; ++mt) {
    const int d0 = 16 * mt + g8;
    if (ha < G) {
      rec[ha * D + d0] = o[mt][0];
      rec[ha * D + d0 + 8] = o[mt][2];
    }
    if (hb < G) {
      rec[hb * D + d0] = o[mt][1];
      rec[hb * D + d0 + 8] = o[mt][3];
    }
  }
  if (g8 == 0) {
    if (ha < G) {
      rec[G * D + ha] = m0;
      rec[G * D + G + ha] = l0;
    }
    if (hb < G) {
      rec[G * D + hb] = m1;
      rec[G * D + G + hb] = l1;
    }
  }
  __syncthreads();

  // merge the warps in a fixed order
  for (int idx = threadIdx.x; idx < G * D; idx += NWARPS * 32) {
    const int g = idx / D;
    const int d = idx % D;
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w)
      Mx = fmaxf(Mx, reinterpret_cast<const float*>(smem + w * S::kWarpStageBytes)[G * D + g]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) {
      const float* r = reinterpret_cast<const float*>(smem + w * S::kWarpStageBytes);
      const float sc = exp2f(r[G * D + g] - Mx);
      num = fmaf(sc, r[g * D + d], num);
      den = fmaf(sc, r[G * D + G + g], den);
    }
    if (nparts == 1 && !cascade) {
      out[idx] = Fmt<T>::from_f32(num / den);
    } else {
      const size_t row = (static_cast<size_t>(b) * a.num_q_heads + h0 + g) * a.num_parts + part;
      a.ws_o[row * D + d] = num;
      if (d == 0) a.ws_ml[row] = make_float2(Mx, den);
    }
  }
}

}  // namespace pkv
