// Paged decode over an FP8 (E4M3) KV cache, queries in fp16 or bf16.
//
// The cache stores code = E4M3(x / scale) with one scale for K and one for
// V (see pkv.h); a K/V tile is half the bytes of a 16-bit one, so a decode
// step streams half the HBM bytes.  Work split, staging and merging are
// those of paged_decode_mma_kernel (decode_mma.cuh): one CTA per (kv-head,
// sequence, partition), warp w walks pages w, w + NWARPS, ... with its own
// ring of TMA-staged tiles (16 rows x D bytes, swizzled), per-warp online
// softmax, fixed-order merge.  What changes is how a page is consumed:
//
//  * Q.K on the 16-bit tensor cores, S^T[16 tokens x 8] = K . Q^T: ldmatrix
//    reads the FP8 tile as 16-bit pairs, so lane (g, t) receives the 4
//    bytes d = 16c + 4t .. 16c + 4t + 3 of chunk c; each E4M3 pair is
//    converted exactly to two 16-bit values.  The MMA's k index 2t, 2t+1,
//    2t+8, 2t+9 then stands for d = 16c + 4t .. + 3, and the queries (the
//    B operand, in registers) are loaded in that same order of d, so the
//    dot product runs over the same pairs.
//  * P.V as O^T[D x 8 queries] += V^T[D x 16 tokens] . P^T[16 x 8], V^T the
//    A operand: a transposed byte load (ldmatrix .m16n16 .trans .b8) of two
//    16-token x 16-byte blocks of the V tile gives lane (g, t) the codes of
//    tokens 4t .. 4t + 3 at d = 16 i + g and 16 i + g + 8 of m-tiles i and
//    i + 1, each pair of them one exact E4M3 -> 16-bit conversion away from
//    an A register.  The MMA's k index then stands for the tokens in the
//    order 0, 1, 4, 5, 8, 9, 12, 13, 2, 3, 6, 7, ..., so the K tile's rows
//    are read in that order too (score_row_token) and the score rows, P^T's
//    k index and V^T's name the same tokens.  P^T is the B operand, taken from the score
//    fragment by movmatrix, in hi + lo 16-bit parts that accumulate into
//    the same registers (two MMAs per m-tile); O^T needs D/16 x 4
//    accumulator registers a lane, half of what O with the queries as M
//    would (whose rows past G are padding).
//  * The K scale is folded into the logit scale, the V scale into the
//    output.
//  * The MMAs run in fp16 whatever the query dtype: E4M3 -> fp16 is one
//    instruction per pair.  bf16 queries are brought into fp16 exactly by
//    a power-of-two factor per query row (its largest magnitude lands in
//    [2^14, 2^15)), undone on that row's logits.
#pragma once

#include <type_traits>

#include "decode_mma.cuh"

namespace pkv {

// E4M3 pair (low byte -> low half) to two fp16 values (exact: every E4M3
// value is an fp16 value).
template <typename T>
__device__ __forceinline__ uint32_t e4m3x2_to(uint32_t pair16);

template <>
__device__ __forceinline__ uint32_t e4m3x2_to<__half>(uint32_t pair16) {
  uint32_t d;
  const unsigned short a = static_cast<unsigned short>(pair16);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(a));
  return d;
}

// Four E4M3 codes (bytes 0..3 of w) to fp16 pairs: lo = bytes 0, 1 and
// hi = bytes 2, 3.
__device__ __forceinline__ void e4m3x4_to_f16(uint32_t w, uint32_t& lo, uint32_t& hi) {
  lo = e4m3x2_to<__half>(w & 0xffffu);
  hi = e4m3x2_to<__half>(w >> 16);
}


// Two 16 x 16 byte matrices, transposed: lanes 0-15 give the row addresses
// of the first, lanes 16-31 those of the second; lane (g, t) receives, of
// each matrix, the bytes (rows 4t .. 4t + 3, column g) in r0 / r2 and
// (rows 4t .. 4t + 3, column g + 8) in r1 / r3.
__device__ __forceinline__ void ldsm_b8_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// The token a score row stands for: rows 2t, 2t + 1 (and 2t + 8, 2t + 9)
// of S^T hold tokens 4t, 4t + 1 (and 4t + 2, 4t + 3), the order in which
// the transposed byte loads deliver V's tokens (ldsm_b8_x2_t), so that the
// k index of P^T and of V^T name the same token.
__device__ __forceinline__ int score_row_token(int row) {
  return ((row & 6) << 1) | (row & 1) | ((row >> 3) << 1);
}

// Byte offset of 16-byte chunk `chunk` of row `row` in an FP8 tile of 16
// rows x D bytes stored with the TMA swizzle matching its row length
// (128-byte rows: chunk ^ (row & 7); 64-byte rows: chunk ^ ((row >> 1) & 3)).
template <int D>
__device__ __forceinline__ uint32_t swz8(int row, int chunk) {
  if constexpr (D == 128)
    return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
  else
    return static_cast<uint32_t>(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

// Eight 16-bit values (T) to eight E4M3 codes: code = E4M3(x / scale), the
// division in float32, nearest value, ties to even, saturating at +-448.
template <typename T>
__device__ __forceinline__ uint2 quant8_e4m3(uint4 in, float scale) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint32_t packed[2];
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    unsigned short q2[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const float2 f = Mma<T>::unpack(w[2 * p + hh]);
      const float x0 = __fdiv_rn(f.x, scale), x1 = __fdiv_rn(f.y, scale);
      // first operand -> upper byte, second -> lower byte
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(q2[hh]) : "f"(x1), "f"(x0));
    }
    packed[p] = static_cast<uint32_t>(q2[0]) | (static_cast<uint32_t>(q2[1]) << 16);
  }
  return make_uint2(packed[0], packed[1]);
}

// The step's writes over an FP8 pool (pkv_decode_step_fp8), made by the one
// warp that later stages sequence b's last page, as fused_step_append does
// for a 16-bit pool: rows 0 .. rows-1 of the copy whose destination is the
// slot's block (codes, copied as bytes), then the new token quantised as
// quant8_e4m3 does.  The caller fences them for the async proxy before
// that page's TMA load.
template <typename T, int D>
__device__ __forceinline__ void fused_step_append_fp8(const DecodeArgs& a, int b, int kvh, int lane, float k_scale,
                                                      float v_scale) {
  constexpr int kRowChunks = D / 16;  // 16-byte chunks of a row of codes
  const int64_t s = a.slots[b];
  const int64_t blk = s >= 0 ? s / kBlockSize : -1;
  const bool ok = s >= 0 && blk < a.num_blocks;
  if (s >= 0 && !ok && lane == 0) raise_error(PKV_ERR_SLOT_RANGE);
  if (!ok) return;
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
  // the token: 8 elements (16 bytes in, 8 codes out) a lane and tensor
  constexpr int kIn = D / 8;
  const size_t row = ((static_cast<size_t>(blk) * a.num_kv_heads + kvh) * kBlockSize + s % kBlockSize) * kIn;
  const size_t in = (static_cast<size_t>(b) * a.num_kv_heads + kvh) * kIn;
  for (int e = lane; e < 2 * kIn; e += 32) {
    const bool is_v = e >= kIn;
    const int c = is_v ? e - kIn : e;
    const uint4 x = reinterpret_cast<const uint4*>(is_v ? a.v_new : a.k_new)[in + c];
    reinterpret_cast<uint2*>(is_v ? vc : kc)[row + c] = quant8_e4m3<T>(x, is_v ? v_scale : k_scale);
  }
}

template <int D, int NWARPS, int NSTAGE>
struct Fp8Shape {
  static constexpr int kTile = kBlockSize * D;  // bytes of a (block, kv-head) tile
  static constexpr int kStage = 2 * kTile;      // K + V
  static constexpr int kChunks = D / 16;        // 16-byte chunks per row
  static constexpr int kWarpStageBytes = NSTAGE * kStage;
  static constexpr size_t kSmemStages = size_t(NWARPS) * kWarpStageBytes;
  static constexpr size_t kSmem = 1024 + kSmemStages + size_t(NWARPS) * NSTAGE * 8;
  static constexpr int kRecM = 8 * D, kRecL = 8 * D + 8;
  static constexpr int kTab = (128 + 32 * NWARPS - 1) / (32 * NWARPS);
  static_assert(D == 64 || D == 128, "a tile row is one swizzle span");
  static_assert(size_t(8) * (D + 2) * sizeof(float) <= size_t(kWarpStageBytes),
                "a warp's merge record must fit in its own stages");
  static_assert(kTile % 512 == 0, "swizzled tiles want 512/1024-byte alignment");
};

// CTAs per SM the FP8 kernel's register budget is sized for
#ifndef PKV_FP8_MIN_CTAS
#define PKV_FP8_MIN_CTAS 8
#endif

// kCascade: the suffix pass of a shared-prefix decode over an FP8 cache
// (pkv_paged_attention_decode_prefix_fp8).  A sequence whose table starts
// with the prefix blocks (and whose context covers them) attends only its
// suffix, partition `part` counted from the prefix's end; any other
// sequence attends its whole context.  Every CTA writes partials (the
// merge kernel combines them with the prefix pass's) and the CTA (kv-head
// 0, part 0) writes the sequence's conformity flag.
template <typename T, int D, int G, int NWARPS, int NSTAGE, bool kCascade = false>
__global__ void __launch_bounds__(NWARPS * 32, PKV_FP8_MIN_CTAS)
    paged_decode_fp8_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v, float v_scale, float k_scale) {
  // The cascade's suffix pass reads nothing the launch before it (the
  // prefix pass) writes: with defer_wait it lets its dependents launch and
  // starts at once, running beside the prefix pass, and waits for that
  // launch only before each CTA exits, so that it still ends after it (the
  // merge after it reads both).  The launches before the prefix pass are
  // complete by then: every prefix CTA waited for them before it let this
  // launch start.
  const bool defer = kCascade && a.defer_wait;
  if (defer)
    pdl_trigger();
  else
    pdl_enter();
  auto exit_wait = [&]() {
    if (defer && threadIdx.x == 0) pdl_wait();
  };
  using S = Fp8Shape<D, NWARPS, NSTAGE>;
  using M = Mma<__half>;      // the MMAs run in fp16 (see above)
  // kPack (G <= 4): the spare query columns [G, 2G) repeat queries [0, G)
  // (identical scores, max and sum), carry P's lo part where columns
  // [0, G) carry its hi part, and the two columns' O^T are added at the
  // end: one P.V MMA per m-tile instead of two.
  constexpr bool kPack = G <= 4;
  // the reference max moves only past 2^kLazyMax (see the softmax below)
  constexpr float kLazyMax = 8.f;
  const int kvh = blockIdx.x;
  const int b = blockIdx.y;
  const int part = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3, lm = lane >> 3, lr = lane & 7;

  int same = 1;
  if constexpr (kCascade)
    for (int j = threadIdx.x; j < a.prefix_pages; j += NWARPS * 32)
      if (a.block_tables[static_cast<long long>(b) * a.bt_stride + j] != a.prefix_blocks[j]) same = 0;
  int ctx = a.context_lens[b];
  if (ctx < 0 || ctx > a.max_ctx) {
    if (threadIdx.x == 0 && kvh == 0 && part == 0) raise_error(PKV_ERR_CONTEXT_RANGE);
    ctx = ctx < 0 ? 0 : a.max_ctx;
  }
  int tok_begin = 0;
  if constexpr (kCascade) {
    const bool conforming = __syncthreads_and(same) && ctx >= a.prefix_pages * kBlockSize;
    if (conforming) tok_begin = a.prefix_pages * kBlockSize;
    if (threadIdx.x == 0 && kvh == 0 && part == 0) a.conform[b] = conforming ? 1 : 0;
  }
  const int span = ctx - tok_begin;
  const int nparts = (span + a.partition - 1) / a.partition;
  if (part >= (nparts > 0 ? nparts : 1)) {
    exit_wait();
    return;
  }
  if (span == 0) {
    if (!kCascade) {  // (the cascade's merge writes the zeros of an empty context)
      T* out = reinterpret_cast<T*>(a.out) + (static_cast<size_t>(b) * a.num_q_heads + kvh * G) * D;
      for (int i = threadIdx.x; i < G * D; i += NWARPS * 32) out[i] = Fmt<T>::from_f32(0.f);
    }
    exit_wait();
    return;
  }
  auto col_row = [&](int n) -> size_t { return static_cast<size_t>(b) * a.num_q_heads + kvh * G + n; };

  extern __shared__ unsigned char smem_raw[];
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

  // Q^T as fp16 B fragments in the d order the converted K fragments use:
  // chunk c: b0 = q[16c + 4t .. +1], b1 = q[16c + 4t + 2 .. +3].  A bf16
  // row is first scaled by 2^kq (exact) so that it fits fp16.
  // With kPack the query columns [G, 2G) repeat queries [0, G).
  uint32_t qb[S::kChunks][2];
  int kq = 0;  // this lane's row (query g8): q was multiplied by 2^kq
  {
    const bool ok = g8 < (kPack ? 2 * G : G);
    const T* qp = reinterpret_cast<const T*>(a.q) + (ok ? col_row(g8 & (G - 1)) : 0) * D;
    float qf[S::kChunks][4];
#pragma unroll
    for (int c = 0; c < S::kChunks; ++c) {
      const float2 lo = ok ? Mma<T>::unpack(*reinterpret_cast<const uint32_t*>(qp + 16 * c + 4 * t4))
                           : make_float2(0.f, 0.f);
      const float2 hi = ok ? Mma<T>::unpack(*reinterpret_cast<const uint32_t*>(qp + 16 * c + 4 * t4 + 2))
                           : make_float2(0.f, 0.f);
      qf[c][0] = lo.x;
      qf[c][1] = lo.y;
      qf[c][2] = hi.x;
      qf[c][3] = hi.y;
    }
    float sc = 1.f;
    if constexpr (!std::is_same<T, __half>::value) {
      float mx = 0.f;
#pragma unroll
      for (int c = 0; c < S::kChunks; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fabsf(qf[c][e]));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
      const int ex = static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu) - 127;  // floor(log2 mx) (normal mx)
      kq = mx > 0.f ? min(max(14 - ex, -126), 126) : 0;
      sc = __uint_as_float(static_cast<uint32_t>(kq + 127) << 23);  // 2^kq
    }
#pragma unroll
    for (int c = 0; c < S::kChunks; ++c) {
      qb[c][0] = M::pack(qf[c][0] * sc, qf[c][1] * sc);
      qb[c][1] = M::pack(qf[c][2] * sc, qf[c][3] * sc);
    }
  }
  // logit scale of this lane's S^T columns 2 t4, 2 t4 + 1 (query rows
  // 2 t4, 2 t4 + 1 held their factor 2^kq in lanes 8 t4, 8 t4 + 4)
  const int kq0 = __shfl_sync(kFull, kq, 8 * t4), kq1 = __shfl_sync(kFull, kq, 8 * t4 + 4);
  const float xs0 = a.qk_scale * __uint_as_float(static_cast<uint32_t>(127 - kq0) << 23);
  const float xs1 = a.qk_scale * __uint_as_float(static_cast<uint32_t>(127 - kq1) << 23);

  const int tok0 = tok_begin + part * a.partition;
  const int tok1 = min(ctx, tok0 + a.partition);
  const int pg0 = tok0 / kBlockSize;
  const int nblk = (tok1 - tok0 + kBlockSize - 1) / kBlockSize;
  const int my_n = warp < nblk ? (nblk - warp + NWARPS - 1) / NWARPS : 0;
  int my_phys[S::kTab];
#pragma unroll
  for (int h = 0; h < S::kTab; ++h) {
    my_phys[h] = -1;
    const int j = lane + 32 * h;
    if (j < my_n) {
      const int e = a.block_tables[static_cast<long long>(b) * a.bt_stride + pg0 + warp + j * NWARPS];
      if (e >= 0 && e < a.num_blocks)
        my_phys[h] = e;
      else
        raise_error(PKV_ERR_BLOCK_RANGE);
    }
  }
  auto phys_of = [&](int i) {
    int r = -1;
#pragma unroll
    for (int h = 0; h < S::kTab; ++h) {
      const int v = __shfl_sync(kFull, my_phys[h], i & 31);
      if ((i >> 5) == h) r = v;
    }
    return r;
  };
  // a fused step (pkv_decode_step_fp8): the warp that stages the sequence's
  // last page (page nblk - 1 of the last partition, its page last_i) makes
  // the step's writes first and fences them before that page's TMA load.
  // In a cascade that is the suffix's last page: the step never writes
  // into the shared prefix blocks, which the prefix pass reads meanwhile.
  int last_i = -1;
  if (a.slots != nullptr && part == nparts - 1 && warp == (nblk - 1) % NWARPS) last_i = (nblk - 1) / NWARPS;
  uint32_t phase_bits = 0;
  auto issue = [&](int i) {
    const int phys = phys_of(i);
    if (i == last_i) {
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
        tma_load_2d(dst, &tmap_k, 0, y, bar);
        tma_load_2d(dst + S::kTile, &tmap_v, 0, y, bar);
      } else {
        mbar_arrive(bar);
      }
    }
  };
  if (last_i >= 0) {
    // the warp's first pages go out before the writes, whose latency
    // overlaps them; the last page waits for them
#pragma unroll
    for (int i = 0; i < NSTAGE; ++i)
      if (i != last_i) issue(i);
    fused_step_append_fp8<T, D>(a, b, kvh, lane, k_scale, v_scale);
    if (last_i < NSTAGE) issue(last_i);
  } else {
#pragma unroll
    for (int i = 0; i < NSTAGE; ++i) issue(i);
  }

  // O^T accumulators: m-tile i, rows g8 / g8 + 8 -> d = 16 i + g8 / + 8,
  // columns 2 t4, 2 t4 + 1 (queries)
  constexpr int kMT = D / 16;
  float o[kMT][4];
#pragma unroll
  for (int i = 0; i < kMT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // query columns 2 t4, 2 t4 + 1
  int consumed = 0;
  bool timed_out = false;

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
    if (phys_of(i) >= 0) {
      const int page_tok = tok0 + (warp + i * NWARPS) * kBlockSize;
      const int nvalid = min(kBlockSize, tok1 - page_tok);
      const uint32_t kt = stage0 + s * S::kStage;
      const uint32_t vt = kt + S::kTile;
      // (1) S^T = K . Q^T, two chunks of d per ldmatrix, into two
      // independent accumulation chains (even and odd chunks)
      float sc[4] = {0.f, 0.f, 0.f, 0.f}, sd[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const int row = lr + ((lm & 1) << 3);
#pragma unroll
        for (int c = 0; c < S::kChunks; c += 2) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kt + swz8<D>(score_row_token(row), c + (lm >> 1)), r0, r1, r2, r3);
          uint32_t f0, f1, f2, f3, f4, f5, f6, f7;
          e4m3x4_to_f16(r0, f0, f2);
          e4m3x4_to_f16(r1, f1, f3);
          e4m3x4_to_f16(r2, f4, f6);
          e4m3x4_to_f16(r3, f5, f7);
          M::run(sc, f0, f1, f2, f3, qb[c][0], qb[c][1]);
          M::run(sd, f4, f5, f6, f7, qb[c + 1][0], qb[c + 1][1]);
        }
      }
      // (2) scale (K scale folded in), mask the tail, online softmax
      const bool v_lo = score_row_token(g8) < nvalid, v_hi = score_row_token(g8 + 8) < nvalid;
      const float x0 = v_lo ? (sc[0] + sd[0]) * xs0 : -INFINITY;
      const float x1 = v_lo ? (sc[1] + sd[1]) * xs1 : -INFINITY;
      const float x2 = v_hi ? (sc[2] + sd[2]) * xs0 : -INFINITY;
      const float x3 = v_hi ? (sc[3] + sd[3]) * xs1 : -INFINITY;
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
      // The reference max m of a column moves only when one of the page's
      // scores passes it by more than kLazyMax (so p <= 2^kLazyMax): most
      // pages then need one vote, no reduction and no rescale.  Any
      // reference is exact once the same m scales l and O.
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
        // this lane's O^T columns are its own query columns 2 t4, 2 t4 + 1
#pragma unroll
        for (int i = 0; i < kMT; ++i) {
          o[i][0] *= al0;
          o[i][1] *= al1;
          o[i][2] *= al0;
          o[i][3] *= al1;
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
      // (4) V^T fragments straight from the tile: the transposed byte load
      // gives lane (g8, t4) the codes of tokens 4 t4 .. 4 t4 + 3 at d =
      // 16 i + g8 and 16 i + g8 + 8 of m-tiles i and i + 1; each pair of
      // codes converts exactly into one 16-bit A register.  Tokens past the
      // context are zeroed (an unused slot may hold a NaN code).
      uint32_t keep = 0xffffffffu;
      if (nvalid < kBlockSize) {
        const int n = nvalid - 4 * t4;
        keep = n >= 4 ? 0xffffffffu : n <= 0 ? 0u : 0xffffffffu >> (32 - 8 * n);
      }
#pragma unroll
      for (int i = 0; i < kMT; i += 2) {
        uint32_t w0, w1, w2, w3;
        ldsm_b8_x2_t(vt + swz8<D>(lane & 15, i + (lane >> 4)), w0, w1, w2, w3);
        uint32_t a0, a1, a2, a3;
        e4m3x4_to_f16(w0 & keep, a0, a2);  // tokens 4 t4, +1 | 4 t4 + 2, +3 at row g8
        e4m3x4_to_f16(w1 & keep, a1, a3);  // the same at row g8 + 8
        if constexpr (!kPack) M::run(o[i], a0, a1, a2, a3, pb0, pb1);
        M::run(o[i], a0, a1, a2, a3, pl0, pl1);
        e4m3x4_to_f16(w2 & keep, a0, a2);
        e4m3x4_to_f16(w3 & keep, a1, a3);
        if constexpr (!kPack) M::run(o[i + 1], a0, a1, a2, a3, pb0, pb1);
        M::run(o[i + 1], a0, a1, a2, a3, pl0, pl1);
      }
    }
    __syncwarp();
    issue(i + NSTAGE);
  }
  if (consumed < my_n) {
    const int last = min(my_n, consumed + NSTAGE);
    for (int i = consumed; i < last; ++i) {
      const int s = i % NSTAGE;
      mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
      phase_bits ^= 1u << s;
    }
  }
#pragma unroll
  for (int msk = 4; msk <= 16; msk <<= 1) {
    l0 += __shfl_xor_sync(kFull, l0, msk);
    l1 += __shfl_xor_sync(kFull, l1, msk);
  }

  if constexpr (kPack) {  // query n: column n (hi) + column n + G (lo)
#pragma unroll
    for (int i = 0; i < kMT; ++i) {
      if constexpr (G == 1) {
        o[i][0] += o[i][1];
        o[i][2] += o[i][3];
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) o[i][e] += __shfl_xor_sync(kFull, o[i][e], G / 2);
      }
    }
  }
  // warp record [o: 8 x D][m: 8][l: 8]
  float* rec = reinterpret_cast<float*>(my_stages);
#pragma unroll
  for (int i = 0; i < kMT; ++i) {
    const int d = 16 * i + g8;
    if (2 * t4 < G) {
      rec[(2 * t4) * D + d] = o[i][0];
      rec[(2 * t4) * D + d + 8] = o[i][2];
    }
    if (2 * t4 + 1 < G) {
      rec[(2 * t4 + 1) * D + d] = o[i][1];
      rec[(2 * t4 + 1) * D + d + 8] = o[i][3];
    }
  }
  if (g8 == 0) {
    if (2 * t4 < G) {
      rec[S::kRecM + 2 * t4] = m0;
      rec[S::kRecL + 2 * t4] = l0;
    }
    if (2 * t4 + 1 < G) {
      rec[S::kRecM + 2 * t4 + 1] = m1;
      rec[S::kRecL + 2 * t4 + 1] = l1;
    }
  }
  if (__syncthreads_or(timed_out)) {
    exit_wait();
    return;
  }

  for (int idx = threadIdx.x; idx < G * D; idx += NWARPS * 32) {
    const int g = idx / D, d = idx % D;
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
    num *= v_scale;
    const size_t row = col_row(g);
    if (nparts == 1 && !kCascade) {
      reinterpret_cast<T*>(a.out)[row * D + d] = Fmt<T>::from_f32(num / den);
    } else {
      const size_t wrow = row * a.num_parts + part;
      a.ws_o[wrow * D + d] = num;
      if (d == 0) a.ws_ml[wrow] = make_float2(Mx, den);
    }
  }
  exit_wait();
}

// The shared prefix of an FP8 cache as exact 16-bit code values, for the
// cascade's prefix pass (which runs on the 16-bit tensor-core path): tile
// (page p, kv-head h) of prefix block prefix_blocks[p] goes to block p of a
// small pool [prefix_pages][Hkv][16][D] of T (every E4M3 value is an fp16
// and a bf16 value, so nothing is rounded; the scales are applied by the
// pass).  One thread converts 8 codes; chunks [0, total) are K, [total,
// 2 total) V.  A prefix entry outside the pool is flagged and its tile
// zeroed.
template <typename T>
__global__ void __launch_bounds__(256)
    dequant_prefix_kernel(const uint2* __restrict__ k_cache, const uint2* __restrict__ v_cache,
                          uint4* __restrict__ k_out, uint4* __restrict__ v_out, const int32_t* __restrict__ prefix_blocks,
                          long long total, int Hkv, int row_chunks, int num_blocks) {
  pdl_enter();
  const long long tile_chunks = static_cast<long long>(kBlockSize) * row_chunks;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < 2 * total; i += stride) {
    const bool is_v = i >= total;
    const long long j = is_v ? i - total : i;
    const long long tile = j / tile_chunks;  // p * Hkv + h
    const long long c = j - tile * tile_chunks;
    const int p = static_cast<int>(tile / Hkv), h = static_cast<int>(tile % Hkv);
    const int blk = prefix_blocks[p];
    uint4 o = make_uint4(0u, 0u, 0u, 0u);
    if (blk >= 0 && blk < num_blocks) {
      const uint2 w = (is_v ? v_cache : k_cache)[(static_cast<long long>(blk) * Hkv + h) * tile_chunks + c];
      uint32_t h2[4];
      e4m3x4_to_f16(w.x, h2[0], h2[1]);
      e4m3x4_to_f16(w.y, h2[2], h2[3]);
      if constexpr (!std::is_same<T, __half>::value) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2[e]));
          h2[e] = Mma<T>::pack(f.x, f.y);  // exact: an E4M3 value is a bf16 value
        }
      }
      o = make_uint4(h2[0], h2[1], h2[2], h2[3]);
    } else if (h == 0 && c == 0 && !is_v) {
      raise_error(PKV_ERR_BLOCK_RANGE);
    }
    (is_v ? v_out : k_out)[j] = o;
  }
}

// Slot-mapped append into an FP8 cache: code = E4M3(x / scale) (x fp16 or
// bf16, the division in float32, round to nearest even, saturating at
// +-448).  One thread converts 8 elements (16 bytes in, 8 bytes out).
// Chunks [0, total) are K, [total, 2 total) V; total = tokens * Hkv * D / 8.
template <typename T>
__global__ void __launch_bounds__(256)
    kv_append_fp8_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                         uint2* __restrict__ k_cache, uint2* __restrict__ v_cache, const int64_t* __restrict__ slots,
                         long long total, int Hkv, int row_chunks, int num_blocks, float k_scale, float v_scale) {
  pdl_enter();
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < 2 * total; i += stride) {
    const bool is_v = i >= total;
    const long long j = is_v ? i - total : i;
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
    const uint4 in = (is_v ? v_new : k_new)[j];
    const long long dst = ((blk * Hkv + h) * kBlockSize + off) * row_chunks + c;
    (is_v ? v_cache : k_cache)[dst] = quant8_e4m3<T>(in, is_v ? v_scale : k_scale);
  }
}

}  // namespace pkv
