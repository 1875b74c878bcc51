// Paged decode attention: partition kernel + log-sum-exp merge kernel.
//
// What is computed ("PagedAttention 与 vLLM 推理加速" §2.3 and §1): for
// sequence b, query head h, kv-head g = h / G, the query attends over the
// n = context_lens[b] keys/values K_j = cache[table[b][j/16], g, j%16, :],
// out = softmax(scale * q.K) V.  The exponentials are taken base 2 on
// logits pre-multiplied by log2(e), which is the same softmax.
//
// How (B200 design):
//  * One CTA per (kv-head, sequence, partition of `partition` tokens).  All
//    G = Hq/Hkv query heads of the kv-head are served by the same CTA, so
//    every K/V tile is read from HBM once per kv-head (GQA packing).
//  * A (block, kv-head) tile is 16 * D contiguous elements in the pool
//    layout [num_blocks, Hkv, 16, D]; K and V tiles are staged into shared
//    memory with 1-D bulk async copies (cp.async.bulk, no tensor map
//    needed), completing on an mbarrier.  Each warp owns NSTAGE stages
//    and walks pages warp, warp + NWARPS, ... of the partition, so every
//    warp keeps NSTAGE tiles in flight without any CTA-wide barrier in the
//    loop.  The block table drives the copies: lane j of a warp holds the
//    physical block of the warp's j-th page.
//  * Q.K: lane (c, r0) owns 16-byte chunk c of rows r0, r0 + RPI, ... of
//    the tile, reads it with one 16-byte shared load (a warp reads whole
//    rows: conflict-free), and forms partial dot products against all G
//    queries held in registers; a transposing butterfly (each shuffle
//    carries half of the remaining partials) finishes the dot products.
//  * Online softmax per warp in fp32 (running max, running sum, rescaled
//    accumulator), then P.V with the same lane layout.
//  * The warps' states are merged in shared memory in a fixed order; a
//    one-partition sequence writes its normalised output directly, a longer
//    one writes (max, sum, partial output) to the workspace and the merge
//    kernel rescales the partitions to their common max.
//  The order of every sum depends only on logical token positions, so the
//  result is bit-identical under any relabelling of physical blocks.
#pragma once

#include <math.h>

#include "common.cuh"

namespace pkv {

struct DecodeArgs {
  void* out;
  const void* q;
  const unsigned char* k_cache;
  const unsigned char* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_o;        // [B][Hq][P][D] partial outputs (unnormalised)
  float2* ws_ml;      // [B][Hq][P] (running max in log2 units, running sum)
  long long bt_stride;  // max_blocks_per_seq
  int max_ctx;        // min(max_context_len, 16 * max_blocks_per_seq)
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int num_blocks;
  int partition;      // tokens per partition, multiple of 16
  int num_parts;      // P = ceil(max_context_len / partition), >= 1
  float qk_scale;     // scale * log2(e)
  // shared-prefix (cascade) mode; prefix_blocks == nullptr otherwise
  const int32_t* prefix_blocks;  // [prefix_pages] blocks every sequence is expected to start with
  int prefix_pages;
  int chunk_pages;     // prefix pages per prefix-pass CTA
  int num_chunks;      // ceil(prefix_pages / chunk_pages)
  int num_qgroups;     // prefix-role CTAs per (kv-head, chunk): ceil(B * G / 8)
  int suffix_z;        // partitions in flight per sequence (suffix-role CTAs per sequence)
  float* wp_o;         // [B][Hq][num_chunks][D] prefix partial outputs
  float2* wp_ml;       // [B][Hq][num_chunks] (max, sum)
  int* conform;        // [B]: 1 when sequence b starts with the prefix
  int y_offset;        // cascade launched in parts: blockIdx.y + y_offset is the role index
  int prefix_ident;    // prefix page i is block i of the pool given (a dequantised copy of the prefix)
  float prefix_out_scale;  // factor on the prefix partial outputs (the V scale of an FP8 cache; else 1)
  // a decode step fused with its append (pkv_decode_step); slots == nullptr
  // otherwise.  One new token per sequence: the CTA that reads sequence b's
  // last page writes k_new[b] / v_new[b] into slot slots[b] (after the
  // copy-on-write copy whose destination is that slot's block) before it
  // stages anything.
  const unsigned char* k_new;  // [B][Hkv][D]
  const unsigned char* v_new;
  const int64_t* slots;        // [B]
  const int32_t* copies;       // [n_copies][3] = (src, dst, rows)
  int n_copies;
  // the preceding launch is this step's copy-on-write copies and append
  // (they write only the sequences' last pages): the decode starts without
  // waiting for it, and only the warp that stages a sequence's last page
  // waits (griddepcontrol.wait) before that page's copy
  int defer_wait;
};

constexpr unsigned kFull = 0xffffffffu;

template <typename T, int D, int G, int NWARPS, int NSTAGE>
struct DecodeShape {
  static constexpr int kEs = sizeof(T);
  static constexpr int kVec = Fmt<T>::kVec;           // elements per 16-byte chunk
  static constexpr int kCpr = D / kVec;               // chunks per row = lanes per row
  static constexpr int kRpi = 32 / kCpr;              // rows per warp iteration
  static constexpr int kIters = kBlockSize / kRpi;    // iterations per tile
  static constexpr int kRowBytes = D * kEs;
  static constexpr int kTile = kBlockSize * kRowBytes;  // one (block, kv-head) tile
  static constexpr int kStage = 2 * kTile;            // K tile + V tile
  static constexpr int kNval = kIters * G;            // partial dot products per lane
  static constexpr int kNpl = kNval >= kCpr ? kNval / kCpr : 1;  // finished dots per lane
  static constexpr int kDup = kNval >= kCpr ? 1 : kCpr / kNval;  // lanes sharing one
  static constexpr int kPairs = (kBlockSize * G + 31) / 32;      // softmax (row, head) per lane
  static constexpr int kWarpStageBytes = NSTAGE * kStage;
  static constexpr size_t kSmemStages = size_t(NWARPS) * kWarpStageBytes;
  static constexpr size_t kSmemBars = size_t(NWARPS) * NSTAGE * 8;
  static constexpr size_t kSmemP = size_t(NWARPS) * kBlockSize * G * sizeof(float);
  static constexpr size_t kSmem = kSmemStages + kSmemBars + kSmemP;
  static_assert(kCpr <= 32 && 32 % kCpr == 0, "a row must split evenly over the warp");
  static_assert(32 % G == 0 && G <= 16, "G must divide 32");
  static_assert(size_t(G) * (D + 2) * sizeof(float) <= size_t(kWarpStageBytes),
                "a warp's merge record must fit in its own stages");
  static_assert((kNval & (kNval - 1)) == 0, "butterfly needs a power of two");
  static_assert(kSmemBars % 16 == 0, "keep the probability scratch 16-byte aligned");
};

// Sum N values across the lanes of a row group (lane bits below 2*MASK) with
// a transposing butterfly: each step a lane keeps one half of its values
// and adds its partner's copy of that half, so N values need N-1 shuffles
// instead of N*log2(lanes).  Afterwards lane c of the group holds the sums
// with indices c * N/lanes ... (c+1) * N/lanes - 1 (or, when N < lanes,
// index c / (lanes/N), shared by lanes/N neighbours).
template <int N, int MASK>
struct XReduce {
  __device__ __forceinline__ static void run(float* v, int lane) {
    if constexpr (MASK == 0) {
      return;
    } else if constexpr (N == 1) {
      v[0] += __shfl_xor_sync(kFull, v[0], MASK);
      XReduce<1, MASK / 2>::run(v, lane);
    } else {
      constexpr int H = N / 2;
      const bool upper = (lane & MASK) != 0;
#pragma unroll
      for (int i = 0; i < H; ++i) {
        const float send = upper ? v[i] : v[i + H];
        const float keep = upper ? v[i + H] : v[i];
        v[i] = keep + __shfl_xor_sync(kFull, send, MASK);
      }
      XReduce<H, MASK / 2>::run(v, lane);
    }
  }
};

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <int G>
__device__ __forceinline__ void load_probs(const float* p, float (&out)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int g = 0; g < G; g += 4) {
      const float4 t = *reinterpret_cast<const float4*>(p + g);
      out[g] = t.x;
      out[g + 1] = t.y;
      out[g + 2] = t.z;
      out[g + 3] = t.w;
    }
  } else if constexpr (G == 2) {
    const float2 t = *reinterpret_cast<const float2*>(p);
    out[0] = t.x;
    out[1] = t.y;
  } else {
    out[0] = p[0];
  }
}

template <typename T, int D, int G, int NWARPS, int NSTAGE>
__global__ void __launch_bounds__(NWARPS * 32)
    paged_decode_partition_kernel(const DecodeArgs a) {
  pdl_enter();
  using S = DecodeShape<T, D, G, NWARPS, NSTAGE>;
  const int kvh = blockIdx.x;
  const int b = blockIdx.y;
  const int part = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int ctx = a.context_lens[b];
  if (ctx < 0 || ctx > a.max_ctx) {
    if (threadIdx.x == 0 && kvh == 0 && part == 0) raise_error(PKV_ERR_CONTEXT_RANGE);
    ctx = ctx < 0 ? 0 : a.max_ctx;
  }
  const int nparts = (ctx + a.partition - 1) / a.partition;
  if (part >= (nparts > 0 ? nparts : 1)) return;

  const int h0 = kvh * G;
  T* out = reinterpret_cast<T*>(a.out) + (static_cast<size_t>(b) * a.num_q_heads + h0) * D;
  if (ctx == 0) {
    for (int i = threadIdx.x; i < G * D; i += NWARPS * 32) out[i] = Fmt<T>::from_f32(0.f);
    return;
  }

  const int tok0 = part * a.partition;
  const int tok1 = min(ctx, tok0 + a.partition);
  const int pg0 = tok0 / kBlockSize;
  const int nblk = (tok1 - tok0 + kBlockSize - 1) / kBlockSize;
  const int my_n = warp < nblk ? (nblk - warp + NWARPS - 1) / NWARPS : 0;

  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* my_stages = smem + static_cast<size_t>(warp) * S::kWarpStageBytes;
  const uint32_t stage0 = smem_addr(my_stages);
  const uint32_t bar0 = smem_addr(smem + S::kSmemStages) + warp * NSTAGE * 8;
  float* psm = reinterpret_cast<float*>(smem + S::kSmemStages + S::kSmemBars) + warp * kBlockSize * G;

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

  const size_t head_off = static_cast<size_t>(kvh) * S::kTile;
  const size_t blk_stride = static_cast<size_t>(a.num_kv_heads) * S::kTile;
  // Stage page i of this warp into stage i % NSTAGE.  An out-of-range page
  // still completes its barrier phase (plain arrive) so phases stay in step.
  auto issue = [&](int i) {
    const int phys = __shfl_sync(kFull, my_phys, i & 31);
    if (lane == 0 && i < my_n) {
      const uint32_t bar = bar0 + 8 * (i % NSTAGE);
      if (phys >= 0) {
        const uint32_t dst = stage0 + (i % NSTAGE) * S::kStage;
        const size_t off = static_cast<size_t>(phys) * blk_stride + head_off;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, S::kStage);
        bulk_g2s(dst, a.k_cache + off, S::kTile, bar);
        bulk_g2s(dst + S::kTile, a.v_cache + off, S::kTile, bar);
      } else {
        mbar_arrive(bar);
      }
    }
  };
#pragma unroll
  for (int i = 0; i < NSTAGE; ++i) issue(i);

  // this lane's slice of every query of the group, pre-scaled
  const int c = lane % S::kCpr;
  const int r0 = lane / S::kCpr;
  float qv[G][S::kVec];
  {
    const T* qp = reinterpret_cast<const T*>(a.q) + (static_cast<size_t>(b) * a.num_q_heads + h0) * D;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float t[S::kVec];
      Fmt<T>::to_f32(*reinterpret_cast<const uint4*>(qp + g * D + c * S::kVec), t);
#pragma unroll
      for (int e = 0; e < S::kVec; ++e) qv[g][e] = t[e] * a.qk_scale;
    }
  }

  float o[G][S::kVec];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < S::kVec; ++e) o[g][e] = 0.f;
  float m_mine = -INFINITY;  // running max of head lane % G (log2 units)
  float l_mine = 0.f;        // this lane's share of that head's running sum
  uint32_t phase_bits = 0;   // barrier phase parity per stage
  int consumed = 0;

  for (int i = 0; i < my_n; ++i) {
    const int s = i % NSTAGE;
    bool ok = mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
    ok = __all_sync(kFull, ok);
    if (!ok) {
      if (lane == 0) raise_error(PKV_ERR_TIMEOUT);
      break;
    }
    phase_bits ^= 1u << s;  // (a stage that timed out keeps its parity: the drain waits on it again)
    consumed = i + 1;
    const int phys = __shfl_sync(kFull, my_phys, i);
    if (phys >= 0) {
      const int page_tok = tok0 + (warp + i * NWARPS) * kBlockSize;
      const int nvalid = min(kBlockSize, tok1 - page_tok);
      // staged tiles (written by the bulk copies, visible after the wait)
      const unsigned char* kt = my_stages + s * S::kStage;
      const unsigned char* vt = kt + S::kTile;

      // (1) partial dot products of this lane's chunk with every query
      float acc[S::kNval];
#pragma unroll
      for (int it = 0; it < S::kIters; ++it) {
        const int r = it * S::kRpi + r0;
        float kf[S::kVec];
        Fmt<T>::to_f32(*reinterpret_cast<const uint4*>(kt + r * S::kRowBytes + c * 16), kf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < S::kVec; ++e) d = fmaf(qv[g][e], kf[e], d);
          acc[it * G + g] = d;
        }
      }
      // (2) finish the dot products across the row's lanes
      XReduce<S::kNval, S::kCpr / 2>::run(acc, lane);
      // (3) logits to shared memory as [row][head]
      if (S::kDup == 1 || (c % S::kDup) == 0) {
#pragma unroll
        for (int j = 0; j < S::kNpl; ++j) {
          const int idx = (S::kNval >= S::kCpr) ? c * S::kNpl + j : c / S::kDup;
          const int it = idx / G;
          const int g = idx % G;
          psm[(it * S::kRpi + r0) * G + g] = acc[j];
        }
      }
      __syncwarp();
      // (4) online softmax: lane handles (row, head) pairs k = lane + 32 j,
      // all of head lane % G
      float sv[S::kPairs];
      float bmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < S::kPairs; ++j) {
        const int k = lane + 32 * j;
        float x = -INFINITY;
        if (k < kBlockSize * G && k / G < nvalid) x = psm[k];
        sv[j] = x;
        bmax = fmaxf(bmax, x);
      }
#pragma unroll
      for (int m = 16; m >= G; m >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, m));
      const float m_new = fmaxf(m_mine, bmax);
      const float alpha_mine = exp2f(m_mine - m_new);
      float psum = 0.f;
#pragma unroll
      for (int j = 0; j < S::kPairs; ++j) {
        const int k = lane + 32 * j;
        const float p = exp2f(sv[j] - m_new);
        psum += p;
        if (k < kBlockSize * G) psm[k] = p;
      }
      l_mine = fmaf(l_mine, alpha_mine, psum);
      m_mine = m_new;
      __syncwarp();
      // (5) rescale the accumulator, then accumulate P.V
      float alpha[G];
#pragma unroll
      for (int g = 0; g < G; ++g) alpha[g] = __shfl_sync(kFull, alpha_mine, g);
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < S::kVec; ++e) o[g][e] *= alpha[g];
#pragma unroll
      for (int it = 0; it < S::kIters; ++it) {
        const int r = it * S::kRpi + r0;
        if (r < nvalid) {
          float vf[S::kVec];
          Fmt<T>::to_f32(*reinterpret_cast<const uint4*>(vt + r * S::kRowBytes + c * 16), vf);
          float p[G];
          load_probs<G>(psm + r * G, p);
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < S::kVec; ++e) o[g][e] = fmaf(p[g], vf[e], o[g][e]);
        }
      }
    }
    __syncwarp();
    issue(i + NSTAGE);
  }

  // after a give-up, wait (bounded) for the copies this warp still has in
  // flight before its shared memory is reused
  if (consumed < my_n) {
    const int last = min(my_n, consumed + NSTAGE);
    for (int i = consumed; i < last; ++i) {
      const int s = i % NSTAGE;
      mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
      phase_bits ^= 1u << s;
    }
  }

  // finish this warp's state: sum the accumulator over its row groups and
  // the running sums over the lanes of each head
#pragma unroll
  for (int m = S::kCpr; m < 32; m <<= 1)
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < S::kVec; ++e) o[g][e] += __shfl_xor_sync(kFull, o[g][e], m);
#pragma unroll
  for (int m = G; m < 32; m <<= 1) l_mine += __shfl_xor_sync(kFull, l_mine, m);

  // warp record [o: G x D][m: G][l: G] in the warp's own (drained) stages
  float* rec = reinterpret_cast<float*>(my_stages);
  if (r0 == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < S::kVec; e += 4)
        *reinterpret_cast<float4*>(rec + g * D + c * S::kVec + e) =
            make_float4(o[g][e], o[g][e + 1], o[g][e + 2], o[g][e + 3]);
  }
  if (lane < G) {
    rec[G * D + lane] = m_mine;
    rec[G * D + G + lane] = l_mine;
  }
  __syncthreads();

  // merge the warps in a fixed order
  for (int idx = threadIdx.x; idx < G * D; idx += NWARPS * 32) {
    const int g = idx / D;
    const int d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w)
      M = fmaxf(M, reinterpret_cast<const float*>(smem + w * S::kWarpStageBytes)[G * D + g]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) {
      const float* r = reinterpret_cast<const float*>(smem + w * S::kWarpStageBytes);
      const float sc = exp2f(r[G * D + g] - M);
      num = fmaf(sc, r[g * D + d], num);
      den = fmaf(sc, r[G * D + G + g], den);
    }
    if (nparts == 1) {
      out[idx] = Fmt<T>::from_f32(num / den);
    } else {
      const size_t row = (static_cast<size_t>(b) * a.num_q_heads + h0 + g) * a.num_parts + part;
      a.ws_o[row * D + d] = num;
      if (d == 0) a.ws_ml[row] = make_float2(M, den);
    }
  }
}

// Merge n partial results (running max m_p in log2 units, running sum l_p,
// unnormalised output o_p) of one (sequence, query head):
//   out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p,   M = max_p m_p.
// A CTA of kMergeWarps warps serves HPC heads with WPH = kMergeWarps / HPC
// warps each (many warps per head when a head has many partials, one when
// it has few).  Warp w of a head accumulates partials w, w + WPH, ... in
// order (independent loads, unrolled); the warps' sums are then added in a
// fixed order.  `ml(p)` / `op(p)` give partial p's (m, l) and output row.
constexpr int kMergeWarps = 8;

template <typename T, int D, int HPC, typename ML, typename OP>
__device__ __forceinline__ void merge_partials(int n, ML ml, OP op, T* out, int hs /* head slot in the CTA */) {
  constexpr int kEpl = D / 32;
  constexpr int WPH = kMergeWarps / HPC;
  static_assert(kMergeWarps % HPC == 0, "heads per CTA must divide the warps");
  __shared__ float red_o[kMergeWarps][D];
  __shared__ float red_den[kMergeWarps];
  __shared__ float red_max[kMergeWarps];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wi = warp % WPH;  // warp within the head
  const int w0 = hs * WPH;    // first warp of the head
  float M = -INFINITY;
  for (int p = wi * 32 + lane; p < n; p += WPH * 32) M = fmaxf(M, ml(p).x);
  M = warp_max(M);
  if (lane == 0) red_max[warp] = M;
  __syncthreads();
  M = red_max[w0];
#pragma unroll
  for (int w = 1; w < WPH; ++w) M = fmaxf(M, red_max[w0 + w]);

  float acc[kEpl];
#pragma unroll
  for (int e = 0; e < kEpl; ++e) acc[e] = 0.f;
  float den = 0.f;
#pragma unroll 4
  for (int p = wi; p < n; p += WPH) {
    const float2 v = ml(p);
    const float w = exp2f(v.x - M);
    den = fmaf(w, v.y, den);
    const float* o = op(p) + lane * kEpl;
#pragma unroll
    for (int e = 0; e < kEpl; ++e) acc[e] = fmaf(w, o[e], acc[e]);
  }
  if constexpr (WPH == 1) {
    if (n > 0) {
#pragma unroll
      for (int e = 0; e < kEpl; ++e) out[lane * kEpl + e] = Fmt<T>::from_f32(acc[e] / den);
    } else {
#pragma unroll
      for (int e = 0; e < kEpl; ++e) out[lane * kEpl + e] = Fmt<T>::from_f32(0.f);
    }
  } else {
#pragma unroll
    for (int e = 0; e < kEpl; ++e) red_o[warp][lane * kEpl + e] = acc[e];
    if (lane == 0) red_den[warp] = den;
    __syncthreads();
    for (int d = wi * 32 + lane; d < D; d += WPH * 32) {
      float num = 0.f, dd = 0.f;
#pragma unroll
      for (int w = 0; w < WPH; ++w) {
        num += red_o[w0 + w][d];
        dd += red_den[w0 + w];
      }
      out[d] = Fmt<T>::from_f32(n > 0 ? num / dd : 0.f);
    }
  }
}

// Split-K merge: per (query head, sequence b = blockIdx.y) whose context
// spans more than one partition, the partitions in order.  Head of this
// warp: blockIdx.x * HPC + warp / (kMergeWarps / HPC).
template <typename T, int D, int HPC>
__global__ void __launch_bounds__(kMergeWarps * 32) paged_decode_reduce_kernel(const DecodeArgs a) {
  pdl_enter();
  const int hs = (threadIdx.x >> 5) / (kMergeWarps / HPC);
  const int h = blockIdx.x * HPC + hs;
  const int b = blockIdx.y;
  int ctx = a.context_lens[b];
  ctx = ctx < 0 ? 0 : (ctx > a.max_ctx ? a.max_ctx : ctx);
  const int nparts = (ctx + a.partition - 1) / a.partition;
  // one partition: written by the partition kernel; a head past Hq: nothing
  // (the CTA-wide barriers below still need every warp, so no early exit)
  const bool skip = nparts <= 1 || h >= a.num_q_heads;
  const int hh = h < a.num_q_heads ? h : 0;
  const size_t row0 = (static_cast<size_t>(b) * a.num_q_heads + hh) * a.num_parts;
  if (__syncthreads_and(skip)) return;
  T* out = reinterpret_cast<T*>(a.out) + (static_cast<size_t>(b) * a.num_q_heads + hh) * D;
  __shared__ T sink[D];  // output of a skipped head slot (discarded)
  merge_partials<T, D, HPC>(
      skip ? 0 : nparts, [&](int p) { return a.ws_ml[row0 + p]; }, [&](int p) { return a.ws_o + (row0 + p) * D; },
      skip ? sink : out, hs);
}

}  // namespace pkv
