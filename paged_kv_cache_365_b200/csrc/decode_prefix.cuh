// Shared-prefix (cascade) decode: the prefix pass and the merge.
//
// "PagedAttention 与 vLLM 推理加速" §3.2(3): requests with the same system
// prompt map the same physical blocks (stored once).  When every sequence of
// a batch starts with the same prefix blocks, the prefix pass reads each of
// those (block, kv-head) tiles from HBM once and attends the queries of ALL
// sequences of that kv-head to it; the paged kernel then covers each
// sequence's own suffix (decode_mma.cuh, cascade mode), and the merge kernel
// combines the prefix and suffix partial results with the same log-sum-exp
// rule as the split-K merge.  The result is the same attention (up to
// rounding); only the order of the work changes.
//
// Prefix pass, one CTA per (kv-head, chunk of prefix pages, group of
// 16 * NW queries): the queries of the kv-head (sequence b, group head g ->
// query b * G + g) are the M dimension of mma.sync m16n8k16, the 16 tokens
// of a page are N, D is K:
//   S[16 q x 16 tok] = Q[16 x D] . K^T      (A = Q in registers, B = K via ldmatrix)
//   O[16 q x D]     += P[16 x 16] . V       (A = P straight from the S fragments,
//                                            B = V via ldmatrix.trans; hi + lo P)
// One warp per 16 queries; every warp consumes every staged page (a CTA-wide
// ring filled by tensor-map TMA, released through an mbarrier counted by the
// warps).  All prefix tokens are full pages, so no tail masking is needed.
#pragma once

#include "decode_mma.cuh"

namespace pkv {

template <typename T, int D, int NW, int NSTAGE>
struct PrefixShape {
  static constexpr int kTile = kBlockSize * D * 2;
  static constexpr int kStage = 2 * kTile;
  static constexpr int kBoxes = D / 64;
  static constexpr int kKSteps = D / 16;  // QK k-steps
  static constexpr int kNTiles = D / 8;   // PV n-tiles (8 columns of D each)
  static constexpr size_t kSmemStages = size_t(NSTAGE) * kStage;
  static constexpr size_t kSmem = 1024 + kSmemStages + 2 * NSTAGE * 8;
  static_assert(kStage % 1024 == 0, "swizzled boxes need 1024-byte alignment");
};

template <typename T, int D, int G, int NW, int NSTAGE>
__global__ void __launch_bounds__(NW * 32)
    paged_decode_prefix_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                               const __grid_constant__ CUtensorMap tmap_v) {
  using S = PrefixShape<T, D, NW, NSTAGE>;
  using M = Mma<T>;
  const int kvh = blockIdx.x;
  const int chunk = blockIdx.y;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g8 = lane >> 2;
  const int t4 = lane & 3;
  const int lm = lane >> 3;
  const int lr = lane & 7;
  const int nq = a.num_seqs * G;  // queries of this kv-head
  const int q0 = (blockIdx.z * NW + warp) * 16;

  const int p_begin = chunk * a.chunk_pages;
  const int p_end = min(a.prefix_pages, p_begin + a.chunk_pages);
  const int npages = p_end - p_begin;

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  unsigned char* smem = smem_raw + pad;
  const uint32_t stage0 = smem_addr(smem);
  const uint32_t full0 = smem_addr(smem + S::kSmemStages);
  const uint32_t empty0 = full0 + 8 * NSTAGE;

  __shared__ int skip_page[NSTAGE];  // stage holds no data (out-of-range block id)
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, NW);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // bounded wait that also gives up once another warp gave up
  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
      if (abort_flag) return false;
      if (clock64() - t0 > (1ll << 32)) {
        abort_flag = 1;
        raise_error(PKV_ERR_TIMEOUT);
        return false;
      }
    }
    return true;
  };

  // Thread 0 stages page i once every warp has released the stage's
  // previous page.  An out-of-range block id is flagged, its stage marked
  // empty and completed without data.
  auto issue = [&](int i) -> bool {
    const int s = i % NSTAGE;
    if (i >= NSTAGE && !wait(empty0 + 8 * s, ((i / NSTAGE) - 1) & 1)) return false;
    const int phys = a.prefix_blocks[p_begin + i];
    const uint32_t bar = full0 + 8 * s;
    const bool valid = phys >= 0 && phys < a.num_blocks;
    skip_page[s] = valid ? 0 : 1;
    if (valid) {
      const uint32_t dst = stage0 + s * S::kStage;
      const int y = (phys * a.num_kv_heads + kvh) * kBlockSize;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(bar, S::kStage);
#pragma unroll
      for (int bx = 0; bx < S::kBoxes; ++bx) {
        tma_load_2d(dst + bx * 2048, &tmap_k, bx * 64, y, bar);
        tma_load_2d(dst + S::kTile + bx * 2048, &tmap_v, bx * 64, y, bar);
      }
    } else {
      raise_error(PKV_ERR_BLOCK_RANGE);
      mbar_arrive(bar);
    }
    return true;
  };
  int issued = 0;  // pages staged so far (thread 0)
  if (threadIdx.x == 0)
    for (int i = 0; i < NSTAGE && i < npages; ++i) issued += issue(i) ? 1 : 0;

  // A fragments of this warp's 16 queries (rows past the batch are zero)
  uint32_t qa[S::kKSteps][4];
  {
    const int qa_row = q0 + g8, qb_row = q0 + g8 + 8;
    const T* pa = qa_row < nq ? reinterpret_cast<const T*>(a.q) +
                                    (static_cast<size_t>(qa_row / G) * a.num_q_heads + kvh * G + qa_row % G) * D
                              : nullptr;
    const T* pb = qb_row < nq ? reinterpret_cast<const T*>(a.q) +
                                    (static_cast<size_t>(qb_row / G) * a.num_q_heads + kvh * G + qb_row % G) * D
                              : nullptr;
#pragma unroll
    for (int ks = 0; ks < S::kKSteps; ++ks) {
      const int d = ks * 16 + 2 * t4;
      qa[ks][0] = pa ? *reinterpret_cast<const uint32_t*>(pa + d) : 0u;
      qa[ks][1] = pb ? *reinterpret_cast<const uint32_t*>(pb + d) : 0u;
      qa[ks][2] = pa ? *reinterpret_cast<const uint32_t*>(pa + d + 8) : 0u;
      qa[ks][3] = pb ? *reinterpret_cast<const uint32_t*>(pb + d + 8) : 0u;
    }
  }

  // O fragments: o[j] = queries g8 (+8), columns 8 j + 2 t4 (+1)
  float o[S::kNTiles][4];
#pragma unroll
  for (int j = 0; j < S::kNTiles; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float mA = -INFINITY, mB = -INFINITY;  // running max of rows g8, g8 + 8
  float lA = 0.f, lB = 0.f;

  bool alive = true;
  for (int i = 0; i < npages; ++i) {
    const int s = i % NSTAGE;
    bool ok = wait(full0 + 8 * s, (i / NSTAGE) & 1);
    ok = __all_sync(kFull, ok);
    if (!ok) {
      alive = false;
      break;
    }
    const bool skip = skip_page[s];
    if (!skip) {
      const uint32_t kt = stage0 + s * S::kStage;
      const uint32_t vt = kt + S::kTile;
      // (1) S = Q . K^T, two n-tiles of 8 tokens
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int row = lr + ((lm >> 1) << 3);  // token
#pragma unroll
        for (int ks = 0; ks < S::kKSteps; ++ks) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kt + swz(row, 2 * ks + (lm & 1)), b0, b1, b2, b3);
          M::run(sc[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
          M::run(sc[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
        }
      }
      // (2) online softmax per query row
      float x[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) x[nt][e] = sc[nt][e] * a.qk_scale;
      float mxA = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
      float mxB = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
#pragma unroll
      for (int msk = 1; msk <= 2; msk <<= 1) {
        mxA = fmaxf(mxA, __shfl_xor_sync(kFull, mxA, msk));
        mxB = fmaxf(mxB, __shfl_xor_sync(kFull, mxB, msk));
      }
      const float nA = fmaxf(mA, mxA), nB = fmaxf(mB, mxB);
      const float alA = exp2f(mA - nA), alB = exp2f(mB - nB);
      mA = nA;
      mB = nB;
      float p[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        p[nt][0] = exp2f(x[nt][0] - nA);
        p[nt][1] = exp2f(x[nt][1] - nA);
        p[nt][2] = exp2f(x[nt][2] - nB);
        p[nt][3] = exp2f(x[nt][3] - nB);
      }
      lA = fmaf(lA, alA, p[0][0] + p[0][1] + p[1][0] + p[1][1]);
      lB = fmaf(lB, alB, p[0][2] + p[0][3] + p[1][2] + p[1][3]);
#pragma unroll
      for (int j = 0; j < S::kNTiles; ++j) {
        o[j][0] *= alA;
        o[j][1] *= alA;
        o[j][2] *= alB;
        o[j][3] *= alB;
      }
      // (3) P as the A operand (k = token): hi + lo 16-bit parts
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
      // (4) O += P . V, two n-tiles of D per ldmatrix
      {
        const int row = lr + ((lm & 1) << 3);  // token
#pragma unroll
        for (int j = 0; j < S::kNTiles; j += 2) {
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
    if (lane == 0) mbar_arrive(empty0 + 8 * s);
    // thread 0 restages this stage with page i + NSTAGE once every warp is done
    if (threadIdx.x == 0 && i + NSTAGE < npages) {
      if (issue(i + NSTAGE))
        ++issued;
      else
        alive = false;
    }
    if (warp == 0) alive = __shfl_sync(kFull, alive, 0);
    if (!alive) break;
  }
  if (!alive || abort_flag) {
    // after a give-up: wait (bounded) for the pages still in flight, i.e.
    // the last page staged into each stage
    if (threadIdx.x == 0) {
      for (int i = (issued > NSTAGE ? issued - NSTAGE : 0); i < issued; ++i) {
        const long long t0 = clock64();
        while (!mbar_try_wait(full0 + 8 * (i % NSTAGE), (i / NSTAGE) & 1) && clock64() - t0 < (1ll << 28)) {
        }
      }
    }
    return;
  }

  // row sums over the four lanes of a row
#pragma unroll
  for (int msk = 1; msk <= 2; msk <<= 1) {
    lA += __shfl_xor_sync(kFull, lA, msk);
    lB += __shfl_xor_sync(kFull, lB, msk);
  }
  // partial results of this chunk for the warp's queries
  const int rows[2] = {q0 + g8, q0 + g8 + 8};
  const float ms[2] = {mA, mB}, ls[2] = {lA, lB};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qi = rows[r];
    if (qi >= nq) continue;
    const int h = kvh * G + qi % G;
    const size_t slot = (static_cast<size_t>(qi / G) * a.num_q_heads + h) * a.num_chunks + chunk;
    float* dst = a.wp_o + slot * D;
#pragma unroll
    for (int j = 0; j < S::kNTiles; ++j)
      *reinterpret_cast<float2*>(dst + 8 * j + 2 * t4) = make_float2(o[j][2 * r], o[j][2 * r + 1]);
    if (t4 == 0) a.wp_ml[slot] = make_float2(ms[r], ls[r]);
  }
}

// Merge for the cascade: per (sequence, query head), the prefix chunks (when
// the sequence starts with the prefix) then the suffix partitions, in order,
// rescaled to their common max.  One warp per head.
template <typename T, int D>
__global__ void __launch_bounds__(128) paged_decode_prefix_merge_kernel(const DecodeArgs a) {
  constexpr int kEpl = D / 32;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x * 4 + warp;
  const int b = blockIdx.y;
  if (h >= a.num_q_heads) return;
  int ctx = a.context_lens[b];
  ctx = ctx < 0 ? 0 : (ctx > a.max_ctx ? a.max_ctx : ctx);
  const bool conforming = a.conform[b] != 0;
  const int tok_begin = conforming ? a.prefix_pages * kBlockSize : 0;
  const int n_suf = (ctx - tok_begin + a.partition - 1) / a.partition;
  const int n_pre = conforming ? a.num_chunks : 0;
  T* out = reinterpret_cast<T*>(a.out) + (static_cast<size_t>(b) * a.num_q_heads + h) * D + lane * kEpl;
  if (n_suf + n_pre == 0) {
#pragma unroll
    for (int e = 0; e < kEpl; ++e) out[e] = Fmt<T>::from_f32(0.f);
    return;
  }
  const size_t pre0 = (static_cast<size_t>(b) * a.num_q_heads + h) * a.num_chunks;
  const size_t suf0 = (static_cast<size_t>(b) * a.num_q_heads + h) * a.num_parts;
  float M = -INFINITY;
  for (int p = lane; p < n_pre; p += 32) M = fmaxf(M, a.wp_ml[pre0 + p].x);
  for (int p = lane; p < n_suf; p += 32) M = fmaxf(M, a.ws_ml[suf0 + p].x);
  M = warp_max(M);

  float acc[kEpl];
#pragma unroll
  for (int e = 0; e < kEpl; ++e) acc[e] = 0.f;
  float den = 0.f;
  auto add = [&](float2 ml, const float* op) {
    const float w = exp2f(ml.x - M);
    den = fmaf(w, ml.y, den);
#pragma unroll
    for (int e = 0; e < kEpl; ++e) acc[e] = fmaf(w, op[e], acc[e]);
  };
  for (int p = 0; p < n_pre; ++p) add(a.wp_ml[pre0 + p], a.wp_o + (pre0 + p) * D + lane * kEpl);
  for (int p = 0; p < n_suf; ++p) add(a.ws_ml[suf0 + p], a.ws_o + (suf0 + p) * D + lane * kEpl);
#pragma unroll
  for (int e = 0; e < kEpl; ++e) out[e] = Fmt<T>::from_f32(acc[e] / den);
}

}  // namespace pkv
