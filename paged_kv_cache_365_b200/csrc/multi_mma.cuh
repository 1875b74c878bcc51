// Paged attention for several query tokens per sequence (fp16 / bf16).
//
// "PagedAttention 与 vLLM 推理加速" §6: the large model verifies the small
// model's guessed tokens, i.e. scores several new tokens of one sequence in
// one pass; "LLM Systems 24 ..." §2.2.1.3: batches mix prefill chunks with
// decode steps.  Sequence b brings n_b new tokens (rows query_start[b] ..
// query_start[b+1]-1 of q), the last n_b of its context_lens[b] tokens;
// new token i sits at position ctx - n_b + i and attends over positions
// 0 .. ctx - n_b + i (§1: every token so far, itself included).
//
// Work split: one CTA per (kv-head, sequence, tile of 8 NT query rows,
// partition of keys).  A tile's rows are (token, head) pairs of one
// kv-head: row r is token r / G, head r % G of the group; they are the
// MMA's N dimension in NT n-tiles of 8, exactly as the GQA group is in the
// decode kernel, so one page's K and V fragments are loaded once and serve
// every row of the tile (NT is chosen per launch from the rows a sequence
// brings: a speculative-verification pass of a few tokens is one tile).
// Within the CTA, warp w walks pages w, w + NWARPS, ... of the partition
// with its own ring of TMA-staged tiles and keeps every row's state; the
// warps' states are merged in a fixed order at the end.  Per page:
//   S^T[16 tokens x 8 NT] = K . Q^T   (A = K via ldmatrix, B = queries)
//   causal mask: token j counts for row r when j <= pos(r)
//   O^T[D x 8 NT] += V^T . P^T         (A = V via ldmatrix.trans,
//                                       B = P^T by movmatrix, hi + lo parts)
// A key partition past a tile's last position is skipped.  Sequences whose
// whole context fits one partition write normalised rows; the others write
// per-partition partials that paged_multi_merge_kernel combines.
#pragma once

#include "decode_mma.cuh"

namespace pkv {

struct MultiArgs {
  void* out;                    // [T, Hq, D]
  const void* q;                // [T, Hq, D]
  const int32_t* block_tables;  // [B, bt_stride]
  const int32_t* context_lens;  // [B] (after this step's appends)
  const int32_t* query_start;   // [B + 1] row offsets into q / out
  float* ws_o;                  // [T][Hq][P][D]
  float2* ws_ml;                // [T][Hq][P] (max in log2 units, sum)
  long long bt_stride;
  int max_ctx;   // min(max_context_len, 16 * bt_stride)
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int num_blocks;
  int partition;
  int num_parts;  // ceil(max_ctx / partition)
  int tiles;      // row tiles per sequence in the grid: ceil(max_query_len * G / 16)
  int max_q;      // max_query_len
  int total_q;    // T
  float qk_scale; // scale * log2(e) (times the K scale over an FP8 pool)
  float v_scale;  // the V scale over an FP8 pool (tcgen05 kernel only)
  int* tc_ctr;           // tcgen05 kernel: [0] claim counter, [1] work-list length
  int2* tc_items;        // tcgen05 kernel: the work list
};

// Range-checked view of sequence b: context length, first row, new tokens.
// Returns false (and flags) when query_start is unusable for b.
__device__ __forceinline__ bool multi_seq(const MultiArgs& a, int b, int& ctx, int& q0, int& nq, bool report) {
  ctx = a.context_lens[b];
  if (ctx < 0 || ctx > a.max_ctx) {
    if (report) raise_error(PKV_ERR_CONTEXT_RANGE);
    ctx = ctx < 0 ? 0 : a.max_ctx;
  }
  q0 = a.query_start[b];
  const int q1 = a.query_start[b + 1];
  if (q0 < 0 || q1 < q0 || q1 > a.total_q || q1 - q0 > a.max_q) {
    if (report) raise_error(PKV_ERR_CONTEXT_RANGE);
    return false;
  }
  nq = q1 - q0;
  if (nq > ctx && report) raise_error(PKV_ERR_CONTEXT_RANGE);  // rows before position 0 give zeros
  return true;
}

template <typename T, int D, int G, int NT, int NWARPS, int NSTAGE>
__global__ void __launch_bounds__(NWARPS * 32)
    paged_multi_mma_kernel(const MultiArgs a, const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_v) {
  pdl_enter();
  using S = MmaShape<T, D, G, NWARPS, NSTAGE>;
  using M = Mma<T>;
  constexpr float kLazyMax = 8.f;  // the reference max moves only past 2^kLazyMax
  constexpr int kCols = 8 * NT;                 // query rows of a tile (the MMA's N)
  constexpr int kRecM = kCols * D, kRecL = kCols * D + kCols;  // warp record: o[kCols][D], m, l
  static_assert(size_t(kRecL + kCols) * sizeof(float) <= size_t(S::kWarpStageBytes),
                "a warp's record must fit in its own stages");
  const int kvh = blockIdx.x;
  const int b = blockIdx.y / a.tiles;
  const int tile = blockIdx.y % a.tiles;
  const int z = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3, lm = lane >> 3, lr = lane & 7;

  int ctx, q0, nq;
  if (!multi_seq(a, b, ctx, q0, nq, threadIdx.x == 0 && kvh == 0 && tile == 0 && z == 0)) return;
  const int R = nq * G;          // rows of this kv-head: row r = token r / G, head r % G
  const int r0 = tile * kCols;   // first row of the tile
  if (r0 >= R) return;
  const int base = ctx - nq;     // position of new token 0
  const int p_hi = base + (min(R, r0 + kCols) - 1) / G;
  const bool direct = ctx <= a.partition;  // one partition holds every key of the sequence
  const int tok0 = z * a.partition;
  const int tok1 = min(min(ctx, tok0 + a.partition), p_hi + 1);
  auto out_row = [&](int tr) -> size_t {  // row of q / out for tile row tr
    return static_cast<size_t>(q0 + tr / G) * a.num_q_heads + kvh * G + tr % G;
  };
  if (tok1 <= tok0) {
    // no key of this partition is visible to the tile; with one partition
    // (z = 0) every row sits before position 0: zeros
    if (direct && z == 0)
      for (int idx = threadIdx.x; idx < kCols * D; idx += NWARPS * 32) {
        const int tr = r0 + idx / D;
        if (tr < R) reinterpret_cast<T*>(a.out)[out_row(tr) * D + idx % D] = Fmt<T>::from_f32(0.f);
      }
    return;
  }

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

  const int pg0 = tok0 / kBlockSize;
  const int nblk = (tok1 - tok0 + kBlockSize - 1) / kBlockSize;
  const int my_n = warp < nblk ? (nblk - warp + NWARPS - 1) / NWARPS : 0;  // <= 32 * S::kTab
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
  uint32_t phase_bits = 0;
  auto issue = [&](int i) {
    const int phys = phys_of(i);
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

  // Q^T B fragments of column g8 of every n-tile (zero past the rows), and
  // the positions of this lane's columns 2 t4, 2 t4 + 1 (-1: sees no key)
  uint32_t qb[NT][S::kKSteps][2];
  int pos[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tr = r0 + 8 * nt + g8;
    const bool ok = tr < R;
    const T* qp = reinterpret_cast<const T*>(a.q) + (ok ? out_row(tr) : 0) * D;
#pragma unroll
    for (int ks = 0; ks < S::kKSteps; ++ks) {
      qb[nt][ks][0] = ok ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 2 * t4) : 0u;
      qb[nt][ks][1] = ok ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 8 + 2 * t4) : 0u;
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int c = r0 + 8 * nt + 2 * t4 + e;
      pos[nt][e] = c < R ? base + c / G : -1;
    }
  }

  // O^T accumulators: o[nt][mt] = rows d = 16 mt + g8 (+8), columns 2 t4 (+1)
  float o[NT][S::kKSteps][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int mt = 0; mt < S::kKSteps; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
  float mr[NT][2], lr_[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) mr[nt][0] = mr[nt][1] = -INFINITY, lr_[nt][0] = lr_[nt][1] = 0.f;
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
      // (1) S^T = K . Q^T for every n-tile, K fragments loaded once
      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
      {
        const int row = lr + ((lm & 1) << 3);
#pragma unroll
        for (int ks = 0; ks < S::kKSteps; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kt + swz(row, 2 * ks + (lm >> 1)), a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) M::run(sc[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
        }
      }
      // (2) causal mask per column, online softmax per column
      const int jA = page_tok + g8, jB = page_tok + g8 + 8;  // this lane's tokens
      uint32_t pb[NT][4];  // P^T B fragments: hi top, hi bottom, lo top, lo bottom
      bool moved = false;
      float al[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float x0 = jA <= pos[nt][0] ? sc[nt][0] * a.qk_scale : -INFINITY;
        const float x1 = jA <= pos[nt][1] ? sc[nt][1] * a.qk_scale : -INFINITY;
        const float x2 = jB <= pos[nt][0] ? sc[nt][2] * a.qk_scale : -INFINITY;
        const float x3 = jB <= pos[nt][1] ? sc[nt][3] * a.qk_scale : -INFINITY;
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
        // the reference max moves only when a score passes it by more than
        // 2^kLazyMax (one vote a page otherwise; see the decode kernel)
        al[nt][0] = al[nt][1] = 1.f;
        if (__any_sync(kFull, mx0 > mr[nt][0] + kLazyMax || mx1 > mr[nt][1] + kLazyMax)) {
#pragma unroll
          for (int msk = 4; msk <= 16; msk <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, msk));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, msk));
          }
          const float n0 = fmaxf(mr[nt][0], mx0), n1 = fmaxf(mr[nt][1], mx1);
          // a column that has seen no key yet keeps max -inf: subtract 0 instead
          const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
          al[nt][0] = exp2_sfu(mr[nt][0] - u0);
          al[nt][1] = exp2_sfu(mr[nt][1] - u1);
          mr[nt][0] = n0;
          mr[nt][1] = n1;
          lr_[nt][0] *= al[nt][0];
          lr_[nt][1] *= al[nt][1];
          moved = true;
        }
        const float u0 = mr[nt][0] == -INFINITY ? 0.f : mr[nt][0], u1 = mr[nt][1] == -INFINITY ? 0.f : mr[nt][1];
        const float p0 = exp2_sfu(x0 - u0), p1 = exp2_sfu(x1 - u1), p2 = exp2_sfu(x2 - u0), p3 = exp2_sfu(x3 - u1);
        lr_[nt][0] += p0 + p2;
        lr_[nt][1] += p1 + p3;
        const uint32_t top_hi = M::pack(p0, p1), bot_hi = M::pack(p2, p3);
        const float2 th = M::unpack(top_hi), bh = M::unpack(bot_hi);
        pb[nt][0] = movm_t(top_hi);
        pb[nt][1] = movm_t(bot_hi);
        pb[nt][2] = movm_t(M::pack(p0 - th.x, p1 - th.y));
        pb[nt][3] = movm_t(M::pack(p2 - bh.x, p3 - bh.y));
      }
      if (__any_sync(kFull, moved)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int mt = 0; mt < S::kKSteps; ++mt) {
            o[nt][mt][0] *= al[nt][0];
            o[nt][mt][1] *= al[nt][1];
            o[nt][mt][2] *= al[nt][0];
            o[nt][mt][3] *= al[nt][1];
          }
      }
      // V^T fragment halves of tokens past the visible range are zeroed (an
      // unwritten slot may hold NaN, and 0 * NaN is NaN)
      uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
      if (nvalid < kBlockSize) {
        keep_lo = (2 * t4 < nvalid ? 0x0000ffffu : 0u) | (2 * t4 + 1 < nvalid ? 0xffff0000u : 0u);
        keep_hi = (2 * t4 + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * t4 + 9 < nvalid ? 0xffff0000u : 0u);
      }
      // (3) O^T += V^T . P^T, V fragments loaded once for every n-tile (the
      // masks only on a partial last page)
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
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            M::run(o[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            M::run(o[nt][mt], a0, a1, a2, a3, pb[nt][2], pb[nt][3]);
          }
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
  if (consumed < my_n) {  // after a give-up: wait (bounded) for copies in flight
    const int last = min(my_n, consumed + NSTAGE);
    for (int i = consumed; i < last; ++i) {
      const int s = i % NSTAGE;
      mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
      phase_bits ^= 1u << s;
    }
  }
  // running sums over the lanes of each column (same t4)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int msk = 4; msk <= 16; msk <<= 1) {
      lr_[nt][0] += __shfl_xor_sync(kFull, lr_[nt][0], msk);
      lr_[nt][1] += __shfl_xor_sync(kFull, lr_[nt][1], msk);
    }

  // warp record [o: kCols x D][m: kCols][l: kCols] in the warp's own stages
  float* rec = reinterpret_cast<float*>(my_stages);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int ca = 8 * nt + 2 * t4, cb = ca + 1;
#pragma unroll
    for (int mt = 0; mt < S::kKSteps; ++mt) {
      const int d0 = 16 * mt + g8;
      rec[ca * D + d0] = o[nt][mt][0];
      rec[ca * D + d0 + 8] = o[nt][mt][2];
      rec[cb * D + d0] = o[nt][mt][1];
      rec[cb * D + d0 + 8] = o[nt][mt][3];
    }
    if (g8 == 0) {
      rec[kRecM + ca] = mr[nt][0];
      rec[kRecL + ca] = lr_[nt][0];
      rec[kRecM + cb] = mr[nt][1];
      rec[kRecL + cb] = lr_[nt][1];
    }
  }
  if (__syncthreads_or(timed_out)) return;

  // merge the warps in a fixed order; rows with no key in this partition
  // are left to the other partitions (the merge never reads them)
  for (int idx = threadIdx.x; idx < kCols * D; idx += NWARPS * 32) {
    const int c = idx / D, d = idx % D;
    const int tr = r0 + c;
    if (tr >= R) continue;
    const int p = base + tr / G;
    const size_t row = out_row(tr);
    if (p < tok0) {
      if (direct) reinterpret_cast<T*>(a.out)[row * D + d] = Fmt<T>::from_f32(0.f);
      continue;
    }
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w)
      Mx = fmaxf(Mx, reinterpret_cast<const float*>(smem + w * S::kWarpStageBytes)[kRecM + c]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) {
      const float* rw = reinterpret_cast<const float*>(smem + w * S::kWarpStageBytes);
      const float sc = exp2f(rw[kRecM + c] - Mx);
      num = fmaf(sc, rw[c * D + d], num);
      den = fmaf(sc, rw[kRecL + c], den);
    }
    if (direct) {
      reinterpret_cast<T*>(a.out)[row * D + d] = Fmt<T>::from_f32(num / den);
    } else {
      const size_t wrow = row * a.num_parts + z;
      a.ws_o[wrow * D + d] = num;
      if (d == 0) a.ws_ml[wrow] = make_float2(Mx, den);
    }
  }
}

// Shared-memory layout of the kernels whose warps all read every page of a
// partition (paged_multi_rows_kernel, paged_multi_fa_kernel): NSTAGE stages
// of KP pages (K tile then V tile each), a full barrier and a release
// counter per stage, the partition's page table.
template <int D, int NW, int NSTAGE, int KP>
struct RowsShape {
  static constexpr int kTile = kBlockSize * D * 2;
  static constexpr int kPage = 2 * kTile;      // K tile, then V tile
  static constexpr int kStage = KP * kPage;
  static constexpr int kKSteps = D / 16;
  static constexpr int kBoxes = D / 64;
  static constexpr int kMaxPages = 128;  // pages of the longest partition (2048 tokens)
  // stages | full barriers | release counters | page table
  static constexpr size_t kBarOff = size_t(NSTAGE) * kStage;
  static constexpr size_t kCntOff = kBarOff + size_t(NSTAGE) * 8;
  static constexpr size_t kTabOff = kCntOff + size_t(NSTAGE) * 4;
  static constexpr size_t kSmem = 1024 + kTabOff + size_t(kMaxPages) * 4;
  static_assert(kPage % 1024 == 0, "swizzled boxes need 1024-byte alignment");
};

// The CTA-wide page ring of the kernels whose warps all read every page of
// a partition: the partition's page table in shared memory, NSTAGE stages
// of KP pages filled by TMA, a full barrier per stage, and a release
// counter per stage.  Every warp waits for step c's stage; after its last
// read of the stage a warp counts itself out, and the warp that completes
// the count refills the stage with step c + NSTAGE, so the warps drift up
// to NSTAGE steps apart instead of meeting at a CTA barrier.
template <int D, int NW, int NSTAGE, int KP>
struct PageRing {
  using S = RowsShape<D, NW, NSTAGE, KP>;
  uint32_t stage0, bar0;
  unsigned int* released;  // warps done with the stage, per stage
  int* table;              // physical block of page i of the partition, or -1
  int nblk, nstep;
  uint32_t phase_bits;

  // Lays the ring out in `smem` (1024-byte aligned), reads the partition's
  // table entries (flagging any outside the pool), initialises the
  // barriers and issues the first NSTAGE steps.  Every thread of the CTA
  // calls it; it ends with a CTA barrier.
  __device__ void init(unsigned char* smem, const MultiArgs& a, int b, int kvh, int tok0, int tok1,
                       const CUtensorMap* mk, const CUtensorMap* mv) {
    stage0 = smem_addr(smem);
    bar0 = smem_addr(smem + S::kBarOff);
    released = reinterpret_cast<unsigned int*>(smem + S::kCntOff);
    table = reinterpret_cast<int*>(smem + S::kTabOff);
    phase_bits = 0;
    const int pg0 = tok0 / kBlockSize;
    nblk = (tok1 - tok0 + kBlockSize - 1) / kBlockSize;  // <= S::kMaxPages
    nstep = (nblk + KP - 1) / KP;
    for (int j = threadIdx.x; j < nblk; j += NW * 32) {
      const int e = a.block_tables[static_cast<long long>(b) * a.bt_stride + pg0 + j];
      const bool in = e >= 0 && e < a.num_blocks;
      if (!in) raise_error(PKV_ERR_BLOCK_RANGE);
      table[j] = in ? e : -1;
    }
    if (threadIdx.x == 0) {
      for (int s = 0; s < NSTAGE; ++s) {
        mbar_init(bar0 + 8 * s, 1);
        released[s] = 0u;
      }
      fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
      for (int c = 0; c < NSTAGE; ++c) issue(c, a.num_kv_heads, kvh, mk, mv);
  }

  // pages KP c .. KP c + KP - 1 into stage c % NSTAGE (one lane); pages past
  // the partition or outside the pool are not copied
  __device__ void issue(int c, int num_kv_heads, int kvh, const CUtensorMap* mk, const CUtensorMap* mv) {
    if (c >= nstep) return;
    const uint32_t bar = bar0 + 8 * (c % NSTAGE);
    uint32_t bytes = 0;
#pragma unroll
    for (int p = 0; p < KP; ++p) {
      const int i = c * KP + p;
      if (i < nblk && table[i] >= 0) bytes += S::kPage;
    }
    if (bytes == 0) {
      mbar_arrive(bar);
      return;
    }
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
    for (int p = 0; p < KP; ++p) {
      const int i = c * KP + p;
      if (i < nblk && table[i] >= 0) {
        const uint32_t dst = stage0 + (c % NSTAGE) * S::kStage + p * S::kPage;
        const int y = (table[i] * num_kv_heads + kvh) * kBlockSize;
#pragma unroll
        for (int bx = 0; bx < S::kBoxes; ++bx) {
          tma_load_2d(dst + bx * 2048, mk, bx * 64, y, bar);
          tma_load_2d(dst + S::kTile + bx * 2048, mv, bx * 64, y, bar);
        }
      }
    }
  }

  // Waits (bounded, the whole warp) for step c's stage; false = gave up.
  __device__ bool wait(int c) {
    const int s = c % NSTAGE;
    const bool ok = __all_sync(kFull, mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u));
    phase_bits ^= 1u << s;
    return ok;
  }

  __device__ uint32_t stage(int c) const { return stage0 + (c % NSTAGE) * S::kStage; }

  // This warp is done with step c's stage; the last of the NW warps to say
  // so refills it (the fences order every warp's reads of the stage before
  // the copy that overwrites it).
  __device__ void release(int c, int num_kv_heads, int kvh, const CUtensorMap* mk, const CUtensorMap* mv) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
      __threadfence_block();
      const unsigned int before = atomicAdd(&released[c % NSTAGE], 1u);
      if (before % NW == NW - 1) {
        __threadfence_block();
        issue(c + NSTAGE, num_kv_heads, kvh, mk, mv);
      }
    }
  }

  // After a give-up, past a CTA barrier: thread 0 waits, bounded, for the
  // last step issued into each stage, so no copy lands after the CTA exits.
  __device__ void drain() {
    if (threadIdx.x == 0) {
      unsigned int issued = 0;  // NSTAGE + the refills (one per NW releases)
      for (int st = 0; st < NSTAGE; ++st) issued += released[st] / NW;
      issued = min(static_cast<unsigned int>(nstep), issued + NSTAGE);
      for (int c = max(0, static_cast<int>(issued) - NSTAGE); c < static_cast<int>(issued); ++c)
        mbar_wait_bounded(bar0 + 8 * (c % NSTAGE), (c / NSTAGE) & 1u);
    }
  }
};

// 17-32 rows per sequence and kv-head (speculative verification with GQA):
// the warps of a CTA split the rows instead of the pages.  Warp w owns the
// 8 rows r0 + 8 w .. r0 + 8 w + 7 (one n-tile, so registers stay as in
// decode) and every warp consumes every page of the partition from the
// CTA's PageRing.  A warp takes a stage's KP pages in one step: their score
// MMAs form independent chains, one max / rescale serves all of them, and
// their P.V products interleave, so a step has KP times the independent
// work of a page at the same per-step softmax cost.  A page is read once
// per CTA for all its 8 NW rows; the warps' rows are disjoint, so each
// writes its own outputs.
//
// Resident warps per SM the register budget is sized for: 5 CTAs of 3
// warps (up to 128 registers a thread, no spills) measured faster than 6
// CTAs (96 registers) or 8 (80).
#ifndef PKV_ROWS_WARPS_PER_SM
#define PKV_ROWS_WARPS_PER_SM 15
#endif
template <typename T, int D, int G, int NW, int NSTAGE, int KP>
__global__ void __launch_bounds__(NW * 32, PKV_ROWS_WARPS_PER_SM / NW)
    paged_multi_rows_kernel(const MultiArgs a, const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v) {
  pdl_enter();
  using S = RowsShape<D, NW, NSTAGE, KP>;
  using M = Mma<T>;
  constexpr float kLazyMax = 8.f;  // the reference max moves only past 2^kLazyMax
  constexpr int kCols = 8 * NW;
  const int kvh = blockIdx.x;
  const int b = blockIdx.y / a.tiles;
  const int tile = blockIdx.y % a.tiles;
  const int z = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3, lm = lane >> 3, lr = lane & 7;

  int ctx, q0, nq;
  if (!multi_seq(a, b, ctx, q0, nq, threadIdx.x == 0 && kvh == 0 && tile == 0 && z == 0)) return;
  const int R = nq * G;
  const int r0 = tile * kCols;
  if (r0 >= R) return;
  const int base = ctx - nq;
  const int p_hi = base + (min(R, r0 + kCols) - 1) / G;
  const bool direct = ctx <= a.partition;
  const int tok0 = z * a.partition;
  const int tok1 = min(min(ctx, tok0 + a.partition), p_hi + 1);
  auto out_row = [&](int tr) -> size_t {
    return static_cast<size_t>(q0 + tr / G) * a.num_q_heads + kvh * G + tr % G;
  };
  if (tok1 <= tok0) {
    if (direct && z == 0)
      for (int idx = threadIdx.x; idx < kCols * D; idx += NW * 32) {
        const int tr = r0 + idx / D;
        if (tr < R) reinterpret_cast<T*>(a.out)[out_row(tr) * D + idx % D] = Fmt<T>::from_f32(0.f);
      }
    return;
  }

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  PageRing<D, NW, NSTAGE, KP> ring;
  ring.init(smem_raw + pad, a, b, kvh, tok0, tok1, &tmap_k, &tmap_v);
  const int nstep = ring.nstep;

  // this warp's column g8 (row r0 + 8 warp + g8) and its lane's columns 2 t4, 2 t4 + 1
  uint32_t qb[S::kKSteps][2];
  int pos0, pos1;
  {
    const int tr = r0 + 8 * warp + g8;
    const bool ok = tr < R;
    const T* qp = reinterpret_cast<const T*>(a.q) + (ok ? out_row(tr) : 0) * D;
#pragma unroll
    for (int ks = 0; ks < S::kKSteps; ++ks) {
      qb[ks][0] = ok ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 2 * t4) : 0u;
      qb[ks][1] = ok ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 8 + 2 * t4) : 0u;
    }
    const int c0 = r0 + 8 * warp + 2 * t4;
    pos0 = c0 < R ? base + c0 / G : -1;
    pos1 = c0 + 1 < R ? base + (c0 + 1) / G : -1;
  }
  float o[S::kKSteps][4];
#pragma unroll
  for (int mt = 0; mt < S::kKSteps; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  bool bad = false;

  for (int c = 0; c < nstep; ++c) {
    if (!ring.wait(c)) {  // this warp gives up; the others time out on the stages it never releases
      if (lane == 0) raise_error(PKV_ERR_TIMEOUT);
      bad = true;
      break;
    }
    // the step's pages: held (copied) or not, and tokens in each
    bool held[KP];
    int nvalid[KP];
    bool full = true;
#pragma unroll
    for (int p = 0; p < KP; ++p) {
      const int i = c * KP + p;
      held[p] = i < ring.nblk && ring.table[i] >= 0;
      nvalid[p] = held[p] ? min(kBlockSize, tok1 - tok0 - i * kBlockSize) : 0;
      full = full && nvalid[p] == kBlockSize;
    }
    const uint32_t st = ring.stage(c);
    // S^T per page in two independent accumulation chains
    float x[KP][4];
#pragma unroll
    for (int p = 0; p < KP; ++p) {
      float sc[4] = {0.f, 0.f, 0.f, 0.f}, sd[4] = {0.f, 0.f, 0.f, 0.f};
      if (held[p]) {
        const uint32_t kt = st + p * S::kPage;
        const int row = lr + ((lm & 1) << 3);
#pragma unroll
        for (int ks = 0; ks < S::kKSteps; ks += 2) {
          uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
          ldsm_x4(kt + swz(row, 2 * ks + (lm >> 1)), a0, a1, a2, a3);
          ldsm_x4(kt + swz(row, 2 * ks + 2 + (lm >> 1)), b0, b1, b2, b3);
          M::run(sc, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
          M::run(sd, b0, b1, b2, b3, qb[ks + 1][0], qb[ks + 1][1]);
        }
      }
      // causal mask (it also cuts the partition's end and a missing page:
      // every column's position is below tok1)
      const int jA = tok0 + (c * KP + p) * kBlockSize + g8, jB = jA + 8;
      const bool h = held[p];
      x[p][0] = h && jA <= pos0 ? (sc[0] + sd[0]) * a.qk_scale : -INFINITY;
      x[p][1] = h && jA <= pos1 ? (sc[1] + sd[1]) * a.qk_scale : -INFINITY;
      x[p][2] = h && jB <= pos0 ? (sc[2] + sd[2]) * a.qk_scale : -INFINITY;
      x[p][3] = h && jB <= pos1 ? (sc[3] + sd[3]) * a.qk_scale : -INFINITY;
    }
    float mx0 = fmaxf(x[0][0], x[0][2]), mx1 = fmaxf(x[0][1], x[0][3]);
#pragma unroll
    for (int p = 1; p < KP; ++p) {
      mx0 = fmaxf(mx0, fmaxf(x[p][0], x[p][2]));
      mx1 = fmaxf(mx1, fmaxf(x[p][1], x[p][3]));
    }
    // the reference max moves only when a score passes it by more than
    // 2^kLazyMax (one vote a step otherwise; see the decode kernel)
    float al0 = 1.f, al1 = 1.f;
    if (__any_sync(kFull, mx0 > m0 + kLazyMax || mx1 > m1 + kLazyMax)) {
#pragma unroll
      for (int msk = 4; msk <= 16; msk <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, msk));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, msk));
      }
      const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
      const float v0 = n0 == -INFINITY ? 0.f : n0, v1 = n1 == -INFINITY ? 0.f : n1;
      al0 = exp2_sfu(m0 - v0);
      al1 = exp2_sfu(m1 - v1);
      m0 = n0;
      m1 = n1;
    }
    const float u0 = m0 == -INFINITY ? 0.f : m0, u1 = m1 == -INFINITY ? 0.f : m1;
    uint32_t pb0[KP], pb1[KP], pl0[KP], pl1[KP];
    float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
    for (int p = 0; p < KP; ++p) {
      const float e0 = exp2_sfu(x[p][0] - u0), e1 = exp2_sfu(x[p][1] - u1);
      const float e2 = exp2_sfu(x[p][2] - u0), e3 = exp2_sfu(x[p][3] - u1);
      sum0 += e0 + e2;
      sum1 += e1 + e3;
      const uint32_t top_hi = M::pack(e0, e1), bot_hi = M::pack(e2, e3);
      const float2 th = M::unpack(top_hi), bh = M::unpack(bot_hi);
      pb0[p] = movm_t(top_hi);
      pb1[p] = movm_t(bot_hi);
      pl0[p] = movm_t(M::pack(e0 - th.x, e1 - th.y));
      pl1[p] = movm_t(M::pack(e2 - bh.x, e3 - bh.y));
    }
    l0 = fmaf(l0, al0, sum0);
    l1 = fmaf(l1, al1, sum1);
    if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
      for (int mt = 0; mt < S::kKSteps; ++mt) {
        o[mt][0] *= al0;
        o[mt][1] *= al1;
        o[mt][2] *= al0;
        o[mt][3] *= al1;
      }
    }
    // O^T += V^T . P^T per page; slots past a page's tokens may hold
    // anything (NaN included), so their V is zeroed
    auto pv = [&](auto masked) {
      uint32_t keep_lo[KP], keep_hi[KP];
      if constexpr (decltype(masked)::value) {
#pragma unroll
        for (int p = 0; p < KP; ++p) {
          const int n = nvalid[p];
          keep_lo[p] = (2 * t4 < n ? 0x0000ffffu : 0u) | (2 * t4 + 1 < n ? 0xffff0000u : 0u);
          keep_hi[p] = (2 * t4 + 8 < n ? 0x0000ffffu : 0u) | (2 * t4 + 9 < n ? 0xffff0000u : 0u);
        }
      }
      const int row = lr + ((lm >> 1) << 3);
#pragma unroll
      for (int mt = 0; mt < S::kKSteps; ++mt) {
#pragma unroll
        for (int p = 0; p < KP; ++p) {
          if constexpr (decltype(masked)::value)
            if (!held[p]) continue;
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(st + p * S::kPage + S::kTile + swz(row, 2 * mt + (lm & 1)), a0, a1, a2, a3);
          if constexpr (decltype(masked)::value) {
            a0 &= keep_lo[p];
            a1 &= keep_lo[p];
            a2 &= keep_hi[p];
            a3 &= keep_hi[p];
          }
          M::run(o[mt], a0, a1, a2, a3, pb0[p], pb1[p]);
          M::run(o[mt], a0, a1, a2, a3, pl0[p], pl1[p]);
        }
      }
    };
    if (full)
      pv(std::false_type{});
    else
      pv(std::true_type{});
    ring.release(c, a.num_kv_heads, kvh, &tmap_k, &tmap_v);
  }
  // every copy this CTA issued lands before the CTA exits
  if (__syncthreads_or(bad)) {
    ring.drain();
    return;
  }
#pragma unroll
  for (int msk = 4; msk <= 16; msk <<= 1) {
    l0 += __shfl_xor_sync(kFull, l0, msk);
    l1 += __shfl_xor_sync(kFull, l1, msk);
  }
  // columns 2 t4, 2 t4 + 1 of this warp: rows d = 16 mt + g8 (+8)
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int tr = r0 + 8 * warp + 2 * t4 + e;
    if (tr >= R) continue;
    const int p = base + tr / G;
    const size_t row = out_row(tr);
    const float mm = e ? m1 : m0, ll = e ? l1 : l0;
    if (p < tok0) {  // no key of this partition (or before position 0)
      if (direct)
#pragma unroll
        for (int mt = 0; mt < S::kKSteps; ++mt) {
          reinterpret_cast<T*>(a.out)[row * D + 16 * mt + g8] = Fmt<T>::from_f32(0.f);
          reinterpret_cast<T*>(a.out)[row * D + 16 * mt + g8 + 8] = Fmt<T>::from_f32(0.f);
        }
      continue;
    }
    if (direct) {
      const float inv = 1.f / ll;
#pragma unroll
      for (int mt = 0; mt < S::kKSteps; ++mt) {
        reinterpret_cast<T*>(a.out)[row * D + 16 * mt + g8] = Fmt<T>::from_f32(o[mt][e] * inv);
        reinterpret_cast<T*>(a.out)[row * D + 16 * mt + g8 + 8] = Fmt<T>::from_f32(o[mt][2 + e] * inv);
      }
    } else {
      const size_t wrow = row * a.num_parts + z;
#pragma unroll
      for (int mt = 0; mt < S::kKSteps; ++mt) {
        a.ws_o[wrow * D + 16 * mt + g8] = o[mt][e];
        a.ws_o[wrow * D + 16 * mt + g8 + 8] = o[mt][2 + e];
      }
      if (g8 == 0) a.ws_ml[wrow] = make_float2(mm, ll);
    }
  }
}

// Many rows per sequence (prefill chunks, long verification runs): the
// rows are the MMA's M dimension, as in FlashAttention-2.  One CTA of NWF
// warps per (kv-head, sequence, tile of 16 NWF rows, key partition); warp w
// owns rows r0 + 16 w .. r0 + 16 w + 15 and keeps their queries in
// registers as A fragments.  Pages come through the same CTA-wide ring as
// in paged_multi_rows_kernel (KP pages per stage, release counters).  Per
// page and warp:
//   S[16 rows x 16 tokens] = Q . K^T   (B = K rows via ldmatrix)
//   causal mask per row, online softmax per row (a quad of lanes holds a
//   row's 16 scores)
//   O[16 x D] += P . V                 (A = P from S's own registers, in
//                                       hi + lo 16-bit parts; B = V via
//                                       ldmatrix.trans)
// A warp skips the arithmetic of pages past its rows' last position.
// Against the row-split kernel a page's fragments serve 16 rows of a warp
// instead of 8 and P needs no transposes: per row, half the shared-memory
// reads and about two thirds of the instructions.
#ifndef PKV_FA_MIN_CTAS
#define PKV_FA_MIN_CTAS 3
#endif
template <typename T, int D, int G, int NWF, int NSTAGE, int KP>
__global__ void __launch_bounds__(NWF * 32, PKV_FA_MIN_CTAS)
    paged_multi_fa_kernel(const MultiArgs a, const __grid_constant__ CUtensorMap tmap_k,
                          const __grid_constant__ CUtensorMap tmap_v) {
  pdl_enter();
  using S = RowsShape<D, NWF, NSTAGE, KP>;
  using M = Mma<T>;
  constexpr int kRows = 16 * NWF;
  constexpr int kNT = D / 8;  // n-tiles of O
  const int kvh = blockIdx.x;
  const int b = blockIdx.y / a.tiles;
  const int tile = blockIdx.y % a.tiles;
  const int z = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3, lm = lane >> 3, lr = lane & 7;

  int ctx, q0, nq;
  if (!multi_seq(a, b, ctx, q0, nq, threadIdx.x == 0 && kvh == 0 && tile == 0 && z == 0)) return;
  const int R = nq * G;
  const int r0 = tile * kRows;
  if (r0 >= R) return;
  const int base = ctx - nq;
  const int p_hi = base + (min(R, r0 + kRows) - 1) / G;
  const bool direct = ctx <= a.partition;
  const int tok0 = z * a.partition;
  const int tok1 = min(min(ctx, tok0 + a.partition), p_hi + 1);
  auto out_row = [&](int tr) -> size_t {
    return static_cast<size_t>(q0 + tr / G) * a.num_q_heads + kvh * G + tr % G;
  };
  if (tok1 <= tok0) {
    if (direct && z == 0)
      for (int idx = threadIdx.x; idx < kRows * D; idx += NWF * 32) {
        const int tr = r0 + idx / D;
        if (tr < R) reinterpret_cast<T*>(a.out)[out_row(tr) * D + idx % D] = Fmt<T>::from_f32(0.f);
      }
    return;
  }

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  PageRing<D, NWF, NSTAGE, KP> ring;
  ring.init(smem_raw + pad, a, b, kvh, tok0, tok1, &tmap_k, &tmap_v);
  const int nstep = ring.nstep;

  // this warp's rows: fragment rows g8 (row A) and g8 + 8 (row B)
  const int wr0 = r0 + 16 * warp;
  const int trA = wr0 + g8, trB = wr0 + g8 + 8;
  const bool okA = trA < R, okB = trB < R;
  const int posA = okA ? base + trA / G : -1, posB = okB ? base + trB / G : -1;
  const int wpos = wr0 < R ? base + (min(R, wr0 + 16) - 1) / G : -1;  // the warp's last position
  uint32_t qa[S::kKSteps][4];
  {
    const T* qA = reinterpret_cast<const T*>(a.q) + (okA ? out_row(trA) : 0) * D;
    const T* qB = reinterpret_cast<const T*>(a.q) + (okB ? out_row(trB) : 0) * D;
#pragma unroll
    for (int ks = 0; ks < S::kKSteps; ++ks) {
      qa[ks][0] = okA ? *reinterpret_cast<const uint32_t*>(qA + ks * 16 + 2 * t4) : 0u;
      qa[ks][1] = okB ? *reinterpret_cast<const uint32_t*>(qB + ks * 16 + 2 * t4) : 0u;
      qa[ks][2] = okA ? *reinterpret_cast<const uint32_t*>(qA + ks * 16 + 8 + 2 * t4) : 0u;
      qa[ks][3] = okB ? *reinterpret_cast<const uint32_t*>(qB + ks * 16 + 8 + 2 * t4) : 0u;
    }
  }
  float o[kNT][4];
#pragma unroll
  for (int j = 0; j < kNT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;  // lA, lB: this lane's part of the row sums
  bool bad = false;

  for (int c = 0; c < nstep; ++c) {
    if (!ring.wait(c)) {  // this warp gives up; the others time out on the stages it never releases
      if (lane == 0) raise_error(PKV_ERR_TIMEOUT);
      bad = true;
      break;
    }
    bool run[KP];
    int nvalid[KP], page_tok[KP];
    bool any = false, full = true;
#pragma unroll
    for (int p = 0; p < KP; ++p) {
      const int i = c * KP + p;
      page_tok[p] = tok0 + i * kBlockSize;
      run[p] = i < ring.nblk && ring.table[i] >= 0 && page_tok[p] <= wpos;
      nvalid[p] = run[p] ? min(kBlockSize, tok1 - page_tok[p]) : 0;
      any = any || run[p];
      full = full && nvalid[p] == kBlockSize;
    }
    if (any) {
      const uint32_t st = ring.stage(c);
      // S per page: n-tile 0 = tokens 0-7, n-tile 1 = tokens 8-15; two
      // accumulation chains (even and odd k-steps) each
      float x[KP][2][4];
#pragma unroll
      for (int p = 0; p < KP; ++p) {
        float sa[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float sb[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        if (run[p]) {
          const uint32_t kt = st + p * S::kPage;
          const int row = lr + ((lm >> 1) << 3);
#pragma unroll
          for (int ks = 0; ks < S::kKSteps; ks += 2) {
            uint32_t k0, k1, k2, k3, u0, u1, u2, u3;
            ldsm_x4(kt + swz(row, 2 * ks + (lm & 1)), k0, k1, k2, k3);
            ldsm_x4(kt + swz(row, 2 * ks + 2 + (lm & 1)), u0, u1, u2, u3);
            M::run(sa[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], k0, k1);
            M::run(sa[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], k2, k3);
            M::run(sb[0], qa[ks + 1][0], qa[ks + 1][1], qa[ks + 1][2], qa[ks + 1][3], u0, u1);
            M::run(sb[1], qa[ks + 1][0], qa[ks + 1][1], qa[ks + 1][2], qa[ks + 1][3], u2, u3);
          }
        }
        // causal mask (it also cuts the partition's end and a skipped page:
        // every row's position is below tok1)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int j = page_tok[p] + nt * 8 + 2 * t4;
          const bool h = run[p];
          x[p][nt][0] = h && j <= posA ? (sa[nt][0] + sb[nt][0]) * a.qk_scale : -INFINITY;
          x[p][nt][1] = h && j + 1 <= posA ? (sa[nt][1] + sb[nt][1]) * a.qk_scale : -INFINITY;
          x[p][nt][2] = h && j <= posB ? (sa[nt][2] + sb[nt][2]) * a.qk_scale : -INFINITY;
          x[p][nt][3] = h && j + 1 <= posB ? (sa[nt][3] + sb[nt][3]) * a.qk_scale : -INFINITY;
        }
      }
      float mxA = -INFINITY, mxB = -INFINITY;
#pragma unroll
      for (int p = 0; p < KP; ++p)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          mxA = fmaxf(mxA, fmaxf(x[p][nt][0], x[p][nt][1]));
          mxB = fmaxf(mxB, fmaxf(x[p][nt][2], x[p][nt][3]));
        }
#pragma unroll
      for (int msk = 1; msk <= 2; msk <<= 1) {
        mxA = fmaxf(mxA, __shfl_xor_sync(kFull, mxA, msk));
        mxB = fmaxf(mxB, __shfl_xor_sync(kFull, mxB, msk));
      }
      const float nA = fmaxf(mA, mxA), nB = fmaxf(mB, mxB);
      const float uA = nA == -INFINITY ? 0.f : nA, uB = nB == -INFINITY ? 0.f : nB;
      const float alA = exp2_sfu(mA - uA), alB = exp2_sfu(mB - uB);
      mA = nA;
      mB = nB;
      // P as A fragments (rows A / B, tokens 2 t4.. of each n-tile), hi + lo
      uint32_t ph[KP][4], pl[KP][4];
      float sumA = 0.f, sumB = 0.f;
#pragma unroll
      for (int p = 0; p < KP; ++p) {
        float e[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          e[nt][0] = exp2_sfu(x[p][nt][0] - uA);
          e[nt][1] = exp2_sfu(x[p][nt][1] - uA);
          e[nt][2] = exp2_sfu(x[p][nt][2] - uB);
          e[nt][3] = exp2_sfu(x[p][nt][3] - uB);
          sumA += e[nt][0] + e[nt][1];
          sumB += e[nt][2] + e[nt][3];
        }
        // a0 = (row A, tokens 2t, 2t+1), a1 = (row B, same), a2 / a3 = tokens + 8
        const float v[4][2] = {{e[0][0], e[0][1]}, {e[0][2], e[0][3]}, {e[1][0], e[1][1]}, {e[1][2], e[1][3]}};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          ph[p][r] = M::pack(v[r][0], v[r][1]);
          const float2 hv = M::unpack(ph[p][r]);
          pl[p][r] = M::pack(v[r][0] - hv.x, v[r][1] - hv.y);
        }
      }
      lA = fmaf(lA, alA, sumA);
      lB = fmaf(lB, alB, sumB);
      if (__any_sync(kFull, alA != 1.f || alB != 1.f)) {
#pragma unroll
        for (int j = 0; j < kNT; ++j) {
          o[j][0] *= alA;
          o[j][1] *= alA;
          o[j][2] *= alB;
          o[j][3] *= alB;
        }
      }
      // O += P . V per page; slots past a page's tokens may hold anything
      // (NaN included), so their V is zeroed on a partial page
      auto pv = [&](auto masked) {
        const int row = lr + ((lm & 1) << 3);
#pragma unroll
        for (int p = 0; p < KP; ++p) {
          if constexpr (decltype(masked)::value)
            if (!run[p]) continue;
          uint32_t klo = 0xffffffffu, khi = 0xffffffffu;
          if constexpr (decltype(masked)::value) {
            const int n = nvalid[p];
            klo = (2 * t4 < n ? 0x0000ffffu : 0u) | (2 * t4 + 1 < n ? 0xffff0000u : 0u);
            khi = (2 * t4 + 8 < n ? 0x0000ffffu : 0u) | (2 * t4 + 9 < n ? 0xffff0000u : 0u);
          }
          const uint32_t vt = st + p * S::kPage + S::kTile;
#pragma unroll
          for (int c2 = 0; c2 < kNT / 2; ++c2) {
            uint32_t v0, v1, v2, v3;
            ldsm_x4_t(vt + swz(row, 2 * c2 + (lm >> 1)), v0, v1, v2, v3);
            if constexpr (decltype(masked)::value) {
              v0 &= klo;
              v1 &= khi;
              v2 &= klo;
              v3 &= khi;
            }
            M::run(o[2 * c2], ph[p][0], ph[p][1], ph[p][2], ph[p][3], v0, v1);
            M::run(o[2 * c2 + 1], ph[p][0], ph[p][1], ph[p][2], ph[p][3], v2, v3);
            M::run(o[2 * c2], pl[p][0], pl[p][1], pl[p][2], pl[p][3], v0, v1);
            M::run(o[2 * c2 + 1], pl[p][0], pl[p][1], pl[p][2], pl[p][3], v2, v3);
          }
        }
      };
      if (full)
        pv(std::false_type{});
      else
        pv(std::true_type{});
    }
    ring.release(c, a.num_kv_heads, kvh, &tmap_k, &tmap_v);
  }
  // every copy this CTA issued lands before the CTA exits
  if (__syncthreads_or(bad)) {
    ring.drain();
    return;
  }
#pragma unroll
  for (int msk = 1; msk <= 2; msk <<= 1) {
    lA += __shfl_xor_sync(kFull, lA, msk);
    lB += __shfl_xor_sync(kFull, lB, msk);
  }
  // rows A and B: d = 8 j + 2 t4, + 1 of every n-tile j
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int tr = e ? trB : trA;
    if (tr >= R) continue;
    const int pos = e ? posB : posA;
    const size_t row = out_row(tr);
    const float mm = e ? mB : mA, ll = e ? lB : lA;
    if (pos < tok0) {  // no key of this partition (or before position 0)
      if (direct)
#pragma unroll
        for (int j = 0; j < kNT; ++j)
          *reinterpret_cast<uint32_t*>(reinterpret_cast<T*>(a.out) + row * D + 8 * j + 2 * t4) = M::pack(0.f, 0.f);
      continue;
    }
    if (direct) {
      const float inv = 1.f / ll;
#pragma unroll
      for (int j = 0; j < kNT; ++j)
        *reinterpret_cast<uint32_t*>(reinterpret_cast<T*>(a.out) + row * D + 8 * j + 2 * t4) =
            M::pack(o[j][2 * e] * inv, o[j][2 * e + 1] * inv);
    } else {
      const size_t wrow = row * a.num_parts + z;
#pragma unroll
      for (int j = 0; j < kNT; ++j)
        *reinterpret_cast<float2*>(a.ws_o + wrow * D + 8 * j + 2 * t4) = make_float2(o[j][2 * e], o[j][2 * e + 1]);
      if (t4 == 0) a.ws_ml[wrow] = make_float2(mm, ll);
    }
  }
}

// Merge of the key partitions of the query rows of one (sequence b =
// blockIdx.x, kv-head blockIdx.y): the row at position pos uses partitions
// 0 .. pos / partition.  A sequence held by one partition was written by
// the partition kernel, so its CTA stops after reading the sequence's
// length.  Otherwise each warp merges whole rows (token, head) on its own:
// the partitions' common max, then their rescaled sums in partition order.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kMergeWarps * 32) paged_multi_merge_kernel(const MultiArgs a) {
  pdl_enter();
  const int b = blockIdx.x, kvh = blockIdx.y;
  int ctx, q0, nq;
  if (!multi_seq(a, b, ctx, q0, nq, false) || ctx <= a.partition) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kEpl = D / 32;
  constexpr int kRows = 8;  // rows a warp merges at once (their loads in flight together)
  const int rows = nq * G;
  for (int r0 = warp; r0 < rows; r0 += kMergeWarps * kRows) {
    size_t w0[kRows];
    int n[kRows];
    int nmax = 0;
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
      const int r = r0 + k * kMergeWarps;
      const int i = r / G;
      const int pos = ctx - nq + i;
      n[k] = r < rows && pos >= 0 ? pos / a.partition + 1 : 0;  // n = 0 writes zeros
      w0[k] = (static_cast<size_t>(q0 + i) * a.num_q_heads + kvh * G + r % G) * a.num_parts;
      nmax = max(nmax, n[k]);
    }
    float M[kRows];
#pragma unroll
    for (int k = 0; k < kRows; ++k) M[k] = -INFINITY;
    for (int p = lane; p < nmax; p += 32)
#pragma unroll
      for (int k = 0; k < kRows; ++k)
        if (p < n[k]) M[k] = fmaxf(M[k], a.ws_ml[w0[k] + p].x);
#pragma unroll
    for (int k = 0; k < kRows; ++k) M[k] = warp_max(M[k]);
    float acc[kRows][kEpl], den[kRows];
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
      den[k] = 0.f;
#pragma unroll
      for (int e = 0; e < kEpl; ++e) acc[k][e] = 0.f;
    }
    for (int p = 0; p < nmax; ++p) {
#pragma unroll
      for (int k = 0; k < kRows; ++k) {
        if (p >= n[k]) continue;
        const float2 v = a.ws_ml[w0[k] + p];
        const float w = exp2f(v.x - M[k]);
        den[k] = fmaf(w, v.y, den[k]);
        // this lane's kEpl (2 or 4) consecutive elements in one load
        const float* o = a.ws_o + (w0[k] + p) * D + lane * kEpl;
        if constexpr (kEpl == 4) {
          const float4 g = *reinterpret_cast<const float4*>(o);
          acc[k][0] = fmaf(w, g.x, acc[k][0]);
          acc[k][1] = fmaf(w, g.y, acc[k][1]);
          acc[k][2] = fmaf(w, g.z, acc[k][2]);
          acc[k][3] = fmaf(w, g.w, acc[k][3]);
        } else {
          const float2 g = *reinterpret_cast<const float2*>(o);
          acc[k][0] = fmaf(w, g.x, acc[k][0]);
          acc[k][1] = fmaf(w, g.y, acc[k][1]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
      const int r = r0 + k * kMergeWarps;
      if (r >= rows) continue;
      T* out = reinterpret_cast<T*>(a.out) + w0[k] / a.num_parts * D + lane * kEpl;
      const float inv = n[k] > 0 ? 1.f / den[k] : 0.f;
#pragma unroll
      for (int e = 0; e < kEpl; ++e) out[e] = Fmt<T>::from_f32(acc[k][e] * inv);
    }
  }
}

}  // namespace pkv
