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
// Work split: one CTA per (kv-head, sequence, tile of 16 query rows,
// partition of keys).  A tile's rows are (token, head) pairs of one
// kv-head: row r is token r / G, head r % G of the group, so one tile
// covers 16 / G tokens and every K/V tile of the sequence is read once per
// kv-head and row tile.  Within the CTA, warp w walks pages w, w + NWARPS,
// ... of the partition with its own ring of TMA-staged tiles (as in the
// decode kernel) and keeps all 16 rows' state; the warps' states are merged
// in a fixed order at the end.  Per page:
//   S[16 rows x 16 tokens] = Q[16 x D] . K^T   (A = Q in registers,
//                                               B = K via ldmatrix)
//   causal mask: token j of row r counts when j <= pos(r)
//   O[16 x D] += P . V                           (A = P from the S
//                                               fragments, hi + lo parts,
//                                               B = V via ldmatrix.trans)
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
  float qk_scale; // scale * log2(e)
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

template <typename T, int D, int G, int NWARPS, int NSTAGE>
__global__ void __launch_bounds__(NWARPS * 32)
    paged_multi_mma_kernel(const MultiArgs a, const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_v) {
  pdl_enter();
  using S = MmaShape<T, D, G, NWARPS, NSTAGE>;
  using M = Mma<T>;
  constexpr int kNTiles = D / 8;  // PV n-tiles (8 columns of d each)
  constexpr int kRec = 16 * D;    // warp record: o[16][D], m[16], l[16]
  static_assert(size_t(kRec + 32) * sizeof(float) <= size_t(S::kWarpStageBytes),
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
  const int R = nq * G;      // rows of this kv-head
  const int r0 = tile * 16;  // first row of the tile
  if (r0 >= R) return;
  const int base = ctx - nq;  // position of new token 0
  const int p_hi = base + (min(R, r0 + 16) - 1) / G;
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
      for (int idx = threadIdx.x; idx < 16 * D; idx += NWARPS * 32) {
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

  // A fragments of the tile's rows g8 and g8 + 8 (zero past the rows), and
  // their positions (-1: sees no key)
  const int ra = r0 + g8, rb = r0 + g8 + 8;
  const int posA = ra < R ? base + ra / G : -1;
  const int posB = rb < R ? base + rb / G : -1;
  uint32_t qa[S::kKSteps][4];
  {
    const T* pa = ra < R ? reinterpret_cast<const T*>(a.q) + out_row(ra) * D : nullptr;
    const T* pb = rb < R ? reinterpret_cast<const T*>(a.q) + out_row(rb) * D : nullptr;
#pragma unroll
    for (int ks = 0; ks < S::kKSteps; ++ks) {
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
  float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
  int consumed = 0;
  bool timed_out = false;

  for (int i = 0; i < my_n; ++i) {
    const int s = i % NSTAGE;
    bool ok = mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
    phase_bits ^= 1u << s;
    ok = __all_sync(kFull, ok);
    if (!ok) {
      if (lane == 0) raise_error(PKV_ERR_TIMEOUT);
      timed_out = true;
      break;
    }
    consumed = i + 1;
    if (phys_of(i) >= 0) {
      const int page_tok = tok0 + (warp + i * NWARPS) * kBlockSize;
      const int nvalid = min(kBlockSize, tok1 - page_tok);
      const uint32_t kt = stage0 + s * S::kStage;
      const uint32_t vt = kt + S::kTile;
      // (1) S = Q . K^T
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
      // (2) scale, causal mask, online softmax per row
      float x[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = page_tok + nt * 8 + 2 * t4 + (e & 1);
          x[nt][e] = j <= (e < 2 ? posA : posB) ? sc[nt][e] * a.qk_scale : -INFINITY;
        }
      float mxA = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
      float mxB = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
#pragma unroll
      for (int msk = 1; msk <= 2; msk <<= 1) {
        mxA = fmaxf(mxA, __shfl_xor_sync(kFull, mxA, msk));
        mxB = fmaxf(mxB, __shfl_xor_sync(kFull, mxB, msk));
      }
      const float nA = fmaxf(mA, mxA), nB = fmaxf(mB, mxB);
      // a row that has seen no key yet keeps max -inf: subtract 0 instead
      const float uA = nA == -INFINITY ? 0.f : nA, uB = nB == -INFINITY ? 0.f : nB;
      const float alA = exp2f(mA - uA), alB = exp2f(mB - uB);
      mA = nA;
      mB = nB;
      float p[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        p[nt][0] = exp2f(x[nt][0] - uA);
        p[nt][1] = exp2f(x[nt][1] - uA);
        p[nt][2] = exp2f(x[nt][2] - uB);
        p[nt][3] = exp2f(x[nt][3] - uB);
      }
      lA = fmaf(lA, alA, p[0][0] + p[0][1] + p[1][0] + p[1][1]);
      lB = fmaf(lB, alB, p[0][2] + p[0][3] + p[1][2] + p[1][3]);
      if (__any_sync(kFull, alA != 1.f || alB != 1.f)) {
#pragma unroll
        for (int j = 0; j < kNTiles; ++j) {
          o[j][0] *= alA;
          o[j][1] *= alA;
          o[j][2] *= alB;
          o[j][3] *= alB;
        }
      }
      // (3) P as A fragments, hi + lo 16-bit parts
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
      // V fragment halves of tokens past the visible range are zeroed (an
      // unwritten slot may hold NaN, and 0 * NaN is NaN)
      uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
      if (nvalid < kBlockSize) {
        keep_lo = (2 * t4 < nvalid ? 0x0000ffffu : 0u) | (2 * t4 + 1 < nvalid ? 0xffff0000u : 0u);
        keep_hi = (2 * t4 + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * t4 + 9 < nvalid ? 0xffff0000u : 0u);
      }
      // (4) O += P . V
      {
        const int row = lr + ((lm & 1) << 3);  // token
#pragma unroll
        for (int j = 0; j < kNTiles; j += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vt + swz(row, j + (lm >> 1)), b0, b1, b2, b3);
          b0 &= keep_lo;
          b1 &= keep_hi;
          b2 &= keep_lo;
          b3 &= keep_hi;
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
  if (consumed < my_n) {  // after a give-up: wait (bounded) for copies in flight
    const int last = min(my_n, consumed + NSTAGE);
    for (int i = consumed + 1; i < last; ++i) {
      const int s = i % NSTAGE;
      mbar_wait_bounded(bar0 + 8 * s, (phase_bits >> s) & 1u);
      phase_bits ^= 1u << s;
    }
  }
#pragma unroll
  for (int msk = 1; msk <= 2; msk <<= 1) {
    lA += __shfl_xor_sync(kFull, lA, msk);
    lB += __shfl_xor_sync(kFull, lB, msk);
  }

  // warp record [o: 16 x D][m: 16][l: 16] in the warp's own (drained) stages
  float* rec = reinterpret_cast<float*>(my_stages);
#pragma unroll
  for (int j = 0; j < kNTiles; ++j) {
    const int d = 8 * j + 2 * t4;
    *reinterpret_cast<float2*>(rec + g8 * D + d) = make_float2(o[j][0], o[j][1]);
    *reinterpret_cast<float2*>(rec + (g8 + 8) * D + d) = make_float2(o[j][2], o[j][3]);
  }
  if (t4 == 0) {
    rec[kRec + g8] = mA;
    rec[kRec + g8 + 8] = mB;
    rec[kRec + 16 + g8] = lA;
    rec[kRec + 16 + g8 + 8] = lB;
  }
  if (__syncthreads_or(timed_out)) return;

  // merge the warps in a fixed order; rows with no key in this partition
  // are left to the other partitions (the merge never reads them)
  for (int idx = threadIdx.x; idx < 16 * D; idx += NWARPS * 32) {
    const int r = idx / D, d = idx % D;
    const int tr = r0 + r;
    if (tr >= R) continue;
    const int pos = base + tr / G;
    const size_t row = out_row(tr);
    if (pos < tok0) {
      if (direct) reinterpret_cast<T*>(a.out)[row * D + d] = Fmt<T>::from_f32(0.f);
      continue;
    }
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w)
      Mx = fmaxf(Mx, reinterpret_cast<const float*>(smem + w * S::kWarpStageBytes)[kRec + r]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) {
      const float* rw = reinterpret_cast<const float*>(smem + w * S::kWarpStageBytes);
      const float sc = exp2f(rw[kRec + r] - Mx);
      num = fmaf(sc, rw[r * D + d], num);
      den = fmaf(sc, rw[kRec + 16 + r], den);
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

// Merge of the key partitions of each query row (token t = blockIdx.x, HPC
// heads per CTA from head blockIdx.y * HPC): the row at position pos uses
// partitions 0 .. pos / partition.
// Sequences held by one partition were written by the partition kernel.
template <typename T, int D, int HPC>
__global__ void __launch_bounds__(kMergeWarps * 32) paged_multi_merge_kernel(const MultiArgs a) {
  pdl_enter();
  const int hs = (threadIdx.x >> 5) / (kMergeWarps / HPC);
  const int h = blockIdx.y * HPC + hs;
  const int t = blockIdx.x;
  // the sequence of row t: last b with query_start[b] <= t
  int lo = 0, hi = a.num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.query_start[mid] <= t)
      lo = mid;
    else
      hi = mid - 1;
  }
  const int b = lo;
  int ctx, q0, nq;
  const bool ok = multi_seq(a, b, ctx, q0, nq, false) && t >= q0 && t < q0 + nq;
  const bool direct = ctx <= a.partition;
  const bool skip = !ok || direct;
  if (__syncthreads_and(skip)) return;  // uniform: same row t for the whole CTA
  const int pos = ctx - nq + (t - q0);
  const bool head_ok = h < a.num_q_heads;
  const int hh = head_ok ? h : 0;
  const size_t row = static_cast<size_t>(t) * a.num_q_heads + hh;
  __shared__ T sink[D];
  T* out = head_ok ? reinterpret_cast<T*>(a.out) + row * D : sink;
  const int n = (head_ok && pos >= 0) ? pos / a.partition + 1 : 0;  // n = 0 writes zeros
  const size_t w0 = row * a.num_parts;
  merge_partials<T, D, HPC>(
      n, [&](int p) { return a.ws_ml[w0 + p]; }, [&](int p) { return a.ws_o + (w0 + p) * D; }, out, hs);
}

}  // namespace pkv
