/*
 * pkv.h -- C ABI of the paged KV-cache decode library (libpkv.so).
 *
 * The KV cache of every sequence is kept in fixed 16-token blocks drawn from
 * one shared pool and reached through a per-sequence block table (logical
 * page n -> physical block), so a sequence never needs contiguous memory and
 * grows one block at a time ("PagedAttention 与 vLLM 推理加速" §2.2-§2.3;
 * "vLLM + PagedAttention：打造高并发LLM推理引擎", "它是怎么工作的").
 *
 * Device entry points take plain device pointers to memory the caller owns
 * (the library never allocates device memory) and enqueue work on the given
 * stream (a cudaStream_t passed as void*; NULL = the legacy default stream).
 * They return after the launch, not after the work.  Every argument the host
 * can check is checked before anything is launched; a bad one returns
 * PKV_EINVAL and launches nothing.  Values that live on the device (block
 * ids in tables, slots, context lengths, copy pairs) are range-checked inside
 * the kernels: an out-of-range value is never dereferenced, the work that
 * needed it is skipped, and a bit is set in the device error word that
 * pkv_get_error() reads back.
 *
 * Layouts (all row-major, contiguous):
 *   q, out            [num_seqs, num_q_heads, head_dim]            dtype
 *   k_new, v_new      [num_tokens, num_kv_heads, head_dim]         dtype
 *   k_cache, v_cache  [num_blocks, num_kv_heads, 16, head_dim]     dtype
 *   block_tables      [num_seqs, max_blocks_per_seq]               int32
 *   context_lens      [num_seqs]                                   int32
 *   slot_mapping      [num_tokens]                                 int64
 *   copy pairs        [num_pairs, 2] = (src, dst)                  int32
 * A slot names one token position of the pool: slot = block * 16 + offset.
 * Query head h reads kv-head h / (num_q_heads / num_kv_heads).
 *
 * Supported: head_dim 64 or 128; dtype fp32, fp16, bf16 (K, V, q and out
 * share it); num_q_heads / num_kv_heads in {1, 2, 4, 8}.  Device pointers
 * must be 16-byte aligned.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PKV_BLOCK_SIZE 16
#define PKV_DEFAULT_PARTITION 512

/* PKV_E4M3: FP8 E4M3 codes (one byte) of an FP8 cache; see
 * pkv_kv_append_fp8.  Byte copies (pkv_kv_append of codes, pkv_copy_blocks,
 * pkv_swap_blocks) take it like the others; attention over an FP8 cache is
 * pkv_paged_attention_decode_fp8. */
typedef enum { PKV_F32 = 0, PKV_F16 = 1, PKV_BF16 = 2, PKV_E4M3 = 3 } pkv_dtype;

typedef enum {
  PKV_OK = 0,
  PKV_EINVAL = 1, /* a bad argument; nothing launched, no state changed */
  PKV_ENOMEM = 2, /* allocator: the pool cannot serve the call; no state changed */
  PKV_ECUDA = 3   /* a CUDA runtime call or launch failed */
} pkv_status;

/* Bits of the device error word (pkv_get_error). */
#define PKV_ERR_BLOCK_RANGE 0x1u   /* a block-table entry inside a sequence's pages is outside [0, num_blocks) */
#define PKV_ERR_CONTEXT_RANGE 0x2u /* a context length < 0, > max_context_len or > 16 * max_blocks_per_seq (clamped) */
#define PKV_ERR_SLOT_RANGE 0x4u    /* an append slot names a block outside the pool (the write is skipped) */
#define PKV_ERR_COPY_RANGE 0x8u    /* a copy pair names a block outside the pool (the copy is skipped) */
#define PKV_ERR_TIMEOUT 0x10u      /* a staging wait gave up after its time limit */

/* Static description of a status code. */
const char* pkv_status_string(pkv_status status);

/* ABI version of this header (increases when a signature changes). */
int pkv_abi_version(void);

/* ------------------------------------------------------------------------
 * pkv_kv_append -- slot-mapped write of new tokens' K/V into the pool.
 *
 * "vLLM + PagedAttention：打造高并发LLM推理引擎", "它是怎么工作的" (items 2
 * and 3): each request's page table records which block its n-th token is
 * in; a growing sequence writes its new token into that slot and never
 * moves old data.
 *
 * For every token i with slot_mapping[i] >= 0:
 *   k_cache[slot / 16, h, slot % 16, :] = k_new[i, h, :]   (all h; V alike)
 * A negative slot is padding and writes nothing.  Slots must be distinct
 * within one call (two tokens writing one slot race).  Bit copy: the stored
 * bytes equal the input bytes.  A slot whose block is >= num_blocks is
 * skipped and sets PKV_ERR_SLOT_RANGE.
 * -------------------------------------------------------------------- */
pkv_status pkv_kv_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int num_blocks, pkv_dtype dtype, void* stream);

/* ------------------------------------------------------------------------
 * pkv_copy_blocks -- copy-on-write block copy.
 *
 * "PagedAttention 与 vLLM 推理加速" §3.2(3) and "LLM Systems 24: Efficient
 * LLM Inference with PagedAttention and vLLM" §3: a block shared by several
 * sequences is never copied while it is only read; before a sequence writes
 * into it, the block is copied to a fresh block that the writer then owns.
 *
 * For each pair (src, dst) in pairs[num_pairs][2] (device memory):
 *   k_cache[dst] = k_cache[src];  v_cache[dst] = v_cache[src]
 * (all num_kv_heads * 16 * head_dim elements; bit copy).  The dst values must
 * be distinct and no dst may also be a src of the same call (otherwise the
 * result depends on the order of the copies); pkv_copy_blocks_check verifies
 * this on a host copy of the pairs.  A pair naming a block outside
 * [0, num_blocks) is skipped and sets PKV_ERR_COPY_RANGE.
 * -------------------------------------------------------------------- */
pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int num_pairs,
                           int num_kv_heads, int head_dim, int num_blocks, pkv_dtype dtype,
                           void* stream);

/* Host-side check of copy pairs (host memory): every id in range, dst ids
 * distinct, no dst equal to any src.  PKV_OK or PKV_EINVAL. */
pkv_status pkv_copy_blocks_check(const int32_t* pairs_host, int num_pairs, int num_blocks);

/* ------------------------------------------------------------------------
 * pkv_kv_append_copy -- a decode step's copy-on-write copies and append in
 * one launch, each copy cut to the rows that hold tokens.
 *
 * "PagedAttention 与 vLLM 推理加速" §3.2(3): a shared, partially filled
 * block is copied before a sharer appends into it.  Only its first rows
 * hold tokens; the rows past them are never read.  For each copy
 * (src, dst, rows) in copies[num_copies][3] (device):
 *   k_cache[dst, :, r, :] = k_cache[src, :, r, :]  for r < rows   (V alike)
 * and for every token i with slot_mapping[i] >= 0 the write of
 * pkv_kv_append.  rows must not exceed the first row a token of this call
 * writes into dst (then copies and appends touch disjoint rows; the result
 * on every row below dst's first unwritten row equals pkv_copy_blocks
 * followed by pkv_kv_append); rows of dst past the appended ones keep what
 * they held.  Layouts, bit-exactness and the slot rules as pkv_kv_append;
 * a copy naming a block outside [0, num_blocks), or rows > 16, is skipped
 * and sets PKV_ERR_COPY_RANGE.
 * -------------------------------------------------------------------- */
pkv_status pkv_kv_append_copy(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                              const int64_t* slot_mapping, int num_tokens, const int32_t* copies, int num_copies,
                              int num_kv_heads, int head_dim, int num_blocks, pkv_dtype dtype, void* stream);

/* ------------------------------------------------------------------------
 * pkv_swap_blocks -- block copy between two pools (preemption by swapping).
 *
 * "LLM Systems 24: Efficient LLM Inference with PagedAttention and vLLM" §3
 * (conclusion): when the pool runs out of KV blocks a request is preempted;
 * its blocks are swapped out to host memory and later swapped back in.
 *
 * For each pair (src, dst) in pairs[num_pairs][2]:
 *   dst_k[dst] = src_k[src];  dst_v[dst] = src_v[src]
 * (all num_kv_heads * 16 * head_dim elements; bit copy).  Both pools have
 * the layout [blocks, num_kv_heads, 16, head_dim] of one dtype; the source
 * has src_blocks blocks, the destination dst_blocks.  Each of the four
 * cache pointers and `pairs` may be device memory of the current device
 * or page-locked host memory mapped into the device's address space
 * (cudaHostAlloc / cudaMallocHost, or cudaHostRegister'ed memory); pageable
 * host memory, another device's memory or an unknown pointer returns
 * PKV_EINVAL.  The pairs pkv_alloc_swap_out / pkv_alloc_swap_in report are
 * (device, host) and (host, device) pairs for this call.  dst values must
 * be distinct (pkv_swap_blocks_check) and the two pools must not overlap.
 * A pair outside [0, src_blocks) x [0, dst_blocks) is skipped and sets
 * PKV_ERR_COPY_RANGE.  Host memory is read or written by the kernel while
 * it runs: keep it allocated and untouched by the host until the stream
 * has passed the call.
 * -------------------------------------------------------------------- */
pkv_status pkv_swap_blocks(void* dst_k, void* dst_v, int dst_blocks, const void* src_k, const void* src_v,
                           int src_blocks, const int32_t* pairs, int num_pairs, int num_kv_heads,
                           int head_dim, pkv_dtype dtype, void* stream);

/* Host-side check of swap pairs (host memory): src in [0, src_blocks), dst
 * in [0, dst_blocks), dst ids distinct.  PKV_OK or PKV_EINVAL. */
pkv_status pkv_swap_blocks_check(const int32_t* pairs_host, int num_pairs, int src_blocks, int dst_blocks);


/* ------------------------------------------------------------------------
 * pkv_decode_workspace_bytes -- device workspace pkv_paged_attention_decode
 * needs for these sizes (0 when no sequence can span two partitions).
 * partition_tokens: 0 = auto (PKV_DEFAULT_PARTITION = 512 tokens, or 1024
 * when max_context_len > 4096), else a multiple of 16 in [16, 2048].
 * Returns 0 for arguments pkv_paged_attention_decode rejects.
 *
 * Workspace layout (fp32): partial outputs [num_seqs][num_q_heads][P][head_dim]
 * followed by (running max, running sum) pairs [num_seqs][num_q_heads][P][2],
 * P = ceil(max_context_len / partition_tokens).
 * -------------------------------------------------------------------- */
size_t pkv_decode_workspace_bytes(int num_seqs, int num_q_heads, int head_dim,
                                  int max_context_len, int partition_tokens);

/* ------------------------------------------------------------------------
 * pkv_paged_attention_decode -- single-query attention of every sequence
 * over its paged K/V.
 *
 * "PagedAttention 与 vLLM 推理加速" §2.3: the kernel walks the sequence's
 * blocks through its block table and takes Q (the current token) x K over
 * every key in them to get the attention scores; §1: each decode step
 * attends over the K/V of every token so far, the current one included
 * (context_lens count the token just appended).  With n = context_lens[b]
 * and g = h / (num_q_heads / num_kv_heads):
 *   K_j = k_cache[block_tables[b][j / 16], g, j % 16, :]   (V_j alike)
 *   s_j = scale * <q[b,h,:], K_j>,   j < n
 *   out[b,h,:] = sum_j softmax(s)_j V_j     (zeros when n == 0)
 * computed in fp32 and rounded once to dtype.  Entries of block_tables past
 * page ceil(n/16) - 1 and the unused slots of the last block are never read.
 *
 * Work is split into partitions of partition_tokens tokens (0 = auto: 512,
 * or 1024 when max_context_len > 4096; else a multiple of 16 in [16, 2048]); each (sequence, kv-head, partition) keeps
 * the running max and sum of its exponentials and a partial output, and a
 * second kernel merges the partitions of sequences longer than one
 * partition by rescaling each to the overall max (log-sum-exp merge).  The
 * summation order depends only on logical token positions, so the output
 * is bit-identical under any relabelling of physical blocks.
 *
 * max_context_len: a host-side bound on context_lens (sizes the grid and the
 *   workspace); max_context_len <= 16 * max_blocks_per_seq.
 * workspace: device scratch of at least pkv_decode_workspace_bytes(...)
 *   bytes, 16-byte aligned (may be NULL when that is 0).  Its contents need
 *   no initialisation and are garbage afterwards.  Two calls that overlap
 *   on the GPU must not share a workspace.
 * -------------------------------------------------------------------- */
pkv_status pkv_paged_attention_decode(void* out, const void* q, const void* k_cache,
                                      const void* v_cache, const int32_t* block_tables,
                                      int max_blocks_per_seq, const int32_t* context_lens,
                                      int max_context_len, int num_seqs, int num_q_heads,
                                      int num_kv_heads, int head_dim, int num_blocks,
                                      float scale, int partition_tokens, pkv_dtype dtype,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * pkv_paged_attention_decode_prefix -- pkv_paged_attention_decode for a
 * batch whose sequences share a common prefix of blocks (cascade decode).
 *
 * "PagedAttention 与 vLLM 推理加速" §3.2(3): requests with the same system
 * prompt map the same physical blocks, stored once.  Here those blocks are
 * also READ once per kv-head: a prefix pass attends the queries of every
 * sequence to each shared (block, kv-head) tile on the tensor cores, the
 * paged pass covers each sequence's own suffix, and a merge kernel combines
 * the two partial results by the log-sum-exp rule.  The output is the same
 * attention as pkv_paged_attention_decode (up to fp32 rounding order).
 *
 * prefix_blocks (device, int32 [prefix_pages]): the shared blocks, in
 *   logical order.  Sequence b "conforms" when its first prefix_pages table
 *   entries equal them and context_lens[b] >= 16 * prefix_pages (all prefix
 *   pages full).  This is checked on the device; a sequence that does not
 *   conform is decoded over its whole context instead (still correct).
 * dtype: PKV_F16 or PKV_BF16 (tensor-core path); 1 <= prefix_pages <=
 *   max_blocks_per_seq; the other arguments are those of
 *   pkv_paged_attention_decode.
 * workspace: at least pkv_decode_prefix_workspace_bytes(...) bytes, 16-byte
 *   aligned, always required; no initialisation needed.
 * An out-of-range id in prefix_blocks sets PKV_ERR_BLOCK_RANGE and that
 * page is skipped.
 * -------------------------------------------------------------------- */
size_t pkv_decode_prefix_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                         int prefix_pages, int partition_tokens);
pkv_status pkv_paged_attention_decode_prefix(void* out, const void* q, const void* k_cache,
                                             const void* v_cache, const int32_t* block_tables,
                                             int max_blocks_per_seq, const int32_t* context_lens,
                                             int max_context_len, const int32_t* prefix_blocks,
                                             int prefix_pages, int num_seqs, int num_q_heads,
                                             int num_kv_heads, int head_dim, int num_blocks, float scale,
                                             int partition_tokens, pkv_dtype dtype, void* workspace,
                                             size_t workspace_bytes, void* stream);

/* The same cascade launched in phases, so that the prefix pass can run on
 * another stream beside the step's copy-on-write copies and append (which
 * never write a full, shared prefix block):
 *   phase 0: the prefix pass (reads q and the prefix blocks; writes the
 *            prefix partials of the workspace);
 *   phase 1: the suffix pass (reads the tables, lengths and suffix blocks
 *            after this step's append; writes the suffix partials and the
 *            per-sequence conformity flags);
 *   phase 2: the merge (needs phases 0 and 1 complete; writes out).
 * All three take the arguments of pkv_paged_attention_decode_prefix and the
 * same workspace; ordering between streams is the caller's (an event from
 * the phase-0 stream before phase 2).  The result is bit-identical to
 * pkv_paged_attention_decode_prefix.  PKV_EINVAL for another phase. */
pkv_status pkv_paged_attention_decode_prefix_phase(void* out, const void* q, const void* k_cache,
                                                   const void* v_cache, const int32_t* block_tables,
                                                   int max_blocks_per_seq, const int32_t* context_lens,
                                                   int max_context_len, const int32_t* prefix_blocks,
                                                   int prefix_pages, int num_seqs, int num_q_heads,
                                                   int num_kv_heads, int head_dim, int num_blocks, float scale,
                                                   int partition_tokens, pkv_dtype dtype, void* workspace,
                                                   size_t workspace_bytes, int phase, void* stream);

/* ------------------------------------------------------------------------
 * pkv_decode_step -- one whole decode step in one launch (plus the merge):
 * the step's copy-on-write copies and append, then the decode.
 *
 * "PagedAttention 与 vLLM 推理加速" §3.2(3) (a shared partial block is copied
 * before a sharer appends into it), "vLLM + PagedAttention：打造高并发LLM
 * 推理引擎", "它是怎么工作的" (the new token goes into its slot; the kernel
 * then reads every block through the table) and §2.3 of the former.  The
 * result -- the pool and out -- is that of
 *   pkv_kv_append_copy(k_new, v_new, ..., slot_mapping, num_seqs, copies, ...)
 * followed by pkv_paged_attention_decode (prefix_pages == 0) or
 * pkv_paged_attention_decode_prefix (prefix_pages > 0, the cascade).
 * Without a prefix the writes are made inside the decode launch: for each
 * sequence b and kv-head, the CTA that reads the sequence's last page first
 * copies rows 0 .. rows-1 of the copy (src, dst, rows) whose dst is
 * slot_mapping[b]'s block, then writes k_new[b] / v_new[b] into the slot,
 * then stages the page -- so the step needs no separate copy / append
 * launch and the copies overlap the streaming of other sequences.  With a
 * prefix the copies and the append are one launch of their own
 * (pkv_kv_append_copy), which the cascade launch does not wait for except
 * where it reads what they write: the warp that stages a sequence's last
 * page waits for it (programmatic dependent launch) just before that page,
 * while the prefix pass and the other pages stream.
 *
 * One new token per sequence: k_new, v_new [num_seqs, num_kv_heads,
 * head_dim] in dtype; slot_mapping int64 [num_seqs] (< 0: no token);
 * context_lens count the new token.  copies int32 [num_copies][3] (device,
 * num_copies <= num_seqs), as pkv_cow_copy_rows makes them from the
 * allocator's step: every dst is the block of one slot of this call, and
 * rows does not pass that slot's row.  The slots must not write into the
 * shared prefix blocks (an allocator's step never does: a shared block is
 * copied first).  dtype PKV_F16 or PKV_BF16; the other arguments, the
 * workspace (pkv_decode_workspace_bytes, or pkv_decode_prefix_workspace_bytes
 * when prefix_pages > 0) and the errors are those of the two calls.
 * -------------------------------------------------------------------- */
pkv_status pkv_decode_step(void* out, const void* q, void* k_cache, void* v_cache, const void* k_new,
                           const void* v_new, const int64_t* slot_mapping, const int32_t* copies, int num_copies,
                           const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                           int max_context_len, const int32_t* prefix_blocks, int prefix_pages, int num_seqs,
                           int num_q_heads, int num_kv_heads, int head_dim, int num_blocks, float scale,
                           int partition_tokens, pkv_dtype dtype, void* workspace, size_t workspace_bytes,
                           void* stream);

/* ------------------------------------------------------------------------
 * pkv_paged_attention_decode_static_ws -- pkv_paged_attention_decode for
 * callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call; it exists for library users.
 * Some callers must not call cudaMalloc: code running under a framework's
 * caching allocator that has already reserved the GPU's memory (a raw
 * cudaMalloc can fail there, or fragment the pool), and code on a
 * latency-critical path, where cudaMalloc/cudaFree may synchronise the
 * device.  Such a caller has no way to provide the split-K workspace that
 * pkv_paged_attention_decode needs for contexts longer than one partition.
 *
 * This variant takes the same arguments minus the workspace and uses a
 * fixed scratch area of PKV_STATIC_WORKSPACE_BYTES that the library itself
 * holds in device memory: every GPU that loads libpkv.so keeps that much
 * memory until the process exits.  It allocates nothing.
 *   - If pkv_decode_workspace_bytes(...) for the call exceeds
 *     PKV_STATIC_WORKSPACE_BYTES, it returns PKV_EINVAL and launches nothing
 *     (use pkv_paged_attention_decode with a caller-owned workspace then).
 *   - The first call on a device looks up that device's address of the
 *     scratch area (a runtime query, no allocation), with the caller's
 *     current device; make that first call before any stream capture.  The
 *     address is kept per device and per context (by the context's unique
 *     id): after the caller destroys and re-creates the device's context
 *     (cudaDeviceReset, or a primary-context reset), the next call looks it
 *     up again, so that call too belongs before any capture.
 *   - All calls on a device share the one scratch area, and it keeps what
 *     the previous call left in it.  The decode writes every scratch value
 *     before it reads it, so nothing needs clearing between calls, but two
 *     calls whose work overlaps on the GPU (different streams without
 *     ordering between them) race on the scratch area.
 * Other arguments, results and errors are those of pkv_paged_attention_decode.
 * -------------------------------------------------------------------- */
#define PKV_STATIC_WORKSPACE_BYTES (16u << 20)
pkv_status pkv_paged_attention_decode_static_ws(void* out, const void* q, const void* k_cache,
                                                const void* v_cache, const int32_t* block_tables,
                                                int max_blocks_per_seq, const int32_t* context_lens,
                                                int max_context_len, int num_seqs, int num_q_heads,
                                                int num_kv_heads, int head_dim, int num_blocks,
                                                float scale, int partition_tokens, pkv_dtype dtype,
                                                void* stream);

/* Read and clear the current device's error word (PKV_ERR_* bits) after the
 * work queued on `stream` so far has finished.  Blocks the host. */
pkv_status pkv_get_error(uint32_t* flags, void* stream);

/* Test hook for the kernels' failure path.  Every wait of a kernel on its
 * staged copies (an mbarrier the TMA completes) is bounded: after 2^32 SM
 * clock cycles (about 2 s) the kernel sets PKV_ERR_TIMEOUT, drains what it
 * issued with bounded waits and returns, leaving the context usable.  This
 * call runs that same wait, with limit_cycles in [1, 2^32] as its bound, on
 * a barrier that nothing completes (one warp, one CTA, async on `stream`):
 * pkv_get_error then reports PKV_ERR_TIMEOUT.  PKV_EINVAL for a limit out of
 * range. */
pkv_status pkv_selftest_bounded_wait(long long limit_cycles, void* stream);

/* ------------------------------------------------------------------------
 * FP8 KV cache: half the bytes of a 16-bit cache per token.
 *
 * The pages name FP8 only as a low-precision format of TensorRT-LLM's
 * operators ("vLLM 推理加速：PagedAttention、FlashAttention 与动态批处理",
 * "TensorRT-LLM"); the format and the scaling are this library's choice:
 * OCP FP8 E4M3 (bias 7, subnormals, max 448, no infinities) with one float
 * scale for all of K and one for all of V.  The pool layout is that of a
 * 16-bit cache with one-byte elements: [num_blocks, num_kv_heads, 16,
 * head_dim] uint8 codes; a stored value is code's value * scale.
 *
 * pkv_kv_append_fp8: for every token i with slot_mapping[i] >= 0,
 *   k_cache[slot / 16, h, slot % 16, d] = E4M3(k_new[i, h, d] / k_scale)
 * (V alike with v_scale): k_new / v_new in src_dtype (fp16 or bf16), the
 * division in float32 (IEEE, round to nearest), then round to the nearest
 * E4M3 value, ties to even, magnitudes past 448 saturating to +-448.  Codes
 * are bit-exact.  Slot rules and errors as pkv_kv_append.  Scales must be
 * finite and > 0.
 *
 * pkv_paged_attention_decode_fp8: pkv_paged_attention_decode over an FP8
 * cache; q and out in q_dtype (fp16 or bf16);
 *   s_j = scale * k_scale * q . code(K_j),  out = v_scale * sum_j softmax(s)_j code(V_j)
 * Same arguments, layouts, workspace (pkv_decode_workspace_bytes) and errors
 * as pkv_paged_attention_decode, except the auto partition (partition_tokens
 * 0): 768 tokens, 1024 when max_context_len > 4096, 2048 when it is
 * > 16384 (an FP8 page is half the bytes, so a work unit covers more tokens
 * for the same fixed cost).  A workspace sized by pkv_decode_workspace_bytes
 * with partition 0 is large enough for it.
 * -------------------------------------------------------------------- */
pkv_status pkv_kv_append_fp8(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                             int num_blocks, pkv_dtype src_dtype, float k_scale, float v_scale, void* stream);
pkv_status pkv_paged_attention_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                                          const int32_t* block_tables, int max_blocks_per_seq,
                                          const int32_t* context_lens, int max_context_len, int num_seqs,
                                          int num_q_heads, int num_kv_heads, int head_dim, int num_blocks,
                                          float scale, float k_scale, float v_scale, int partition_tokens,
                                          pkv_dtype q_dtype, void* workspace, size_t workspace_bytes,
                                          void* stream);

/* pkv_decode_step_fp8 -- pkv_decode_step over an FP8 cache: the step's
 * copy-on-write copies, the quantised append of the new token and the
 * decode, with no launch of their own for the copies and the append.
 *
 * Same passages as pkv_decode_step.  The result -- the pool and out -- is
 * that of pkv_kv_append_copy's copies (whole rows of codes), then
 * pkv_kv_append_fp8(k_new, v_new, ..., k_scale, v_scale), then
 * pkv_paged_attention_decode_fp8 (prefix_pages == 0) or
 * pkv_paged_attention_decode_prefix_fp8 (prefix_pages > 0): the CTA that
 * reads a sequence's last page (in the cascade: of its suffix pass) first
 * copies rows 0 .. rows-1 of the copy whose dst is slot_mapping[b]'s block,
 * then writes the token's codes (E4M3(x / scale), as pkv_kv_append_fp8
 * rounds them), then stages the page.  The slots must not write into the
 * shared prefix blocks (an allocator's step never does).
 * k_new, v_new [num_seqs, num_kv_heads, head_dim] in q_dtype (fp16 or
 * bf16); slot_mapping int64 [num_seqs] (< 0: no token); copies int32
 * [num_copies][3] (device, num_copies <= num_seqs) as for pkv_decode_step.
 * The other arguments, the workspace (pkv_decode_workspace_bytes, or
 * pkv_decode_prefix_fp8_workspace_bytes when prefix_pages > 0) and the
 * errors are those of the FP8 decode called and of pkv_decode_step.
 * -------------------------------------------------------------------- */
pkv_status pkv_decode_step_fp8(void* out, const void* q, void* k_cache, void* v_cache, const void* k_new,
                               const void* v_new, const int64_t* slot_mapping, const int32_t* copies, int num_copies,
                               const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                               int max_context_len, const int32_t* prefix_blocks, int prefix_pages, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int num_blocks, float scale,
                               float k_scale, float v_scale, int partition_tokens, pkv_dtype q_dtype, void* workspace,
                               size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * pkv_paged_attention_decode_prefix_fp8 -- the shared-prefix (cascade)
 * decode of pkv_paged_attention_decode_prefix over an FP8 cache.
 *
 * "PagedAttention 与 vLLM 推理加速" §3.2(3): sequences with one system prompt
 * share its blocks; here an FP8 pool's shared prefix is read once per
 * kv-head too.  Same result as pkv_paged_attention_decode_fp8 (up to fp32
 * rounding order):
 *   s_j = scale * k_scale * q . code(K_j),  out = v_scale * sum_j softmax(s)_j code(V_j).
 * The call converts the prefix tiles to their exact 16-bit code values in
 * the workspace (every E4M3 value is an fp16 and a bf16 value), runs the
 * cascade's prefix pass over them on the 16-bit tensor-core path, the
 * suffix pass over the FP8 cache, and the cascade's merge.  Sequences that
 * do not start with the prefix, or whose context does not cover it, are
 * decoded over their whole context (checked on the device).  Arguments as
 * pkv_paged_attention_decode_prefix, with the scales of
 * pkv_paged_attention_decode_fp8; q and out in q_dtype (fp16 or bf16).
 * workspace: pkv_decode_prefix_fp8_workspace_bytes(...) bytes, 16-byte
 * aligned, always required; no initialisation needed.
 * -------------------------------------------------------------------- */
size_t pkv_decode_prefix_fp8_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                             int max_context_len, int prefix_pages, int partition_tokens);
pkv_status pkv_paged_attention_decode_prefix_fp8(void* out, const void* q, const void* k_cache,
                                                 const void* v_cache, const int32_t* block_tables,
                                                 int max_blocks_per_seq, const int32_t* context_lens,
                                                 int max_context_len, const int32_t* prefix_blocks,
                                                 int prefix_pages, int num_seqs, int num_q_heads, int num_kv_heads,
                                                 int head_dim, int num_blocks, float scale, float k_scale,
                                                 float v_scale, int partition_tokens, pkv_dtype q_dtype,
                                                 void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * pkv_paged_attention_multi -- paged attention for several query tokens
 * per sequence (speculative-decoding verification, prefill chunks).
 *
 * "PagedAttention 与 vLLM 推理加速" §6 (the large model verifies several
 * tokens the small model guessed, in one pass) and "LLM Systems 24 ..."
 * §2.2.1.3 (batches mixing prefill chunks and decode steps); §1 of the
 * former: a token attends over every token so far, itself included.
 *
 * Sequence b brings n_b = query_start[b+1] - query_start[b] new tokens,
 * rows query_start[b] .. query_start[b+1]-1 of q / out, whose K/V are
 * already appended (context_lens[b] counts them).  New token i sits at
 * position p = context_lens[b] - n_b + i; for every query head h:
 *   out[row, h, :] = softmax_j(scale * q[row, h, :] . K_j) V_j,  j = 0 .. p
 * with K_j / V_j read through block_tables as in pkv_paged_attention_decode.
 * A row with p < 0 (n_b > context_lens[b]) is zeros and sets
 * PKV_ERR_CONTEXT_RANGE.  One query token per sequence is decode.
 *
 * q, out [total_query_tokens, num_q_heads, head_dim]; query_start int32
 * [num_seqs + 1] (device), non-decreasing, query_start[num_seqs] <=
 * total_query_tokens, every n_b <= max_query_len (a sequence that breaks
 * this is skipped, its rows left unwritten, and PKV_ERR_CONTEXT_RANGE set).
 * fp16 / bf16 only (tensor cores).  With R = max_query_len * G rows per
 * kv-head: R <= 32 takes one tile per sequence (num_seqs <= 65535), else
 * tiles of 128 rows on the tcgen05 tensor cores (ceil(R / 128) <= 32767),
 * in a persistent kernel fed by a work list it writes into the workspace.
 * workspace: pkv_multi_workspace_bytes(...) bytes, 16-byte aligned (it
 * may be NULL when R <= 32 and max_context_len <= the partition).
 * partition_tokens as in pkv_paged_attention_decode, except the auto
 * partition (0): 2048 tokens, or 1024 when max_context_len > 4096 (several
 * rows a sequence make every partial n_b times the merge work, so short
 * contexts stay unsplit; long ones are split for balance across the SMs);
 * 8192 for the tcgen05 kernel (its items are claimed dynamically, longest
 * first, so long partitions leave no tail, while every split adds a merge).
 * -------------------------------------------------------------------- */
size_t pkv_multi_workspace_bytes(int total_query_tokens, int num_q_heads, int head_dim, int max_context_len,
                                 int partition_tokens);
pkv_status pkv_paged_attention_multi(void* out, const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, int max_blocks_per_seq,
                                     const int32_t* context_lens, int max_context_len,
                                     const int32_t* query_start, int max_query_len, int total_query_tokens,
                                     int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                     int num_blocks, float scale, int partition_tokens, pkv_dtype dtype,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* pkv_paged_attention_multi_fp8 -- pkv_paged_attention_multi over an FP8
 * (E4M3) pool written by pkv_kv_append_fp8: the rows, causal rule, tiles,
 * partitions, workspace and errors of pkv_paged_attention_multi, and the
 * cache layout and scales of pkv_paged_attention_decode_fp8 (a stored K
 * value is code * k_scale, V alike; k_scale, v_scale finite and > 0, else
 * PKV_EINVAL).  q and out in q_dtype (fp16 or bf16).  Every shape runs on
 * the tcgen05 kernel: tiles of 128 rows (num_seqs * ceil(max_query_len * G
 * / 128) <= 65535); each key block's codes are copied (TMA) into shared
 * memory and widened there to fp16 (exact), bf16 queries are rescaled into
 * fp16 per row by a power of two, the K scale goes into the logits and the
 * V scale into the output. */
pkv_status pkv_paged_attention_multi_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_tables, int max_blocks_per_seq,
                                         const int32_t* context_lens, int max_context_len,
                                         const int32_t* query_start, int max_query_len, int total_query_tokens,
                                         int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                         int num_blocks, float scale, float k_scale, float v_scale,
                                         int partition_tokens, pkv_dtype q_dtype, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Step planning on the host (no CUDA call; host arrays).
 *
 * pkv_partition_tokens -- the tokens per split-K partition that a call of
 * `op` makes with this partition_tokens argument (0 = its auto rule) and
 * max_context_len.  `extra` is PKV_OP_DECODE_PREFIX's prefix_pages and
 * PKV_OP_MULTI's rows per kv-head (max_query_len * num_q_heads /
 * num_kv_heads; 0 if unknown), and is read by those two ops only.
 * Auto rules:
 *   PKV_OP_DECODE         512, or 1024 when max_context_len > 4096;
 *   PKV_OP_DECODE_FP8     768, 1024 when max_context_len > 4096, 2048 when
 *                         it is > 16384;
 *   PKV_OP_MULTI          2048, or 1024 when max_context_len > 4096; with
 *                         more than 32 rows per kv-head (the tcgen05
 *                         kernel) 8192;
 *   PKV_OP_MULTI_FP8      8192 (the tcgen05 kernel);
 *   PKV_OP_DECODE_PREFIX  the longest suffix (max_context_len - 16 *
 *                         prefix_pages) rounded up to a page, kept in
 *                         [512, 2048] (the cascade's suffix pass).
 * An explicit partition_tokens must be a multiple of 16 in [16, 2048].
 * Returns -1 for an invalid op or partition_tokens.
 * -------------------------------------------------------------------- */
typedef enum {
  PKV_OP_DECODE = 0,        /* pkv_paged_attention_decode (and _static_ws) */
  PKV_OP_DECODE_FP8 = 1,    /* pkv_paged_attention_decode_fp8 */
  PKV_OP_MULTI = 2,         /* pkv_paged_attention_multi */
  PKV_OP_DECODE_PREFIX = 3, /* pkv_paged_attention_decode_prefix (suffix pass) */
  PKV_OP_MULTI_FP8 = 4      /* pkv_paged_attention_multi_fp8 */
} pkv_op;
int pkv_partition_tokens(pkv_op op, int partition_tokens, int max_context_len, int extra);

/* pkv_cow_copy_rows -- the rows each copy-on-write copy of a step must move.
 *
 * "PagedAttention 与 vLLM 推理加速" §3.2(3): a shared block is copied before
 * a sharer appends into it.  Such a block is partial (a full shared block
 * is never copied), so only its first rows hold tokens.  For each pair
 * (src, dst) of pairs[num_pairs][2]:
 *   copies[i] = (src, dst, rows),  rows = min over the slots s >= 0 of
 *   slots[num_slots] with s / 16 == dst of s % 16  (16 when none),
 * the first row this step writes into dst: rows 0 .. rows-1 hold the
 * sequence's earlier tokens and are what pkv_kv_append_copy copies.
 * copies: int32 [num_pairs][3], host memory the caller owns.  PKV_EINVAL
 * for a negative count or block id, or a NULL array that must be read. */
pkv_status pkv_cow_copy_rows(const int32_t* pairs, int num_pairs, const int64_t* slots, int num_slots,
                             int32_t* copies);

/* pkv_common_prefix_pages -- leading pages that every sequence of a batch
 * shares and fills completely.
 *
 * "PagedAttention 与 vLLM 推理加速" §3.2(3): requests with one system prompt
 * map the same physical blocks, which sit at the start of their block
 * tables (§2.3).  *prefix_pages = the largest p such that, for every page
 * j < p, all num_seqs tables hold one block id at column j and every
 * context_lens[b] >= 16 (j + 1); 0 when num_seqs < 2.  block_tables: int32
 * [num_seqs][width], context_lens: int32 [num_seqs], host memory.
 * PKV_EINVAL for negative sizes or lengths, or NULL arrays. */
pkv_status pkv_common_prefix_pages(const int32_t* block_tables, int num_seqs, int width,
                                   const int32_t* context_lens, int* prefix_pages);

/* pkv_cascade_prefix_pages -- the prefix pages to give
 * pkv_paged_attention_decode_prefix for this batch, or 0 when the plain
 * decode is the better call: the common prefix of pkv_common_prefix_pages
 * when dtype is PKV_F16 / PKV_BF16 (the cascade's tensor-core path) or
 * PKV_E4M3 (pkv_paged_attention_decode_prefix_fp8), at least
 * PKV_CASCADE_MIN_SEQS sequences share it and it spans at least
 * PKV_CASCADE_MIN_PAGES pages (below that the prefix pass and the merge
 * cost more than reading the few shared pages once per sequence). */
#define PKV_CASCADE_MIN_PAGES 8
#define PKV_CASCADE_MIN_SEQS 4
pkv_status pkv_cascade_prefix_pages(const int32_t* block_tables, int num_seqs, int width,
                                    const int32_t* context_lens, pkv_dtype dtype, int* prefix_pages);

/* ------------------------------------------------------------------------
 * Host block allocator.
 *
 * "vLLM + PagedAttention：打造高并发LLM推理引擎", "它是怎么工作的": blocks are
 * taken on demand as a request grows and go back to the pool when it ends.
 * "PagedAttention 与 vLLM 推理加速" §3.2(3) and "LLM Systems 24 ..." §3:
 * requests share blocks (common prefixes, parallel samples) through
 * reference counts, and a shared block is copied only when one of them
 * writes into it.
 *
 * Policy (the pages leave it open; this is the plain deterministic one):
 *   - the free list is FIFO, initialised from initial_free_order (NULL =
 *     0..num_blocks-1); allocation pops the front; a block whose count drops
 *     to 0 is pushed to the back; free_seq releases a table in table order;
 *   - fork: the child gets a copy of the parent's table and length, and every
 *     block in it gains one reference;
 *   - appending at position p: when p % 16 == 0 a fresh block is appended to
 *     the table; otherwise, when the last block is shared (count > 1), a
 *     fresh block replaces it, the old block loses one reference and the
 *     pair (old, new) is reported for pkv_copy_blocks; otherwise the token
 *     goes into the last block.  A full shared block is never copied;
 *   - slot = table[p / 16] * 16 + p % 16.
 * Every call either succeeds or returns an error and changes nothing.
 * The handle is not thread-safe; one thread at a time.
 * -------------------------------------------------------------------- */
typedef struct pkv_alloc pkv_alloc;

/* Create an allocator over num_blocks blocks (> 0).  initial_free_order,
 * when not NULL, must be a permutation of 0..num_blocks-1 (host memory). */
pkv_status pkv_alloc_create(int num_blocks, const int32_t* initial_free_order, pkv_alloc** out);
void pkv_alloc_destroy(pkv_alloc* a);

/* Add an empty sequence (EINVAL if the id exists). */
pkv_status pkv_alloc_add_seq(pkv_alloc* a, int64_t seq_id);
/* Child shares the parent's blocks (EINVAL: no parent, or child exists). */
pkv_status pkv_alloc_fork(pkv_alloc* a, int64_t parent, int64_t child);
/* Drop a sequence and its references (EINVAL: unknown id). */
pkv_status pkv_alloc_free_seq(pkv_alloc* a, int64_t seq_id);

/* Append one token.  *slot receives its slot; *cow_src / *cow_dst receive the
 * copy pair, or -1 / -1 when no copy is needed. */
pkv_status pkv_alloc_append_slot(pkv_alloc* a, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                                 int32_t* cow_dst);
/* Append n >= 0 tokens to one sequence: slots[n]; cow_pairs[2] receives the
 * single possible copy pair and *n_cow 0 or 1.  All or nothing. */
pkv_status pkv_alloc_append_tokens(pkv_alloc* a, int64_t seq_id, int n, int64_t* slots,
                                   int32_t* cow_pairs, int* n_cow);
/* One decode step: append one token to each of seq_ids[n] (distinct, known)
 * in order.  slots[n]; cow_pairs[2 * n] receives *n_cow pairs in order.
 * All or nothing (PKV_ENOMEM if the pool cannot serve the whole step). */
pkv_status pkv_alloc_step(pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* slots,
                          int32_t* cow_pairs, int* n_cow);
/* pkv_alloc_step, its copy pairs cut to rows by pkv_cow_copy_rows:
 * copies[3 * n] receives *n_copies (src, dst, rows) triples in order, ready
 * for pkv_kv_append_copy with this step's slots.  All or nothing. */
pkv_status pkv_alloc_step_copies(pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* slots,
                                 int32_t* copies, int* n_copies);

/* One sequence's table (up to cap entries), its block count and length. */
pkv_status pkv_alloc_block_table(const pkv_alloc* a, int64_t seq_id, int32_t* out, int cap,
                                 int* n_blocks, int64_t* context_len);
/* Dense tables for a batch: tables[n][width] (entries past a sequence's
 * last block set to pad) and context_lens[n].  EINVAL if a table is wider
 * than width or a length exceeds INT32_MAX. */
pkv_status pkv_alloc_block_tables(const pkv_alloc* a, const int64_t* seq_ids, int n,
                                  int32_t* tables, int width, int32_t pad, int32_t* context_lens);
/* Free list in order (free_list[num_blocks] may be NULL) and the count of
 * every block (refcounts[num_blocks] may be NULL). */
pkv_status pkv_alloc_state(const pkv_alloc* a, int32_t* free_list, int* n_free,
                           int32_t* refcounts);
int pkv_alloc_num_free(const pkv_alloc* a);
int pkv_alloc_num_blocks(const pkv_alloc* a);
/* Resident sequences (swapped ones not counted). */
int pkv_alloc_num_seqs(const pkv_alloc* a);

/* Preemption by swapping ("LLM Systems 24 ..." §3, conclusion).  The pages
 * give no policy; this one is:
 *   - a host-side pool of num_host_blocks blocks with its own FIFO free list
 *     (0..num_host_blocks-1) and reference counts, set (or re-set) by
 *     pkv_alloc_set_host_pool while no sequence is swapped out (else
 *     EINVAL);
 *   - swap_out(seq_ids[n]) (distinct, resident): every distinct device block
 *     of the listed tables, in id order then table order, gets the next
 *     free host block, and the pair (device, host) is written to
 *     pairs[cap][2] (*n_pairs pairs).  A block shared by several listed
 *     sequences maps to one host block that they share; each holder drops
 *     one device reference (a block reaching 0 goes to the back of the
 *     device free list; blocks shared with sequences not listed stay with
 *     them) and the listed sequences become swapped;
 *   - swap_in(seq_ids[n]) (distinct, swapped): the same with the roles of
 *     the pools exchanged; pairs are (host, device);
 *   - all or nothing: PKV_ENOMEM when the destination pool has too few free
 *     blocks, PKV_EINVAL when cap is smaller than the number of pairs;
 *   - a swapped sequence may only be freed (its host references are
 *     dropped) or swapped in; append, step, fork and block_table reject it.
 * The caller copies the pairs with pkv_swap_blocks: a swap-out's copy must
 * be enqueued before anything that writes the released device blocks, a
 * swap-in's before the sequence is next read. */
pkv_status pkv_alloc_set_host_pool(pkv_alloc* a, int num_host_blocks);
pkv_status pkv_alloc_swap_out(pkv_alloc* a, const int64_t* seq_ids, int n, int32_t* pairs, int cap,
                              int* n_pairs);
pkv_status pkv_alloc_swap_in(pkv_alloc* a, const int64_t* seq_ids, int n, int32_t* pairs, int cap,
                             int* n_pairs);
/* Host free list in order (free_list[num_host_blocks] may be NULL) and the
 * count of every host block (refcounts[num_host_blocks] may be NULL). */
pkv_status pkv_alloc_host_state(const pkv_alloc* a, int32_t* free_list, int* n_free, int32_t* refcounts);
/* A swapped sequence's host table (up to cap entries), block count, length. */
pkv_status pkv_alloc_swapped_table(const pkv_alloc* a, int64_t seq_id, int32_t* out, int cap, int* n_blocks,
                                   int64_t* context_len);
int pkv_alloc_num_swapped(const pkv_alloc* a);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
