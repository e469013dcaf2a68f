/*
 * kv8.h -- C ABI of libkv8: paged INT8 KV-cache decode attention for B200
 * (sm_100a).
 *
 * The method [KV-Cache 全栈优化系统, 主要特性 "低比特线性与 KV-cache 压缩"]:
 * keys and values are quantised dynamically per token to INT8, kept
 * compressed in the cache, and restored on demand inside attention.  The
 * cache is paged [KV Cache 优化全景解析——从基础原理到工程实践, §4.2
 * PagedAttention]: each sequence's logical 16-token blocks map through a
 * block table to physically scattered blocks, and several sequences may list
 * the same physical block (shared prefixes).  Query heads are grouped onto KV
 * heads [same page, §3.3 GQA].  Decode attention is
 * softmax(q K^T / sqrt(d)) V [same page, §2.1] with FP32 accumulation
 * [大模型推理加速：KV Cache与vLLM技术解析, §4.1 混合精度计算].
 *
 * Conventions shared by every entry point
 *   - Every pointer argument except the stream is a DEVICE pointer owned by
 *     the caller.  The library allocates nothing and keeps no state between
 *     calls that changes a result (it caches only per-device facts such as
 *     the SM count, and the device status word below).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; a KV8_OK return means the
 *     work was launched, not that it finished.
 *   - Argument checks are made on the host before anything is launched; a
 *     failed check launches nothing and returns KV8_ERR_INVALID_ARG,
 *     KV8_ERR_UNSUPPORTED or KV8_ERR_WORKSPACE.  KV8_ERR_CUDA reports a launch
 *     error (cudaGetLastError).  Nothing aborts, exits or traps.
 *   - Device-resident indices (slot_mapping, block_tables, context_lens) are
 *     trusted: they must lie in range (the caller's contract).
 *   - Supported shapes: head_dim == 128, block_size == 16,
 *     num_q_heads / num_kv_heads in {1, 2, 4, 8}; other values return
 *     KV8_ERR_UNSUPPORTED.  Device pointers must be 16-byte aligned.
 *
 * Memory layout (row-major, innermost last)
 *   k_cache, v_cache  int8    [num_blocks][num_kv_heads][block_size][head_dim]
 *   k_scales,v_scales float32 [num_blocks][num_kv_heads][block_size]
 *   One (block, kv_head) "page" is block_size*head_dim = 2048 contiguous code
 *   bytes plus 64 contiguous scale bytes.  Token t of sequence b lives in
 *   physical block block_tables[b][t / block_size] at offset t % block_size.
 */
#ifndef KV8_H
#define KV8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KV8_API __attribute__((visibility("default")))
#else
#define KV8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define KV8_OK 0
#define KV8_ERR_INVALID_ARG 1 /* null pointer, bad shape, misaligned buffer */
#define KV8_ERR_UNSUPPORTED 2 /* valid but not built: head_dim, block, group */
#define KV8_ERR_WORKSPACE 3   /* workspace missing or smaller than required */
#define KV8_ERR_CUDA 4        /* a CUDA launch or attribute call failed */

/* Output element types for kv8_paged_decode_attention / kv8_split_reduce. */
#define KV8_OUT_BF16 0
#define KV8_OUT_F32 1

/* Human-readable name of a status code (static string, never NULL). */
KV8_API const char *kv8_status_string(int32_t status);

/*
 * kv8_quantize_append -- quantise new K/V rows and store them in the cache.
 *
 * Defined by [KV-Cache 全栈优化系统, 主要特性]: per-token dynamic INT8
 * quantisation, with the quantisation group one KV head's head_dim values
 * [大模型推理加速, §4.1: quant group size 128].  For every token i and KV head
 * h, separately for K and for V:
 *     a = max_j |x_j|                      (exact, fp32)
 *     s = a / 127 in IEEE fp32 (round to nearest even); s = 0 when a == 0
 *     c_j = clamp(rint(x_j / s), -127, 127), x_j / s an IEEE fp32 division,
 *           rint ties to even; c_j = 0 when s == 0
 * Codes go to block slot_mapping[i] / block_size at offset
 * slot_mapping[i] % block_size [KV Cache 优化全景解析, §4.2: the block table
 * maps logical to physical blocks]; the scale goes beside them.
 *
 *   k_new, v_new   bf16 [n_tokens][num_kv_heads][head_dim], read only
 *   slot_mapping   int64 [n_tokens]; slot < 0 means padding: token skipped
 *   k_cache, v_cache, k_scales, v_scales   written at the mapped slots only
 * The caller must not point two tokens at one slot in a call, nor point a
 * slot at a block other sequences share (copy it first).
 * n_tokens == 0 launches nothing and returns KV8_OK.
 */
KV8_API int32_t kv8_quantize_append(const void *k_new, const void *v_new,
                            const int64_t *slot_mapping, int64_t n_tokens,
                            int32_t num_kv_heads, int32_t head_dim,
                            int32_t block_size, int64_t num_blocks,
                            int8_t *k_cache, int8_t *v_cache, float *k_scales,
                            float *v_scales, void *stream);

/*
 * kv8_decode_workspace_bytes -- bytes of workspace a split launch needs.
 *
 * Workspace holds, per (sequence, query head, context chunk), the chunk's
 * running max and sum (2 fp32) and its unnormalised output (head_dim fp32),
 * plus one 32-bit merge ticket per (sequence, query head).
 * Returns 0 when chunk_tokens == 0 or every context fits one chunk.
 */
KV8_API size_t kv8_decode_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                  int32_t head_dim, int32_t max_context_len,
                                  int32_t chunk_tokens);

/*
 * kv8_decode_chunk_tokens -- a chunk_tokens for kv8_paged_decode_attention
 * that keeps every SM of the current device busy.
 *
 * The split is a scheduling choice the pages leave open.  A decode launch
 * hands one (sequence, KV head, chunk) to each warp at a time, about 12
 * warps per SM; with few sequences or short contexts whole chunks leave
 * warps idle and make the slowest warp's chain of pages the launch time.
 * Finer chunks are not free: each costs its warp a q load, a partial written
 * and read back and a merge step.  This returns the chunk length, a multiple
 * of 16 between 64 and 512, that cuts max_context_len into equal chunks so
 * that batch * num_kv_heads * chunks is at least the resident warps of the
 * current device (148 SMs are assumed when no device can be queried), or 0
 * (no split) when max_context_len <= 64.  Size the workspace with the returned
 * value (kv8_decode_workspace_bytes).  Returns 0 for non-positive arguments.
 */
KV8_API int32_t kv8_decode_chunk_tokens(int32_t batch, int32_t num_kv_heads,
                                        int32_t max_context_len);

/*
 * kv8_paged_decode_attention -- one decode step of GQA attention over the
 * paged INT8 cache, for one new query token per sequence.
 *
 * For sequence b and query head h (KV head h / (num_q_heads/num_kv_heads),
 * [KV Cache 优化全景解析, §3.3]) over the n = context_lens[b] cached tokens
 * t (the token appended this step included, [大模型推理加速, §2.1: append the
 * new K/V, then attend over the whole cache]):
 *     k_hat_t = kc_t * ks_t,  v_hat_t = vc_t * vs_t      (dequantise)
 *     score_t = softmax_scale * <q, k_hat_t>
 *     out     = sum_t softmax(score)_t * v_hat_t
 * [KV Cache 优化全景解析, §2.1], accumulated in fp32 with an online softmax.
 * n == 0 gives an all-zero output row.
 *
 *   q              bf16 [batch][num_q_heads][head_dim]
 *   block_tables   int32 [batch][max_blocks_per_seq]; entries past
 *                  ceil(n / block_size) are never read
 *   context_lens   int32 [batch]; every value <= max_context_len
 *   max_context_len  host-side bound on context_lens (sizes the grid);
 *                  must be <= max_blocks_per_seq * block_size
 *   softmax_scale  <= 0 selects 1/sqrt(head_dim)
 *   chunk_tokens   0: one pass per (sequence, KV head), no workspace.
 *                  > 0 (a multiple of block_size): the context is split into
 *                  chunks of that many tokens processed in parallel; a
 *                  sequence that fits one chunk writes `out` directly, the
 *                  others write per-chunk partials to `workspace`, and the
 *                  last chunk of each (sequence, KV head) to finish merges
 *                  them into `out` in the same kernel (the merge that
 *                  kv8_split_reduce performs).  The call enqueues a memset
 *                  of the merge tickets and one kernel.
 *   workspace      device buffer of >= kv8_decode_workspace_bytes(...) bytes
 *                  (may be NULL when that is 0); contents are scratch
 *   out            [batch][num_q_heads][head_dim] of bf16 (out_dtype ==
 *                  KV8_OUT_BF16, round to nearest even) or fp32 (KV8_OUT_F32)
 * The caches are only read; blocks may be shared between sequences.
 */
KV8_API int32_t kv8_paged_decode_attention(
    const void *q, const int8_t *k_cache, const int8_t *v_cache,
    const float *k_scales, const float *v_scales, const int32_t *block_tables,
    const int32_t *context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void *workspace,
    size_t workspace_bytes, void *out, int32_t out_dtype, void *stream);

/*
 * kv8_paged_decode_attention_append -- one decode step in one launch: the
 * step's new token of every sequence is quantised into the cache and then
 * attended to, as kv8_quantize_append followed by kv8_paged_decode_attention
 * [大模型推理加速：KV Cache与vLLM技术解析, §2.1: the new K/V join the cache
 * before the step attends to it], with the same codes, scales and output bit
 * for bit.
 *
 * Arguments as kv8_paged_decode_attention (form KV8_FORM_AUTO), with the
 * caches and scales writable, plus
 *   k_new, v_new   bf16 [batch][num_kv_heads][head_dim] device, read only:
 *                  sequence b's new token, which sits at position
 *                  context_lens[b] - 1 (context_lens counts it) in the block
 *                  block_tables[b][(context_lens[b] - 1) / block_size]; a
 *                  sequence with context_lens[b] == 0 has no new token
 * The warp that takes a sequence's last chunk (its last page) quantises the
 * token for its KV head before copying that page, so no other launch is
 * needed and no other warp reads the page.  As for kv8_quantize_append the
 * caller must not point the position at a block other sequences share.  The
 * call enqueues a memset of the merge tickets (split launches) and one
 * kernel.
 */
KV8_API int32_t kv8_paged_decode_attention_append(
    const void *q, const void *k_new, const void *v_new, int8_t *k_cache,
    int8_t *v_cache, float *k_scales, float *v_scales,
    const int32_t *block_tables, const int32_t *context_lens, int32_t batch,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, float softmax_scale, int32_t chunk_tokens,
    void *workspace, size_t workspace_bytes, void *out, int32_t out_dtype,
    void *stream);

/*
 * kv8_paged_decode_attention_prefix -- kv8_paged_decode_attention for a
 * batch in which groups of sequences share the first tokens of their
 * context, stored once: the same physical blocks open every member's block
 * table [KV Cache 优化全景解析, §4.2 PagedAttention: several sequences map
 * one physical block].  The shared pages are read, converted and scored once
 * for the whole group instead of once per member, the way serving systems
 * group the requests that share a prefix [garden.houmin.site
 * infra/kv-cache-optimize, §4.3.1 Prefix-aware Scheduling (BatchLLM)].
 * The shared chunks run on the 5th-generation tensor cores, all of a group's
 * query rows (members x heads of a KV head) against each shared key tile,
 * with fp16 operands as in kv8_paged_extend_attention: the K and V codes
 * exactly, q scaled per row by a power of two, the probabilities rounded to
 * fp16.  Results are those of kv8_paged_decode_attention on the same inputs
 * within the decode tolerance (|difference| <= 2e-3 for unit-scale V; the
 * probability rounding bounds it by 2^-11 max |v_hat|), not bit for bit.
 *
 * Arguments as kv8_paged_decode_attention (form KV8_FORM_AUTO), plus
 *   prefix_group    int32 [batch] device: the group of sequence b, or -1
 *   prefix_lens     int32 [num_groups] device: tokens group g's members
 *                   share at the start of their contexts.  The whole chunks
 *                   of that prefix (prefix_lens[g] / chunk_tokens of them)
 *                   are computed once for the group; the rest of each
 *                   member's context as usual.  Every member's
 *                   context_lens must be >= prefix_lens[g], and its block
 *                   table must list the group's blocks for those tokens (a
 *                   member found shorter sets bit 1 of the device status
 *                   word and its row is left incomplete).
 *   num_groups      number of groups (0: a plain decode call)
 *   max_group_size  host bound on the members of any group (any size;
 *                   members are served 128 / G at a time, G = query heads
 *                   per KV head)
 *   max_prefix_len  host bound on prefix_lens (<= max_context_len)
 *   chunk_tokens    must be > 0
 * A sequence belongs to at most one group.  The call enqueues a memset of
 * the merge tickets, the shared-prefix kernel and the decode kernel.
 */
KV8_API int32_t kv8_paged_decode_attention_prefix(
    const void *q, const int8_t *k_cache, const int8_t *v_cache,
    const float *k_scales, const float *v_scales, const int32_t *block_tables,
    const int32_t *context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    const int32_t *prefix_group, const int32_t *prefix_lens,
    int32_t num_groups, int32_t max_group_size, int32_t max_prefix_len,
    float softmax_scale, int32_t chunk_tokens, void *workspace,
    size_t workspace_bytes, void *out, int32_t out_dtype, void *stream);

/*
 * kv8_paged_extend_attention -- extend (prefill) attention over the paged
 * INT8 cache: every sequence's new query rows attend causally to its cache.
 *
 * A prompt's tokens are processed together and fill the cache; a long prompt
 * may enter in chunks, each attending to everything cached before it
 * [KV Cache 优化全景解析——从基础原理到工程实践, §2.2 Prefill 与 Decode 两阶段,
 * §11.2 chunked prefill].  The new K/V rows are appended first
 * (kv8_quantize_append), as in decode.  Sequence b has n_b = q_start[b+1] -
 * q_start[b] new rows, its last n_b cached positions; row i sits at position
 * p = context_lens[b] - n_b + i and attends to tokens 0..p:
 *     out = softmax(q K_hat^T / sqrt(d)) V_hat     [same page, §2.1]
 * with K_hat = code * ks, V_hat = code * vs and fp32 accumulation.  Both
 * products run on the 5th-generation tensor cores (fp16 operands: the INT8
 * codes exactly, q scaled per row by a power of two, the probabilities
 * rounded to fp16).
 *
 *   q            bf16 [q_start[batch]][num_q_heads][head_dim], rows packed
 *                by sequence
 *   q_start      int32 [batch + 1] device, non-decreasing from 0;
 *                n_b <= context_lens[b]
 *   max_q_len    host bound on n_b (sizes the grid)
 *   out          [q_start[batch]][num_q_heads][head_dim], bf16 or fp32
 * Other arguments as kv8_paged_decode_attention; no workspace.  The call
 * enqueues one kernel.
 */
KV8_API int32_t kv8_paged_extend_attention(
    const void *q, const int8_t *k_cache, const int8_t *v_cache,
    const float *k_scales, const float *v_scales, const int32_t *block_tables,
    const int32_t *context_lens, const int32_t *q_start, int32_t batch,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_q_len, float softmax_scale, void *out, int32_t out_dtype,
    void *stream);

/*
 * Context-parallel decode: one long context spread over several GPUs.
 *
 * Context partitioning splits a sequence's context across devices that each
 * process their own part [garden.houmin.site infra/kv-cache-optimize,
 * §4.1.2 KV-Runahead]; for decode, each rank holds the blocks of its part of
 * every sequence (its own cache, block tables and context lengths for that
 * part), computes the chunk partials (m, l, o) of its part, the ranks
 * exchange the partials (an all-gather of (2 + head_dim) floats per chunk and
 * query head), and the log-sum-exp merge over every rank's chunks gives the
 * attention over the whole context, the merge kv8_split_reduce performs for
 * one rank.
 *
 * kv8_decode_partials_bytes -- bytes of one rank's partials: per (sequence,
 * query head, chunk slot) (m, l) then o, for C = ceil(max_context_len /
 * chunk_tokens) slots (at least 1).  0 for invalid arguments.
 *
 * kv8_paged_decode_attention_partials -- the decode call of one rank: the
 * same arguments as kv8_paged_decode_attention (its local cache, tables and
 * context lengths), chunk_tokens > 0, every chunk slot of every (sequence,
 * query head) written to `partials` (empty slots as m = -inf, l = 0, o = 0),
 * nothing merged, no output.  Every rank must use the same batch,
 * num_q_heads, max_context_len (a bound on every rank's local lengths) and
 * chunk_tokens, so that the layouts match.
 *
 * kv8_merge_partials -- the log-sum-exp merge over `ranks` partial buffers,
 * rank r's at partials + r * rank_stride bytes (each written by
 * kv8_paged_decode_attention_partials with the same batch, num_q_heads,
 * max_context_len and chunk_tokens), into out [batch][num_q_heads][head_dim]
 * (bf16 or fp32).
 */
KV8_API size_t kv8_decode_partials_bytes(int32_t batch, int32_t num_q_heads,
                                         int32_t head_dim,
                                         int32_t max_context_len,
                                         int32_t chunk_tokens);

KV8_API int32_t kv8_paged_decode_attention_partials(
    const void *q, const int8_t *k_cache, const int8_t *v_cache,
    const float *k_scales, const float *v_scales, const int32_t *block_tables,
    const int32_t *context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void *partials,
    size_t partials_bytes, void *stream);

KV8_API int32_t kv8_merge_partials(const void *partials, size_t rank_stride,
                                   int32_t ranks, int32_t batch,
                                   int32_t num_q_heads, int32_t head_dim,
                                   int32_t max_context_len,
                                   int32_t chunk_tokens, void *out,
                                   int32_t out_dtype, void *stream);

/*
 * kv8_split_reduce -- merge the per-chunk partials of a split decode launch.
 *
 * For each (b, h) whose context spans C = ceil(n / chunk_tokens) > 1 chunks,
 * with chunk partials (m_c, l_c, o_c) written in base-2 exponent form
 * (o_c = sum_t 2^(s_t - m_c) v_hat_t, l_c = sum_t 2^(s_t - m_c),
 * s_t = score_t * log2(e)):
 *     M = max_c m_c,  L = sum_c l_c 2^(m_c - M),
 *     out = sum_c o_c 2^(m_c - M) / L
 * i.e. the log-sum-exp merge of the chunk softmaxes.  Rows with C <= 1 are
 * left untouched (the split launch wrote them).  kv8_paged_decode_attention
 * performs this merge inside its own kernel; this entry point re-runs it
 * from the partials a split launch left in the workspace (for pipelining
 * and for tests), with the same arithmetic in the same order.
 *
 *   workspace      as written by a split launch with the same batch,
 *                  num_q_heads, head_dim, max_context_len and chunk_tokens
 *   context_lens   int32 [batch], the same values the split launch read
 */
KV8_API int32_t kv8_split_reduce(const void *workspace, size_t workspace_bytes,
                         const int32_t *context_lens, int32_t batch,
                         int32_t num_q_heads, int32_t head_dim,
                         int32_t max_context_len, int32_t chunk_tokens,
                         void *out, int32_t out_dtype, void *stream);

/* Decode forms for kv8_paged_decode_attention_form. */
#define KV8_FORM_AUTO 0      /* KV8_FORM_MMA_I8 for groups of <= 4 heads,
                                KV8_FORM_MMA_F16PV for groups of 8 */
#define KV8_FORM_CUDA_CORE 1 /* codes converted to fp32, fp32 FMA */
#define KV8_FORM_MMA_F16PV 2 /* warp mma: int8 q.k, fp16 p.v */
#define KV8_FORM_TCGEN05 3   /* 5th-generation tensor cores, TMEM accumulators */
#define KV8_FORM_MMA_I8 4    /* warp mma: int8 q.k, int8 p.v on raw V codes */

/*
 * kv8_paged_decode_attention_form -- kv8_paged_decode_attention with the
 * decode form chosen by the caller, for every call separately:
 *   KV8_FORM_AUTO       the form kv8_paged_decode_attention uses:
 *                       KV8_FORM_MMA_I8 for groups of 1, 2 or 4 query
 *                       heads per KV head, KV8_FORM_MMA_F16PV for 8,
 *   KV8_FORM_CUDA_CORE  codes converted to fp32 in registers, fp32 FMA,
 *   KV8_FORM_MMA_F16PV  warp tensor cores (mma.sync): q.k as int8 products
 *                       of the K codes with exact int8 digit planes of q;
 *                       p.v on V codes converted exactly to fp16, fp32
 *                       accumulation,
 *   KV8_FORM_TCGEN05    q.k and p.v both as int8 products on the
 *                       5th-generation tensor cores (digit planes of q and of
 *                       the probabilities), int32 accumulators in tensor
 *                       memory, K and V codes read as TMA stages them,
 *   KV8_FORM_MMA_I8     warp tensor cores (mma.sync), both products int8:
 *                       q.k as in KV8_FORM_MMA_F16PV; p.v multiplies the V
 *                       codes as stored (a transposing shared-memory load)
 *                       by exact byte planes of the integer-rounded
 *                       probabilities, int32 accumulation.  Groups of 1, 2
 *                       or 4 query heads per KV head; a group of 8 runs
 *                       KV8_FORM_MMA_F16PV.
 * Every form computes the same function; results differ only by rounding
 * order, each within the accuracy kv8_paged_decode_attention states.  Any
 * other `form` returns KV8_ERR_INVALID_ARG.  The choice lives in the call:
 * the library keeps no selector between calls.
 */
KV8_API int32_t kv8_paged_decode_attention_form(
    const void *q, const int8_t *k_cache, const int8_t *v_cache,
    const float *k_scales, const float *v_scales, const int32_t *block_tables,
    const int32_t *context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void *workspace,
    size_t workspace_bytes, void *out, int32_t out_dtype, int32_t form,
    void *stream);

/*
 * kv8_read_device_status -- synchronise the current device, then read the
 * library's sticky device status word (0 = clean; bit 0 = a kernel gave up
 * waiting for one of its own shared-memory copies and skipped that work
 * instead of hanging; bit 1 = a shared-prefix group listed a member whose
 * context is shorter than the group's prefix).  clear != 0 resets the word
 * to 0 afterwards.
 */
KV8_API int32_t kv8_read_device_status(uint32_t *status, int32_t clear);

/*
 * kv8_paged_decode_attention_noalloc -- kv8_paged_decode_attention for
 * callers that cannot allocate device memory.
 *
 * The source pages have no counterpart for this entry point; it exists for
 * callers that cannot hand the split-K decode a workspace: code running
 * inside a framework that owns every byte of device memory (a serving engine
 * that reserves almost the whole GPU for its KV pool up front, a plugin whose
 * host offers no workspace), or latency-critical code that must not call
 * cudaMalloc because it can synchronise the device.
 *
 * Arguments and results are those of kv8_paged_decode_attention without
 * `workspace` / `workspace_bytes`: the caller still passes every input and
 * the output.  The chunk partials go to a fixed scratch array inside the
 * library, KV8_NOALLOC_WORKSPACE_BYTES long, which every GPU that loads the
 * library holds until the process exits.  Nothing is allocated or freed.
 *   - Limit: a launch whose split needs more than
 *     KV8_NOALLOC_WORKSPACE_BYTES (kv8_decode_workspace_bytes(...) of the
 *     same arguments) returns KV8_ERR_WORKSPACE and launches nothing; use a
 *     larger chunk_tokens (fewer chunks) or the allocating entry point.
 *   - The first call on each device looks up the array's device address on
 *     that device (cudaGetSymbolAddress) and keeps it; make that first call
 *     before any stream capture.  Resetting the device after that first call
 *     is not supported (the kept address would be stale).
 *   - Every call shares the one array, which keeps the last call's contents.
 *     The chunk partials need no initial value; the merge tickets at the end
 *     of the array must start at zero, and each call clears them on its
 *     stream before its kernel.  Calls whose kernels overlap on the GPU
 *     (e.g. on unordered streams) race on the partials and the tickets:
 *     order them.
 */
#define KV8_NOALLOC_WORKSPACE_BYTES (16u << 20) /* 16 MiB per device */

KV8_API int32_t kv8_paged_decode_attention_noalloc(
    const void *q, const int8_t *k_cache, const int8_t *v_cache,
    const float *k_scales, const float *v_scales, const int32_t *block_tables,
    const int32_t *context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void *out, int32_t out_dtype,
    void *stream);

/*
 * The INT4 variant of the cache.
 *
 * Historical tokens' K and V may be kept in 4 bits [nano-KvLLM, §2.2
 * 量化感知缓存], half a byte per element [KV Cache 优化全景解析, §2.3
 * table]; the pages give no formula, so the INT8 scheme carries over with 7
 * levels each side of zero, per (token, KV head):
 *     s = fl32(max_j |x_j| / 7) (IEEE division; s = 0 for an all-zero row)
 *     c_j = clamp(rint(fl32(x_j / s)), -7, 7), ties to even; 0 when s == 0
 * stored as the nibble c_j + 8, dims 2i and 2i+1 in the low and high nibble
 * of byte i.  Layout: k_cache / v_cache uint8 [num_blocks][num_kv_heads]
 * [block_size][head_dim / 2] (64 bytes a token, 1 KB a page), k_scales /
 * v_scales fp32 [num_blocks][num_kv_heads][block_size].
 *
 * kv8_int4_quantize_append -- kv8_quantize_append into the INT4 cache (same
 * arguments, same rules on slots and padding).
 */
KV8_API int32_t kv8_int4_quantize_append(const void *k_new, const void *v_new,
                                         const int64_t *slot_mapping,
                                         int64_t n_tokens, int32_t num_kv_heads,
                                         int32_t head_dim, int32_t block_size,
                                         int64_t num_blocks, uint8_t *k_cache,
                                         uint8_t *v_cache, float *k_scales,
                                         float *v_scales, void *stream);

/*
 * kv8_int4_paged_decode_attention -- kv8_paged_decode_attention over the
 * INT4 cache: k_hat = c * ks, v_hat = c * vs with c = nibble - 8.  Same
 * arguments, workspace (kv8_decode_workspace_bytes), split and status codes;
 * groups of 1, 2, 4 or 8 query heads per KV head (8: two sub-groups of 4,
 * each its own item, reading the same pages).  Both products run on the
 * warp tensor cores with the nibbles as unsigned 8-bit operands; the +8 bias
 * is removed exactly in integer arithmetic.
 */
KV8_API int32_t kv8_int4_paged_decode_attention(
    const void *q, const uint8_t *k_cache, const uint8_t *v_cache,
    const float *k_scales, const float *v_scales, const int32_t *block_tables,
    const int32_t *context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void *workspace,
    size_t workspace_bytes, void *out, int32_t out_dtype, void *stream);

/*
 * kv8_check_indices -- debug check of the device-resident indices the other
 * calls trust (they are the caller's contract and are not checked there).
 * A debug aid with no counterpart on the pages.
 * Counts, into counts[0..2] (device uint32, zeroed by the call first):
 *   counts[0]  sequences with context_lens[b] < 0 or > max_context_len
 *   counts[1]  block-table entries a decode would read (the first
 *              ceil(len / block_size) of row b, len clamped to [0,
 *              min(max_context_len, max_blocks_per_seq * 16)]) outside
 *              [0, num_blocks)
 *   counts[2]  slot_mapping entries >= num_blocks * 16 (negative entries are
 *              padding)
 * batch may be 0 (no table check) and n_tokens may be 0 (no slot check;
 * slot_mapping may be NULL).  The kernels read only those arrays, within the
 * bounds given here, so the check is safe on inputs a decode must not see.
 * Asynchronous on `stream`: read counts after synchronising.  Status codes
 * as elsewhere.
 */
KV8_API int32_t kv8_check_indices(const int32_t *block_tables,
                                  const int32_t *context_lens, int32_t batch,
                                  int32_t max_blocks_per_seq,
                                  int64_t num_blocks, int32_t max_context_len,
                                  const int64_t *slot_mapping, int64_t n_tokens,
                                  uint32_t *counts, void *stream);

/*
 * The KIVI variant of the cache [KV Cache 优化全景解析——从基础原理到工程实践,
 * §7.1 量化的核心挑战 and §7.2 KIVI：2bit 无损非对称量化]: 2-bit asymmetric
 * codes, keys grouped per channel (channels differ widely) and values per
 * token (a token's channels are even).  The page gives the axes, the width
 * and the asymmetry; the library's readings:
 *   - a group x is stored as its minimum z, a scale
 *     s = fl32(fl32(max - z) / 3) (IEEE subtraction and division) and codes
 *     c = clamp(rint(fl32(fl32(x - z) / s)), 0, 3), ties to even; s = 0 and
 *     c = 0 for a constant group; x_hat = c * s + z;
 *   - a key group is one channel of one 16-token page (one block of one KV
 *     head); a value group is one token of one KV head (128 channels);
 *   - a page is quantised when its 16th token is appended.  Until then the
 *     page's K and V rows stay in bf16 in the sequence's tail and attention
 *     reads them as they are (recent tokens keep their precision
 *     [nano-KvLLM, §2.2 量化感知缓存]).
 *
 * Layout
 *   kivi_cache  uint8 [num_blocks][num_kv_heads][KV8_KIVI_PAGE_BYTES], one
 *               page record per (block, KV head):
 *       [   0,  512)  K codes: 128 little-endian 32-bit words, word j =
 *                     channel j, token t in bits 2t and 2t+1
 *       [ 512, 1024)  V codes, the same layout
 *       [1024, 1536)  K scales, fp32 [128] (per channel)
 *       [1536, 2048)  K zero points, fp32 [128]
 *       [2048, 2112)  V scales, fp32 [16] (per token)
 *       [2112, 2176)  V zero points, fp32 [16]
 *   kivi_tail   bf16 [batch][num_kv_heads][2][block_size][head_dim]: the K
 *               rows (index 0) and V rows (index 1) of each sequence's last
 *               page while it holds fewer than 16 tokens; row r = position
 *               % 16.  Row b of the tail belongs to the sequence in batch
 *               row b, in every append and decode call.
 * 136 bytes a token per KV head, against 264 for the INT8 cache.
 */
#define KV8_KIVI_PAGE_BYTES 2176

/*
 * kv8_kivi_append -- append new tokens to the KIVI cache.
 *
 *   k_new, v_new   bf16 [cu_new[batch]][num_kv_heads][head_dim]: sequence
 *                  b's new rows are rows cu_new[b] .. cu_new[b+1]-1, for
 *                  positions context_lens[b] - n_b .. context_lens[b] - 1
 *                  (n_b = cu_new[b+1] - cu_new[b]; context_lens counts them)
 *   cu_new         int32 [batch + 1], cu_new[0] = 0, non-decreasing
 *   context_lens   int32 [batch], n_b <= context_lens[b] <= max_blocks_per_seq
 *                  * block_size
 *   block_tables   int32 [batch][max_blocks_per_seq]; the blocks of the
 *                  pages this call completes are written
 *   max_new_tokens host-side bound on every n_b (sizes the grid); 0 = no-op
 * Every page that one of the new positions completes (positions 16j .. 16j+15
 * all present after the call) is quantised from the tail's earlier rows and
 * the new rows into its record; then the new rows of the last, partial page
 * are copied into the tail.  The tail rows of positions before this call
 * must hold what earlier calls appended.  The caller must not point a new
 * position at a block other sequences share.  Two kernels on `stream`.
 */
KV8_API int32_t kv8_kivi_append(const void *k_new, const void *v_new,
                                const int32_t *cu_new,
                                const int32_t *context_lens,
                                const int32_t *block_tables, int32_t batch,
                                int32_t num_kv_heads, int32_t head_dim,
                                int32_t block_size, int32_t max_blocks_per_seq,
                                int64_t num_blocks, int32_t max_new_tokens,
                                uint8_t *kivi_cache, void *kivi_tail,
                                void *stream);

/*
 * kv8_kivi_paged_decode_attention -- kv8_paged_decode_attention over the
 * KIVI cache: for sequence b with n = context_lens[b] and F = 16 * floor(n /
 * 16), tokens t < F are dequantised from their page record,
 *     k_hat_t[j] = c * k_scale[j] + k_zero[j],  v_hat_t[j] = c * v_scale[t]
 *                  + v_zero[t],
 * and tokens F <= t < n are the bf16 rows of the tail.  Same arguments,
 * workspace (kv8_decode_workspace_bytes), split, output types and status
 * codes as kv8_paged_decode_attention; groups of 1, 2, 4 or 8 query heads per
 * KV head (8: two sub-groups of 4).  fp32 arithmetic on the CUDA cores; one
 * kernel (and a memset of the merge tickets when split).
 */
KV8_API int32_t kv8_kivi_paged_decode_attention(
    const void *q, const uint8_t *kivi_cache, const void *kivi_tail,
    const int32_t *block_tables, const int32_t *context_lens, int32_t batch,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, float softmax_scale, int32_t chunk_tokens,
    void *workspace, size_t workspace_bytes, void *out, int32_t out_dtype,
    void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KV8_H */
