/*
 * kv8_oracle.c -- plain, slow, single-threaded CPU oracle for paged INT8 KV
 * decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the bench's CPU-baseline
 * leg use it.  It shares no code, header, table or helper with the CUDA
 * library; it is written from the definitions on the source pages:
 *
 *   [KV-Cache 全栈优化系统, 主要特性 "低比特线性与 KV-cache 压缩"]
 *       K/V are quantised dynamically per token to INT8, stored compressed and
 *       restored on demand inside attention.
 *   [大模型推理加速：KV Cache与vLLM技术解析, §4.1 混合精度计算]
 *       quant group size 128 (one head_dim); attention accumulates in FP32.
 *   [KV Cache 优化全景解析——从基础原理到工程实践, §2.1 formula
 *    Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V]
 *   [same page, §3.3 GQA]   h query heads split into G groups sharing one K/V.
 *   [same page, §4.2 PagedAttention]   logical blocks -> physical blocks via a
 *       block table; several sequences may map to the same physical block.
 *   [same page, §2.3 KV Cache 内存计算公式]
 *       memory = 2 * L * B * T * H_kv * d_h * bytes_per_element.
 *   [same page, §7.1 and §7.2 KIVI]   the KIVI variant: 2-bit asymmetric
 *       codes, keys per channel, values per token (its readings are stated
 *       where it is defined, below).
 *   [nano-KvLLM, §2.2 量化感知缓存]   the INT4 variant of historical tokens,
 *       and recent tokens kept at their original precision.
 *
 * Readings where the pages are silent (all listed in the design notes):
 *   - one scale per (token, KV head), s = fl32(max|x| / 127), stored as fp32;
 *   - code = clamp(rint(fl32(x / s)), -127, 127), IEEE single division and
 *     ties-to-even rounding; s = 0 and all codes 0 for an all-zero vector;
 *   - attention is computed in fp64 over the dequantised cache
 *     k_hat = code * scale (exact in double), softmax scale 1/sqrt(d);
 *   - GQA grouping is contiguous: KV head = query head / (H_q / H_kv);
 *   - a context of length 0 gives an all-zero output row.
 *
 * Layouts (the same ones the library documents, restated here on purpose):
 *   x (bf16 bits)  [n_tokens][H_kv][D]
 *   cache (int8)   [num_blocks][H_kv][block_size][D]
 *   scales (fp32)  [num_blocks][H_kv][block_size]
 *   q (bf16 bits)  [B][H_q][D]
 *   block_tables   int32 [B][max_blocks_per_seq]
 *   out (fp64)     [B][H_q][D]
 *
 * Build: gcc -O2 -std=c99 -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NONFINITE 2
#define ORACLE_NOMEM 3

/* bf16 is the top half of an IEEE binary32. */
static float bf16_bits_to_float(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/*
 * Quantise one tensor (K or V) of new tokens and write it into the paged
 * cache through slot_mapping (slot = physical_block * block_size + offset;
 * a negative slot means "padding, skip this token").
 * Returns ORACLE_OK, ORACLE_BAD_ARG (slot out of range) or ORACLE_NONFINITE.
 */
int oracle_quantize_append(const uint16_t *x, const int64_t *slot_mapping,
                           int64_t n_tokens, int32_t num_kv_heads,
                           int32_t head_dim, int32_t block_size,
                           int64_t num_blocks, int8_t *cache, float *scales)
{
    if (n_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < n_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        int64_t blk = slot / block_size;
        int64_t off = slot % block_size;
        if (blk >= num_blocks)
            return ORACLE_BAD_ARG;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            const uint16_t *row = x + (i * num_kv_heads + h) * (int64_t)head_dim;
            /* step 1-2: amax over the head's d values, exact in fp32 */
            float a = 0.0f;
            for (int32_t j = 0; j < head_dim; ++j) {
                float v = bf16_bits_to_float(row[j]);
                if (!isfinite(v))
                    return ORACLE_NONFINITE;
                float m = fabsf(v);
                if (m > a)
                    a = m;
            }
            /* step 3-4: the scale, one IEEE single division */
            float s = (a == 0.0f) ? 0.0f : a / 127.0f;
            int64_t base = (blk * num_kv_heads + h) * (int64_t)block_size + off;
            int8_t *dst = cache + base * head_dim;
            /* step 5-6: code = clamp(rint(x / s)) */
            for (int32_t j = 0; j < head_dim; ++j) {
                int code = 0;
                if (s != 0.0f) {
                    float y = bf16_bits_to_float(row[j]) / s;
                    float r = nearbyintf(y); /* default mode: ties to even */
                    if (r > 127.0f)
                        r = 127.0f;
                    if (r < -127.0f)
                        r = -127.0f;
                    code = (int)r;
                }
                dst[j] = (int8_t)code;
            }
            /* step 7: the scale beside the codes */
            scales[base] = s;
        }
    }
    return ORACLE_OK;
}

/*
 * Exact attention of one query row over the first n tokens of sequence b's
 * paged cache (KV head kvh), fp64.  out_row receives head_dim doubles; n == 0
 * gives a zero row.
 */
/*
 * Code j of the cache row starting at row index `base` (row = one token of
 * one KV head): an int8 code (bits == 8), or the nibble of an INT4 row
 * (bits == 4; head_dim / 2 bytes per row, dims 2i / 2i+1 in the low / high
 * nibble of byte i, stored as code + 8).
 */
static int code_at(const void *cache, int64_t base, int32_t head_dim,
                   int32_t bits, int32_t j)
{
    if (bits == 8)
        return ((const int8_t *)cache)[base * head_dim + j];
    uint8_t byte = ((const uint8_t *)cache)[base * (head_dim / 2) + j / 2];
    int nib = (j & 1) ? (byte >> 4) : (byte & 15);
    return nib - 8;
}

static int attend_row_bits(const uint16_t *qrow, const void *k_cache,
                           const void *v_cache, const float *k_scales,
                           const float *v_scales, const int32_t *block_tables,
                           int32_t num_kv_heads, int32_t head_dim,
                           int32_t block_size, int32_t max_blocks_per_seq,
                           int64_t num_blocks, double softmax_scale, int32_t b,
                           int32_t kvh, int32_t n, int32_t bits,
                           double *out_row)
{
    for (int32_t j = 0; j < head_dim; ++j)
        out_row[j] = 0.0;
    if (n == 0)
        return ORACLE_OK;
    if (n < 0 || n > max_blocks_per_seq * block_size)
        return ORACLE_BAD_ARG;

    double *score = (double *)malloc(sizeof(double) * (size_t)n);
    if (!score)
        return ORACLE_NOMEM;

    /* scores: softmax_scale * sum_j q_j * (kc * ks) */
    double smax = -INFINITY;
    for (int32_t t = 0; t < n; ++t) {
        int64_t phys = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
        int64_t off = t % block_size;
        if (phys < 0 || phys >= num_blocks) {
            free(score);
            return ORACLE_BAD_ARG;
        }
        int64_t base = (phys * num_kv_heads + kvh) * (int64_t)block_size + off;
        double ks = (double)k_scales[base];
        double dot = 0.0;
        for (int32_t j = 0; j < head_dim; ++j)
            dot += (double)bf16_bits_to_float(qrow[j]) *
                   ((double)code_at(k_cache, base, head_dim, bits, j) * ks);
        score[t] = softmax_scale * dot;
        if (score[t] > smax)
            smax = score[t];
    }
    /* softmax weights and the weighted sum of dequantised V rows */
    double denom = 0.0;
    for (int32_t t = 0; t < n; ++t) {
        score[t] = exp(score[t] - smax);
        denom += score[t];
    }
    for (int32_t t = 0; t < n; ++t) {
        int64_t phys = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
        int64_t off = t % block_size;
        int64_t base = (phys * num_kv_heads + kvh) * (int64_t)block_size + off;
        double vs = (double)v_scales[base];
        double w = score[t] / denom;
        for (int32_t j = 0; j < head_dim; ++j)
            out_row[j] += w * ((double)code_at(v_cache, base, head_dim, bits, j) * vs);
    }
    free(score);
    for (int32_t j = 0; j < head_dim; ++j)
        if (!isfinite(out_row[j]))
            return ORACLE_NONFINITE;
    return ORACLE_OK;
}

static int attend_row(const uint16_t *qrow, const int8_t *k_cache,
                      const int8_t *v_cache, const float *k_scales,
                      const float *v_scales, const int32_t *block_tables,
                      int32_t num_kv_heads, int32_t head_dim,
                      int32_t block_size, int32_t max_blocks_per_seq,
                      int64_t num_blocks, double softmax_scale, int32_t b,
                      int32_t kvh, int32_t n, double *out_row)
{
    return attend_row_bits(qrow, k_cache, v_cache, k_scales, v_scales,
                           block_tables, num_kv_heads, head_dim, block_size,
                           max_blocks_per_seq, num_blocks, softmax_scale, b,
                           kvh, n, 8, out_row);
}

/*
 * Exact decode attention for one (sequence b, query head h), fp64: the
 * sequence's one query row over all context_lens[b] cached tokens.
 */
static int attend_one(const uint16_t *q, const int8_t *k_cache,
                      const int8_t *v_cache, const float *k_scales,
                      const float *v_scales, const int32_t *block_tables,
                      const int32_t *context_lens, int32_t num_q_heads,
                      int32_t num_kv_heads, int32_t head_dim,
                      int32_t block_size, int32_t max_blocks_per_seq,
                      int64_t num_blocks, double softmax_scale, int32_t b,
                      int32_t h, double *out_row)
{
    int32_t group = num_q_heads / num_kv_heads;
    const uint16_t *qrow = q + ((int64_t)b * num_q_heads + h) * head_dim;
    return attend_row(qrow, k_cache, v_cache, k_scales, v_scales, block_tables,
                      num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                      num_blocks, softmax_scale, b, h / group, context_lens[b],
                      out_row);
}

/*
 * Decode attention for a list of (b, h) pairs (pairs = 2*n_pairs int32, NULL
 * meaning every pair in row-major order).  out holds n_pairs * head_dim
 * doubles (B * H_q * head_dim when pairs == NULL).
 * softmax_scale <= 0 selects 1/sqrt(head_dim).
 */
int oracle_decode_attention(const uint16_t *q, const int8_t *k_cache,
                            const int8_t *v_cache, const float *k_scales,
                            const float *v_scales, const int32_t *block_tables,
                            const int32_t *context_lens, int32_t batch,
                            int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t head_dim, int32_t block_size,
                            int32_t max_blocks_per_seq, int64_t num_blocks,
                            double softmax_scale, const int32_t *pairs,
                            int64_t n_pairs, double *out)
{
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_q_heads % num_kv_heads != 0)
        return ORACLE_BAD_ARG;
    if (softmax_scale <= 0.0)
        softmax_scale = 1.0 / sqrt((double)head_dim);
    int64_t count = pairs ? n_pairs : (int64_t)batch * num_q_heads;
    for (int64_t p = 0; p < count; ++p) {
        int32_t b, h;
        if (pairs) {
            b = pairs[2 * p];
            h = pairs[2 * p + 1];
        } else {
            b = (int32_t)(p / num_q_heads);
            h = (int32_t)(p % num_q_heads);
        }
        if (b < 0 || b >= batch || h < 0 || h >= num_q_heads)
            return ORACLE_BAD_ARG;
        int rc = attend_one(q, k_cache, v_cache, k_scales, v_scales,
                            block_tables, context_lens, num_q_heads,
                            num_kv_heads, head_dim, block_size,
                            max_blocks_per_seq, num_blocks, softmax_scale, b, h,
                            out + p * head_dim);
        if (rc != ORACLE_OK)
            return rc;
    }
    return ORACLE_OK;
}

/*
 * Extend (prefill) attention over the paged cache, fp64
 * [KV Cache 优化全景解析, §2.2 Prefill 与 Decode 两阶段: the prompt's tokens
 * are processed together and fill the cache; §11.2 chunked prefill: a long
 * prompt enters in chunks, each attending to everything cached before it].
 * Sequence b has n_new_b = q_start[b+1] - q_start[b] new query tokens, the
 * last n_new_b of its context_lens[b] cached tokens (appended before the
 * call, as in decode).  Query row i of sequence b sits at position
 * p = context_lens[b] - n_new_b + i and attends causally to cached tokens
 * 0..p, i.e. to the first p + 1 tokens [same page, §2.1: softmax(QK^T /
 * sqrt(d)) V; causal because generation sees only earlier tokens].
 *   q   (bf16 bits) [q_start[batch]][H_q][D], rows packed by sequence
 *   out (fp64)      [q_start[batch]][H_q][D]
 * Returns ORACLE_BAD_ARG when n_new_b > context_lens[b] or q_start is not
 * non-decreasing from 0.
 */
int oracle_extend_attention(const uint16_t *q, const int8_t *k_cache,
                            const int8_t *v_cache, const float *k_scales,
                            const float *v_scales, const int32_t *block_tables,
                            const int32_t *context_lens, const int32_t *q_start,
                            int32_t batch, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim,
                            int32_t block_size, int32_t max_blocks_per_seq,
                            int64_t num_blocks, double softmax_scale,
                            double *out)
{
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_q_heads % num_kv_heads != 0 || q_start[0] != 0)
        return ORACLE_BAD_ARG;
    if (softmax_scale <= 0.0)
        softmax_scale = 1.0 / sqrt((double)head_dim);
    int32_t group = num_q_heads / num_kv_heads;
    for (int32_t b = 0; b < batch; ++b) {
        int32_t n_new = q_start[b + 1] - q_start[b];
        if (n_new < 0 || n_new > context_lens[b])
            return ORACLE_BAD_ARG;
        for (int32_t i = 0; i < n_new; ++i) {
            int64_t row = (int64_t)q_start[b] + i;
            int32_t keys = context_lens[b] - n_new + i + 1;
            for (int32_t h = 0; h < num_q_heads; ++h) {
                const uint16_t *qrow = q + (row * num_q_heads + h) * head_dim;
                double *orow = out + (row * num_q_heads + h) * head_dim;
                int rc = attend_row(qrow, k_cache, v_cache, k_scales, v_scales,
                                    block_tables, num_kv_heads, head_dim,
                                    block_size, max_blocks_per_seq, num_blocks,
                                    softmax_scale, b, h / group, keys, orow);
                if (rc != ORACLE_OK)
                    return rc;
            }
        }
    }
    return ORACLE_OK;
}

/*
 * INT4 variant of the cache.  The K/V of historical tokens are quantised to
 * 4 bits [nano-KvLLM, §2.2 量化感知缓存]; INT4 takes 0.5 byte per element
 * [KV Cache 优化全景解析, §2.3 table].  Readings (the pages give no formula):
 * the same symmetric per-(token, KV head) scheme as INT8 with 7 levels each
 * side, s = fl32(max|x| / 7) (IEEE division; s = 0 for an all-zero row),
 * c_j = clamp(rint(fl32(x_j / s)), -7, 7) (ties to even; 0 when s == 0).
 * Storage: the nibble c_j + 8 (1..15; 8 for a zero row), dims 2i and 2i+1
 * in the low and high nibble of byte i; cache [num_blocks][H_kv][BS][D/2]
 * bytes, scales [num_blocks][H_kv][BS] fp32.
 */
int oracle_quantize_append_int4(const uint16_t *x, const int64_t *slot_mapping,
                                int64_t n_tokens, int32_t num_kv_heads,
                                int32_t head_dim, int32_t block_size,
                                int64_t num_blocks, uint8_t *cache,
                                float *scales)
{
    if (n_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || (head_dim & 1))
        return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < n_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        int64_t blk = slot / block_size;
        int64_t off = slot % block_size;
        if (blk >= num_blocks)
            return ORACLE_BAD_ARG;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            const uint16_t *row = x + (i * num_kv_heads + h) * (int64_t)head_dim;
            float a = 0.0f;
            for (int32_t j = 0; j < head_dim; ++j) {
                float v = bf16_bits_to_float(row[j]);
                if (!isfinite(v))
                    return ORACLE_NONFINITE;
                float m = fabsf(v);
                if (m > a)
                    a = m;
            }
            float s = (a == 0.0f) ? 0.0f : a / 7.0f;
            int64_t base = (blk * num_kv_heads + h) * (int64_t)block_size + off;
            uint8_t *dst = cache + base * (head_dim / 2);
            for (int32_t j = 0; j < head_dim; j += 2) {
                int nib[2];
                for (int k = 0; k < 2; ++k) {
                    int code = 0;
                    if (s != 0.0f) {
                        float y = bf16_bits_to_float(row[j + k]) / s;
                        float r = nearbyintf(y);
                        if (r > 7.0f)
                            r = 7.0f;
                        if (r < -7.0f)
                            r = -7.0f;
                        code = (int)r;
                    }
                    nib[k] = code + 8;
                }
                dst[j / 2] = (uint8_t)(nib[0] | (nib[1] << 4));
            }
            scales[base] = s;
        }
    }
    return ORACLE_OK;
}

/*
 * Decode attention over the INT4 cache, fp64: as oracle_decode_attention,
 * with k_hat = (nibble - 8) * ks and v_hat = (nibble - 8) * vs.
 */
int oracle_decode_attention_int4(const uint16_t *q, const uint8_t *k_cache,
                                 const uint8_t *v_cache, const float *k_scales,
                                 const float *v_scales,
                                 const int32_t *block_tables,
                                 const int32_t *context_lens, int32_t batch,
                                 int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t block_size,
                                 int32_t max_blocks_per_seq, int64_t num_blocks,
                                 double softmax_scale, double *out)
{
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_q_heads % num_kv_heads != 0 || (head_dim & 1))
        return ORACLE_BAD_ARG;
    if (softmax_scale <= 0.0)
        softmax_scale = 1.0 / sqrt((double)head_dim);
    int32_t group = num_q_heads / num_kv_heads;
    for (int32_t b = 0; b < batch; ++b)
        for (int32_t h = 0; h < num_q_heads; ++h) {
            const uint16_t *qrow = q + ((int64_t)b * num_q_heads + h) * head_dim;
            int rc = attend_row_bits(qrow, k_cache, v_cache, k_scales, v_scales,
                                     block_tables, num_kv_heads, head_dim,
                                     block_size, max_blocks_per_seq, num_blocks,
                                     softmax_scale, b, h / group,
                                     context_lens[b], 4,
                                     out + ((int64_t)b * num_q_heads + h) * head_dim);
            if (rc != ORACLE_OK)
                return rc;
        }
    return ORACLE_OK;
}

/*
 * The KIVI variant of the cache: 2-bit asymmetric codes, keys grouped per
 * channel and values per token [KV Cache 优化全景解析——从基础原理到工程实践,
 * §7.1 量化的核心挑战 (keys differ strongly between channels, values are even
 * within a token) and §7.2 KIVI：2bit 无损非对称量化 (2-bit asymmetric codes,
 * K per channel, V per token)].  The page fixes the axes, the width and the
 * asymmetry and nothing else; these readings fill the rest:
 *   - a group is quantised by its minimum z and its range:
 *       s = fl32(fl32(max - z) / 3)
 *       c = clamp(rint(fl32(fl32(x - z) / s)), 0, 3)  (ties to even)
 *     with s = 0 and every c = 0 when the group is constant, and
 *     dequantised as x_hat = c * s + z (exact in double);
 *   - a key group is one channel of one page (16 tokens of one KV head):
 *     the block the block table maps, so a group never spans pages;
 *   - a page is quantised when its 16th token arrives; until then its
 *     tokens' K and V rows stay in bf16 in the sequence's tail ("recent
 *     tokens keep their original precision", [nano-KvLLM, §2.2 量化感知缓存]),
 *     and attention reads them there exactly;
 *   - values are quantised per token at the same moment as the page's keys.
 *
 * Plain layouts (one code per byte; the library packs its own):
 *   k_codes, v_codes  uint8 [num_blocks][H_kv][BS][D]
 *   k_scale, k_zero   fp32  [num_blocks][H_kv][D]    (per channel)
 *   v_scale, v_zero   fp32  [num_blocks][H_kv][BS]   (per token)
 *   tail (bf16 bits)  [batch][H_kv][2][BS][D]        (K rows, then V rows)
 */

/* Asymmetric 2-bit quantisation of one group of n values x[i * stride]. */
static int kivi_quantise_group(const float *x, int32_t n, int64_t stride,
                               uint8_t *codes, int64_t code_stride,
                               float *scale, float *zero)
{
    float lo = x[0], hi = x[0];
    for (int32_t i = 1; i < n; ++i) {
        float v = x[i * stride];
        if (v < lo)
            lo = v;
        if (v > hi)
            hi = v;
    }
    float s = (hi - lo) / 3.0f;
    if (!isfinite(s))
        return ORACLE_NONFINITE;
    for (int32_t i = 0; i < n; ++i) {
        int code = 0;
        if (s != 0.0f) {
            float y = (x[i * stride] - lo) / s;
            float r = nearbyintf(y);
            if (r > 3.0f)
                r = 3.0f;
            if (r < 0.0f)
                r = 0.0f;
            code = (int)r;
        }
        codes[i * code_stride] = (uint8_t)code;
    }
    *scale = s;
    *zero = lo;
    return ORACLE_OK;
}

/*
 * Quantise the full page that sequence b's tail holds (all heads) into
 * physical block blk: keys per channel over the 16 tokens, values per token
 * over the D channels.
 */
static int kivi_quantise_page(const uint16_t *tail_b, int32_t num_kv_heads,
                              int32_t head_dim, int32_t block_size,
                              int64_t blk, uint8_t *k_codes, float *k_scale,
                              float *k_zero, uint8_t *v_codes, float *v_scale,
                              float *v_zero)
{
    const int64_t row_elems = (int64_t)block_size * head_dim;
    float *x = (float *)malloc(sizeof(float) * (size_t)row_elems);
    if (!x)
        return ORACLE_NOMEM;
    int rc = ORACLE_OK;
    for (int32_t h = 0; h < num_kv_heads && rc == ORACLE_OK; ++h) {
        const int64_t page = blk * num_kv_heads + h;
        for (int kv = 0; kv < 2 && rc == ORACLE_OK; ++kv) {
            const uint16_t *rows = tail_b + ((int64_t)h * 2 + kv) * row_elems;
            for (int64_t i = 0; i < row_elems; ++i) {
                x[i] = bf16_bits_to_float(rows[i]);
                if (!isfinite(x[i]))
                    rc = ORACLE_NONFINITE;
            }
            if (rc != ORACLE_OK)
                break;
            if (kv == 0) {
                /* keys: one group per channel j, tokens t = 0..BS-1 */
                for (int32_t j = 0; j < head_dim && rc == ORACLE_OK; ++j)
                    rc = kivi_quantise_group(
                        x + j, block_size, head_dim,
                        k_codes + page * row_elems + j, head_dim,
                        &k_scale[page * head_dim + j],
                        &k_zero[page * head_dim + j]);
            } else {
                /* values: one group per token t, channels j = 0..D-1 */
                for (int32_t t = 0; t < block_size && rc == ORACLE_OK; ++t)
                    rc = kivi_quantise_group(
                        x + (int64_t)t * head_dim, head_dim, 1,
                        v_codes + page * row_elems + (int64_t)t * head_dim, 1,
                        &v_scale[page * block_size + t],
                        &v_zero[page * block_size + t]);
            }
        }
    }
    free(x);
    return rc;
}

/*
 * Append new tokens to the KIVI cache, one token at a time in position
 * order.  Sequence b gets the n_b = cu_new[b+1] - cu_new[b] rows
 * k_new/v_new[cu_new[b] .. cu_new[b+1]) (bf16 bits, [*][H_kv][D]) at
 * positions context_lens[b] - n_b .. context_lens[b] - 1 (context_lens
 * counts them).  Each row goes to tail row (position % BS); when a position
 * completes a page (position % BS == BS - 1) the tail's page is quantised
 * into block block_tables[b][position / BS].  Returns ORACLE_BAD_ARG for
 * n_b < 0, n_b > context_lens[b], a context longer than the table or a
 * block out of range; ORACLE_NONFINITE for a non-finite input or scale.
 */
int oracle_kivi_append(const uint16_t *k_new, const uint16_t *v_new,
                       const int32_t *cu_new, const int32_t *context_lens,
                       const int32_t *block_tables, int32_t batch,
                       int32_t num_kv_heads, int32_t head_dim,
                       int32_t block_size, int32_t max_blocks_per_seq,
                       int64_t num_blocks, uint8_t *k_codes, float *k_scale,
                       float *k_zero, uint8_t *v_codes, float *v_scale,
                       float *v_zero, uint16_t *tail)
{
    if (batch < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        cu_new[0] != 0)
        return ORACLE_BAD_ARG;
    const int64_t row_elems = (int64_t)block_size * head_dim;
    for (int32_t b = 0; b < batch; ++b) {
        const int32_t n_new = cu_new[b + 1] - cu_new[b];
        const int32_t len = context_lens[b];
        if (n_new < 0 || n_new > len ||
            len > (int64_t)max_blocks_per_seq * block_size)
            return ORACLE_BAD_ARG;
        uint16_t *tail_b = tail + (int64_t)b * num_kv_heads * 2 * row_elems;
        for (int32_t i = 0; i < n_new; ++i) {
            const int32_t pos = len - n_new + i;
            const int64_t tok = (int64_t)cu_new[b] + i;
            for (int32_t h = 0; h < num_kv_heads; ++h)
                for (int kv = 0; kv < 2; ++kv) {
                    const uint16_t *src = (kv ? v_new : k_new) +
                                          (tok * num_kv_heads + h) * head_dim;
                    uint16_t *dst = tail_b + ((int64_t)h * 2 + kv) * row_elems +
                                    (int64_t)(pos % block_size) * head_dim;
                    memcpy(dst, src, sizeof(uint16_t) * (size_t)head_dim);
                }
            if (pos % block_size == block_size - 1) {
                const int64_t blk = block_tables[(int64_t)b * max_blocks_per_seq +
                                                 pos / block_size];
                if (blk < 0 || blk >= num_blocks)
                    return ORACLE_BAD_ARG;
                int rc = kivi_quantise_page(tail_b, num_kv_heads, head_dim,
                                            block_size, blk, k_codes, k_scale,
                                            k_zero, v_codes, v_scale, v_zero);
                if (rc != ORACLE_OK)
                    return rc;
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Decode attention over the KIVI cache, fp64: as oracle_decode_attention,
 * with, for sequence b's n cached tokens and F = BS * floor(n / BS):
 *   t <  F: k_hat_t[j] = kc * k_scale[j] + k_zero[j]   (page of token t)
 *           v_hat_t[j] = vc * v_scale[t] + v_zero[t]
 *   t >= F: k_hat_t, v_hat_t = the bf16 rows in tail row t % BS.
 * out (fp64) [B][H_q][D].
 */
int oracle_kivi_decode_attention(const uint16_t *q, const uint8_t *k_codes,
                                 const float *k_scale, const float *k_zero,
                                 const uint8_t *v_codes, const float *v_scale,
                                 const float *v_zero, const uint16_t *tail,
                                 const int32_t *block_tables,
                                 const int32_t *context_lens, int32_t batch,
                                 int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t block_size,
                                 int32_t max_blocks_per_seq, int64_t num_blocks,
                                 double softmax_scale, double *out)
{
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_q_heads % num_kv_heads != 0)
        return ORACLE_BAD_ARG;
    if (softmax_scale <= 0.0)
        softmax_scale = 1.0 / sqrt((double)head_dim);
    const int32_t group = num_q_heads / num_kv_heads;
    const int64_t row_elems = (int64_t)block_size * head_dim;
    for (int32_t b = 0; b < batch; ++b) {
        const int32_t n = context_lens[b];
        if (n < 0 || n > (int64_t)max_blocks_per_seq * block_size)
            return ORACLE_BAD_ARG;
        const int32_t full = n / block_size * block_size;
        double *khat = (double *)malloc(sizeof(double) * (size_t)(n + 1) * head_dim);
        double *vhat = (double *)malloc(sizeof(double) * (size_t)(n + 1) * head_dim);
        double *score = (double *)malloc(sizeof(double) * (size_t)(n + 1));
        if (!khat || !vhat || !score) {
            free(khat);
            free(vhat);
            free(score);
            return ORACLE_NOMEM;
        }
        for (int32_t kvh = 0; kvh < num_kv_heads; ++kvh) {
            /* the dequantised rows of this KV head */
            for (int32_t t = 0; t < n; ++t) {
                const int32_t r = t % block_size;
                for (int32_t j = 0; j < head_dim; ++j) {
                    double kx, vx;
                    if (t < full) {
                        const int64_t blk =
                            block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
                        if (blk < 0 || blk >= num_blocks) {
                            free(khat);
                            free(vhat);
                            free(score);
                            return ORACLE_BAD_ARG;
                        }
                        const int64_t page = blk * num_kv_heads + kvh;
                        const int64_t at = page * row_elems + (int64_t)r * head_dim + j;
                        kx = (double)k_codes[at] * (double)k_scale[page * head_dim + j] +
                             (double)k_zero[page * head_dim + j];
                        vx = (double)v_codes[at] * (double)v_scale[page * block_size + r] +
                             (double)v_zero[page * block_size + r];
                    } else {
                        const uint16_t *tb =
                            tail + ((int64_t)b * num_kv_heads + kvh) * 2 * row_elems;
                        kx = (double)bf16_bits_to_float(tb[(int64_t)r * head_dim + j]);
                        vx = (double)bf16_bits_to_float(
                            tb[row_elems + (int64_t)r * head_dim + j]);
                    }
                    khat[(int64_t)t * head_dim + j] = kx;
                    vhat[(int64_t)t * head_dim + j] = vx;
                }
            }
            for (int32_t g = 0; g < group; ++g) {
                const int32_t h = kvh * group + g;
                const uint16_t *qrow = q + ((int64_t)b * num_q_heads + h) * head_dim;
                double *orow = out + ((int64_t)b * num_q_heads + h) * head_dim;
                for (int32_t j = 0; j < head_dim; ++j)
                    orow[j] = 0.0;
                if (n == 0)
                    continue;
                double smax = -INFINITY;
                for (int32_t t = 0; t < n; ++t) {
                    double dot = 0.0;
                    for (int32_t j = 0; j < head_dim; ++j)
                        dot += (double)bf16_bits_to_float(qrow[j]) *
                               khat[(int64_t)t * head_dim + j];
                    score[t] = softmax_scale * dot;
                    if (score[t] > smax)
                        smax = score[t];
                }
                double denom = 0.0;
                for (int32_t t = 0; t < n; ++t) {
                    score[t] = exp(score[t] - smax);
                    denom += score[t];
                }
                for (int32_t t = 0; t < n; ++t)
                    for (int32_t j = 0; j < head_dim; ++j)
                        orow[j] += score[t] / denom * vhat[(int64_t)t * head_dim + j];
                for (int32_t j = 0; j < head_dim; ++j)
                    if (!isfinite(orow[j])) {
                        free(khat);
                        free(vhat);
                        free(score);
                        return ORACLE_NONFINITE;
                    }
            }
        }
        free(khat);
        free(vhat);
        free(score);
    }
    return ORACLE_OK;
}

/*
 * KV-cache size closed form [KV Cache 优化全景解析, §2.3]:
 *   2 * L * B * T * H_kv * d_h * bytes_per_element,
 * with bytes_per_element = elem_bytes_num / elem_bytes_den (INT4 = 1/2).
 * Returned as a double (exact for every value below 2^53).
 */
double oracle_kv_cache_bytes(int64_t layers, int64_t batch, int64_t seq_len,
                             int64_t kv_heads, int64_t head_dim,
                             int64_t elem_bytes_num, int64_t elem_bytes_den)
{
    double elems = 2.0 * (double)layers * (double)batch * (double)seq_len *
                   (double)kv_heads * (double)head_dim;
    return elems * (double)elem_bytes_num / (double)elem_bytes_den;
}

/*
 * Extra bytes the INT8 format spends on its fp32 scales: one per
 * (K or V, layer, sequence, token, KV head).  Not part of the page formula.
 */
double oracle_kv8_scale_bytes(int64_t layers, int64_t batch, int64_t seq_len,
                              int64_t kv_heads)
{
    return 2.0 * (double)layers * (double)batch * (double)seq_len *
           (double)kv_heads * 4.0;
}
