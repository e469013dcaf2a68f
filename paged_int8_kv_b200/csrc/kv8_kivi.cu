// kv8_kivi.cu -- the KIVI variant of the paged cache: 2-bit asymmetric
// codes, keys grouped per channel and values per token [KV Cache 优化全景解析
// ——从基础原理到工程实践, §7.1 量化的核心挑战 (keys differ between channels,
// values are even within a token) and §7.2 KIVI：2bit 无损非对称量化].
//
// A group of values x is stored as its minimum z, a scale
// s = fl32(fl32(max - z) / 3) and codes c = clamp(rint(fl32(fl32(x - z) / s)),
// 0, 3) (s = 0 and c = 0 for a constant group); x_hat = c s + z.  A key group
// is one channel of one 16-token page, so a page can only be quantised once
// its 16th token has arrived: until then the page's K and V rows stay in bf16
// in the sequence's tail, and attention reads them there as they are (recent
// tokens at their original precision [nano-KvLLM, §2.2 量化感知缓存]).
//
// Page record, one per (block, KV head), 2176 bytes (16-byte aligned):
//   [   0,  512)  K codes: 128 words of 32 bits, word j = channel j, token t
//                 in bits 2t, 2t+1
//   [ 512, 1024)  V codes: the same layout
//   [1024, 1536)  K scales, fp32 [128] (per channel)
//   [1536, 2048)  K zero points, fp32 [128]
//   [2048, 2112)  V scales, fp32 [16] (per token)
//   [2112, 2176)  V zero points, fp32 [16]
// Channel-major codes give lane l of a warp the 16 bytes of channels
// 4l .. 4l+3 (all 16 tokens) in one 16-byte load.
//
// Kernels:
//   kivi_page_kernel   one warp per (sequence, page completed by this append,
//                      KV head): gathers the page's 16 K and V rows (from the
//                      tail and the new tokens), quantises, writes the record
//   kivi_tail_kernel   one warp per (sequence, KV head): copies the new rows
//                      of the sequence's last, partial page into the tail
//                      (after the page kernel, which may read the old tail)
//   kivi_decode_kernel one warp per (chunk, sequence, KV head, sub-group of
//                      up to 4 query heads), fp32 CUDA-core arithmetic with
//                      an online base-2 softmax; split chunks merge by ticket
//                      through the same log-sum-exp routine as the INT8 path.
//
// Decode arithmetic per page and head (q pre-scaled by softmax_scale log2 e):
//   score_t = sum_j q_j (s_j c_tj + z_j) = sum_j (q_j s_j) c_tj + sum_j q_j z_j
//   out    += sum_t p_t (s_t c_tj + z_t) = sum_t (p_t s_t) c_tj + sum_t p_t z_t
// Lane l holds channels 4l .. 4l+3: its partial score of every token is
// summed over the warp by a transposing butterfly (16 values, 16 shuffles),
// after which lanes 2t and 2t+1 hold token t's score.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <cmath>

#include "../../include/kv8.h"
#include "kv8_internal.h"
#include "kv8_merge.cuh"

namespace kv8 {
namespace {

constexpr int kRec = KV8_KIVI_PAGE_BYTES;  // 2176
constexpr int kOffVc = 512, kOffKs = 1024, kOffKz = 1536, kOffVs = 2048,
              kOffVz = 2112;
constexpr unsigned kAll = 0xffffffffu;
constexpr int kWarps = 4;  // warps per block of every KIVI kernel

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Four bf16 values at p (8-byte aligned) as floats.
__device__ __forceinline__ void load4_bf16(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
  x[0] = bf16_lo(w.x);
  x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y);
  x[3] = bf16_hi(w.y);
}

// Code of token t (bits 2t, 2t+1 of w) as an exact float: the integer in
// the low mantissa bits of 2^23, minus 2^23.
__device__ __forceinline__ float code_f(uint32_t w, int t) {
  return __uint_as_float(0x4B000000u | ((w >> (2 * t)) & 3u)) - 8388608.0f;
}

// The asymmetric 2-bit code of x in a group with minimum z and scale s.
__device__ __forceinline__ uint32_t quant2(float x, float z, float s) {
  if (s == 0.0f) return 0u;
  const float r = rintf(__fdiv_rn(__fsub_rn(x, z), s));
  return static_cast<uint32_t>(fminf(fmaxf(r, 0.0f), 3.0f));
}

// ---------------------------------------------------------------------------
// Append: pages completed by this call.
// ---------------------------------------------------------------------------
struct AppendArgs {
  const __nv_bfloat16* k_new;  // [cu_new[B]][H][128]
  const __nv_bfloat16* v_new;
  const int32_t* cu_new;        // [B + 1]
  const int32_t* context_lens;  // [B], after the append
  const int32_t* block_tables;  // [B][MBS]
  uint8_t* cache;               // [NB][H] page records
  __nv_bfloat16* tail;          // [B][H][2][16][128]
  int32_t num_kv_heads;
  int32_t max_blocks_per_seq;
};

__global__ void __launch_bounds__(kWarps * 32)
kivi_page_kernel(AppendArgs a) {
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x;  // b * H + kvh
  const int b = bh / a.num_kv_heads, kvh = bh - b * a.num_kv_heads;
  const int len = a.context_lens[b];
  const int nn = a.cu_new[b + 1] - a.cu_new[b];
  const int start = len - nn;  // first position appended by this call
  // nothing appended; or counts the caller's contract rules out (kept off
  // the block table's bounds)
  if (nn <= 0 || start < 0 ||
      static_cast<int64_t>(len) > static_cast<int64_t>(a.max_blocks_per_seq) * kBlockSize)
    return;
  const int j_end = len / kBlockSize;  // pages below are full after the call
  const int stride = gridDim.y * kWarps;
  const __nv_bfloat16* tail_k =
      a.tail + static_cast<int64_t>(bh) * 2 * kBlockSize * kHeadDim;
  const __nv_bfloat16* tail_v = tail_k + kBlockSize * kHeadDim;
  for (int j = start / kBlockSize + blockIdx.y * kWarps + (threadIdx.x >> 5);
       j < j_end; j += stride) {
    const int64_t blk = a.block_tables[static_cast<int64_t>(b) * a.max_blocks_per_seq + j];
    uint8_t* rec = a.cache + (blk * a.num_kv_heads + kvh) * kRec;
    // row r of the page: from the tail if appended before this call
    auto row_ptr = [&](const __nv_bfloat16* fresh, const __nv_bfloat16* old,
                       int r) -> const __nv_bfloat16* {
      const int pos = j * kBlockSize + r;
      if (pos < start) return old + r * kHeadDim + 4 * lane;
      const int64_t tok = a.cu_new[b] + (pos - start);
      return fresh + (tok * a.num_kv_heads + kvh) * kHeadDim + 4 * lane;
    };
    float x[kBlockSize][4];
    // keys: one group per channel (lane-local over the 16 rows)
#pragma unroll
    for (int r = 0; r < kBlockSize; ++r) load4_bf16(row_ptr(a.k_new, tail_k, r), x[r]);
    {
      uint32_t w[4];
      float s[4], z[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float lo = x[0][i], hi = x[0][i];
#pragma unroll
        for (int r = 1; r < kBlockSize; ++r) {
          lo = fminf(lo, x[r][i]);
          hi = fmaxf(hi, x[r][i]);
        }
        s[i] = __fdiv_rn(__fsub_rn(hi, lo), 3.0f);
        z[i] = lo;
        w[i] = 0u;
#pragma unroll
        for (int r = 0; r < kBlockSize; ++r) w[i] |= quant2(x[r][i], lo, s[i]) << (2 * r);
      }
      *reinterpret_cast<uint4*>(rec + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<float4*>(rec + kOffKs + 16 * lane) = make_float4(s[0], s[1], s[2], s[3]);
      *reinterpret_cast<float4*>(rec + kOffKz + 16 * lane) = make_float4(z[0], z[1], z[2], z[3]);
    }
    // values: one group per token (a warp-wide min / max of each row)
#pragma unroll
    for (int r = 0; r < kBlockSize; ++r) load4_bf16(row_ptr(a.v_new, tail_v, r), x[r]);
    {
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      float my_s = 0.0f, my_z = 0.0f;
#pragma unroll
      for (int r = 0; r < kBlockSize; ++r) {
        float lo = fminf(fminf(x[r][0], x[r][1]), fminf(x[r][2], x[r][3]));
        float hi = fmaxf(fmaxf(x[r][0], x[r][1]), fmaxf(x[r][2], x[r][3]));
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
          lo = fminf(lo, __shfl_xor_sync(kAll, lo, m));
          hi = fmaxf(hi, __shfl_xor_sync(kAll, hi, m));
        }
        const float s = __fdiv_rn(__fsub_rn(hi, lo), 3.0f);
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] |= quant2(x[r][i], lo, s) << (2 * r);
        if (lane == r) {
          my_s = s;
          my_z = lo;
        }
      }
      *reinterpret_cast<uint4*>(rec + kOffVc + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
      if (lane < kBlockSize) {
        reinterpret_cast<float*>(rec + kOffVs)[lane] = my_s;
        reinterpret_cast<float*>(rec + kOffVz)[lane] = my_z;
      }
    }
  }
}

// The new rows of each sequence's last, partial page, into its tail.
__global__ void __launch_bounds__(32) kivi_tail_kernel(AppendArgs a) {
  const int lane = threadIdx.x;
  const int bh = blockIdx.x;
  const int b = bh / a.num_kv_heads, kvh = bh - b * a.num_kv_heads;
  const int len = a.context_lens[b];
  const int nn = a.cu_new[b + 1] - a.cu_new[b];
  const int start = len - nn;
  if (nn <= 0 || start < 0) return;
  const int first = max(start, len / kBlockSize * kBlockSize);
  __nv_bfloat16* tk = a.tail + static_cast<int64_t>(bh) * 2 * kBlockSize * kHeadDim;
  __nv_bfloat16* tv = tk + kBlockSize * kHeadDim;
  for (int pos = first; pos < len; ++pos) {
    const int64_t tok = a.cu_new[b] + (pos - start);
    const int64_t src = (tok * a.num_kv_heads + kvh) * kHeadDim + 4 * lane;
    const int dst = (pos % kBlockSize) * kHeadDim + 4 * lane;
    *reinterpret_cast<uint2*>(tk + dst) = __ldg(reinterpret_cast<const uint2*>(a.k_new + src));
    *reinterpret_cast<uint2*>(tv + dst) = __ldg(reinterpret_cast<const uint2*>(a.v_new + src));
  }
}

// ---------------------------------------------------------------------------
// Decode.
// ---------------------------------------------------------------------------
struct KiviDecode {
  const __nv_bfloat16* q;       // [B][Hq][128]
  const uint8_t* cache;         // [NB][H] page records
  const __nv_bfloat16* tail;    // [B][H][2][16][128]
  const int32_t* block_tables;  // [B][MBS]
  const int32_t* context_lens;  // [B]
  float* ws_ml;                 // [B][Hq][max_chunks][2]
  float* ws_o;                  // [B][Hq][max_chunks][128]
  uint32_t* ws_ctr;             // [B][Hq] tickets, zero at launch
  void* out;                    // [B][Hq][128]
  int32_t batch, num_q_heads, num_kv_heads, max_blocks_per_seq;
  int32_t chunk_tokens;         // > 0, multiple of 16
  int32_t max_chunks;
  int32_t subs;                 // sub-groups of query heads per KV head
  int32_t out_f32;
  float q_scale;                // softmax_scale * log2(e)
  int64_t items;                // max_chunks * B * H * subs
};

// Sum of v[0..15] over the warp, transposed: lane l returns the total of
// token (l >> 1).  Each step halves the values a lane keeps: it keeps the
// half its lane bit selects and adds the partner's copy of that half.
__device__ __forceinline__ float reduce16(const float (&v)[16], int lane) {
  float w[8], x[4], y[2];
  bool h = lane & 16;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float send = h ? v[i] : v[i + 8];
    w[i] = (h ? v[i + 8] : v[i]) + __shfl_xor_sync(kAll, send, 16);
  }
  h = lane & 8;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = h ? w[i] : w[i + 4];
    x[i] = (h ? w[i + 4] : w[i]) + __shfl_xor_sync(kAll, send, 8);
  }
  h = lane & 4;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = h ? x[i] : x[i + 2];
    y[i] = (h ? x[i + 2] : x[i]) + __shfl_xor_sync(kAll, send, 4);
  }
  h = lane & 2;
  const float send = h ? y[0] : y[1];
  float z = (h ? y[1] : y[0]) + __shfl_xor_sync(kAll, send, 2);
  return z + __shfl_xor_sync(kAll, z, 1);
}

// One quantised page's registers (lane l: channels 4l .. 4l+3; token l >> 1
// for the per-token values).
struct PageRegs {
  uint4 kw, vw;
  float4 ks, kz;
  float vs, vz;
};

__device__ __forceinline__ PageRegs load_page(const uint8_t* rec, int lane) {
  PageRegs r;
  r.kw = __ldg(reinterpret_cast<const uint4*>(rec) + lane);
  r.vw = __ldg(reinterpret_cast<const uint4*>(rec + kOffVc) + lane);
  r.ks = __ldg(reinterpret_cast<const float4*>(rec + kOffKs) + lane);
  r.kz = __ldg(reinterpret_cast<const float4*>(rec + kOffKz) + lane);
  r.vs = __ldg(reinterpret_cast<const float*>(rec + kOffVs) + (lane >> 1));
  r.vz = __ldg(reinterpret_cast<const float*>(rec + kOffVz) + (lane >> 1));
  return r;
}

// Online-softmax state of G query heads.
template <int G>
struct HeadState {
  float q[G][4];    // q * q_scale, channels 4l .. 4l+3
  float m[G];       // running base-2 max
  float l[G];       // running sum of 2^(s - m)
  float acc[G][4];  // running sum of 2^(s - m) v_hat
};

// The softmax step of one page for G heads, given every head's token score
// `sc` (lane l: token l >> 1, -inf when masked), the token's V scale and
// zero point (1 and 0 for bf16 rows).  Returns the per-token weights w that
// multiply the codes (lane 2t: token t) and folds alpha and sum_t p_t z_t
// into the accumulators.
template <int G>
__device__ __forceinline__ void softmax_step(HeadState<G>& st, const float (&sc)[G],
                                             float vs, float vz, int lane,
                                             float (&w)[G]) {
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float pm = sc[g];
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) pm = fmaxf(pm, __shfl_xor_sync(kAll, pm, m));
    const float mn = fmaxf(st.m[g], pm);
    const float alpha = ex2(st.m[g] - mn);
    const float p = ex2(sc[g] - mn);
    w[g] = p * vs;
    float pe = (lane & 1) ? 0.0f : p;  // each token once
    float pz = (lane & 1) ? 0.0f : p * vz;
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
      pe += __shfl_xor_sync(kAll, pe, m);
      pz += __shfl_xor_sync(kAll, pz, m);
    }
    st.l[g] = st.l[g] * alpha + pe;
#pragma unroll
    for (int i = 0; i < 4; ++i) st.acc[g][i] = fmaf(st.acc[g][i], alpha, pz);
    st.m[g] = mn;
  }
}

template <int G>
__device__ __forceinline__ void quantised_page(HeadState<G>& st, const PageRegs& pg,
                                               int lane) {
  const float ks[4] = {pg.ks.x, pg.ks.y, pg.ks.z, pg.ks.w};
  const float kz[4] = {pg.kz.x, pg.kz.y, pg.kz.z, pg.kz.w};
  const uint32_t kw[4] = {pg.kw.x, pg.kw.y, pg.kw.z, pg.kw.w};
  const uint32_t vw[4] = {pg.vw.x, pg.vw.y, pg.vw.z, pg.vw.w};
  float u[G][4], part[G][16];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float base = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      u[g][i] = st.q[g][i] * ks[i];
      base = fmaf(st.q[g][i], kz[i], base);
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) part[g][t] = base;
  }
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    float c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = code_f(kw[i], t);
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int i = 0; i < 4; ++i) part[g][t] = fmaf(u[g][i], c[i], part[g][t]);
  }
  float sc[G], w[G];
#pragma unroll
  for (int g = 0; g < G; ++g) sc[g] = reduce16(part[g], lane);
  softmax_step<G>(st, sc, pg.vs, pg.vz, lane, w);
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    float c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = code_f(vw[i], t);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float wt = __shfl_sync(kAll, w[g], 2 * t);
#pragma unroll
      for (int i = 0; i < 4; ++i) st.acc[g][i] = fmaf(wt, c[i], st.acc[g][i]);
    }
  }
}

// The sequence's partial page: its first `valid` rows, bf16, from the tail.
template <int G>
__device__ __forceinline__ void tail_page(HeadState<G>& st, const __nv_bfloat16* tk,
                                          int valid, int lane) {
  const __nv_bfloat16* tv = tk + kBlockSize * kHeadDim;
  float part[G][16];
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (t < valid) load4_bf16(tk + t * kHeadDim + 4 * lane, x);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float s = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) s = fmaf(st.q[g][i], x[i], s);
      part[g][t] = s;
    }
  }
  float sc[G], w[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    sc[g] = reduce16(part[g], lane);
    if ((lane >> 1) >= valid) sc[g] = -INFINITY;
  }
  softmax_step<G>(st, sc, 1.0f, 0.0f, lane, w);
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (t < valid) load4_bf16(tv + t * kHeadDim + 4 * lane, x);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float wt = __shfl_sync(kAll, w[g], 2 * t);
#pragma unroll
      for (int i = 0; i < 4; ++i) st.acc[g][i] = fmaf(wt, x[i], st.acc[g][i]);
    }
  }
}

template <int G>
__global__ void __launch_bounds__(kWarps * 32)
kivi_decode_kernel(KiviDecode p) {
  const int lane = threadIdx.x & 31;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (item >= p.items) return;
  // item = ((c * B + b) * H + kvh) * subs + sub
  int64_t r = item;
  const int sub = static_cast<int>(r % p.subs);
  r /= p.subs;
  const int kvh = static_cast<int>(r % p.num_kv_heads);
  r /= p.num_kv_heads;
  const int b = static_cast<int>(r % p.batch);
  const int c = static_cast<int>(r / p.batch);
  const int h0 = (kvh * p.subs + sub) * G;
  const int64_t row0 = static_cast<int64_t>(b) * p.num_q_heads + h0;

  const int n = p.context_lens[b];
  const int nchunks = (n + p.chunk_tokens - 1) / p.chunk_tokens;
  if (n <= 0) {  // an empty context: zero rows, written by chunk 0's item
    if (c == 0)
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int i = 0; i < 4; ++i) store_out(p.out, (row0 + g) * kHeadDim + 4 * lane + i, 0.0f, p.out_f32);
    return;
  }
  if (c >= nchunks) return;
  const int t0 = c * p.chunk_tokens;
  const int t1 = min(n, t0 + p.chunk_tokens);
  const int full = n / kBlockSize;  // pages held as codes

  HeadState<G> st;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float x[4];
    load4_bf16(p.q + (row0 + g) * kHeadDim + 4 * lane, x);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      st.q[g][i] = x[i] * p.q_scale;
      st.acc[g][i] = 0.0f;
    }
    st.m[g] = -INFINITY;
    st.l[g] = 0.0f;
  }

  const int32_t* bt = p.block_tables + static_cast<int64_t>(b) * p.max_blocks_per_seq;
  const int j0 = t0 / kBlockSize;
  const int j1 = (t1 + kBlockSize - 1) / kBlockSize;  // pages [j0, j1)
  const int jq = min(j1, full);                        // quantised: [j0, jq)
  auto rec_of = [&](int j) {
    return p.cache + (static_cast<int64_t>(bt[j]) * p.num_kv_heads + kvh) * kRec;
  };
  if (j0 < jq) {
    PageRegs cur = load_page(rec_of(j0), lane);
    for (int j = j0; j < jq; ++j) {
      PageRegs nxt = cur;
      if (j + 1 < jq) nxt = load_page(rec_of(j + 1), lane);
      quantised_page<G>(st, cur, lane);
      cur = nxt;
    }
  }
  if (jq < j1)  // the partial page (j1 - 1 == full), rows [0, n - 16 full)
    tail_page<G>(st,
                 p.tail + (static_cast<int64_t>(b) * p.num_kv_heads + kvh) * 2 *
                              kBlockSize * kHeadDim,
                 n - full * kBlockSize, lane);

  if (nchunks == 1) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float inv = 1.0f / st.l[g];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        store_out(p.out, (row0 + g) * kHeadDim + 4 * lane + i, st.acc[g][i] * inv, p.out_f32);
    }
    return;
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int64_t ci = (row0 + g) * p.max_chunks + c;
    if (lane == 0) {
      p.ws_ml[2 * ci] = st.m[g];
      p.ws_ml[2 * ci + 1] = st.l[g];
    }
    reinterpret_cast<float4*>(p.ws_o + ci * kHeadDim)[lane] =
        make_float4(st.acc[g][0], st.acc[g][1], st.acc[g][2], st.acc[g][3]);
  }
  __threadfence();
  __syncwarp();
  uint32_t ticket = 0;
  if (lane == 0) ticket = atomicAdd(&p.ws_ctr[row0], 1u);
  ticket = __shfl_sync(kAll, ticket, 0);
  if (ticket != static_cast<uint32_t>(nchunks - 1)) return;
  __threadfence();
  merge_group_warp<G>(p.ws_ml, p.ws_o, row0, p.max_chunks, nchunks, p.out, p.out_f32);
}

bool aligned(const void* ptr, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0;
}

}  // namespace
}  // namespace kv8

using namespace kv8;

extern "C" {

int32_t kv8_kivi_append(const void* k_new, const void* v_new,
                        const int32_t* cu_new, const int32_t* context_lens,
                        const int32_t* block_tables, int32_t batch,
                        int32_t num_kv_heads, int32_t head_dim,
                        int32_t block_size, int32_t max_blocks_per_seq,
                        int64_t num_blocks, int32_t max_new_tokens,
                        uint8_t* kivi_cache, void* kivi_tail, void* stream) {
  if (batch < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_blocks_per_seq <= 0 || num_blocks <= 0 || max_new_tokens < 0)
    return KV8_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || block_size != kBlockSize) return KV8_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(batch) * num_kv_heads > INT32_MAX ||
      num_blocks > INT64_MAX / (static_cast<int64_t>(num_kv_heads) * kRec))
    return KV8_ERR_UNSUPPORTED;
  if (batch == 0 || max_new_tokens == 0) return KV8_OK;
  if (!k_new || !v_new || !cu_new || !context_lens || !block_tables ||
      !kivi_cache || !kivi_tail)
    return KV8_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(kivi_cache, 16) ||
      !aligned(kivi_tail, 16) || !aligned(cu_new, 4) || !aligned(context_lens, 4) ||
      !aligned(block_tables, 4))
    return KV8_ERR_INVALID_ARG;
  AppendArgs a;
  a.k_new = static_cast<const __nv_bfloat16*>(k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(v_new);
  a.cu_new = cu_new;
  a.context_lens = context_lens;
  a.block_tables = block_tables;
  a.cache = kivi_cache;
  a.tail = static_cast<__nv_bfloat16*>(kivi_tail);
  a.num_kv_heads = num_kv_heads;
  a.max_blocks_per_seq = max_blocks_per_seq;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // pages a sequence can complete: those holding one of its <= max_new_tokens
  // new positions, at most max_new_tokens / 16 + 1
  const int64_t pages = static_cast<int64_t>(max_new_tokens) / kBlockSize + 1;
  const int64_t gy = (pages + kWarps - 1) / kWarps;
  const dim3 grid(static_cast<unsigned>(static_cast<int64_t>(batch) * num_kv_heads),
                  static_cast<unsigned>(gy < 65535 ? gy : 65535));
  kivi_page_kernel<<<grid, kWarps * 32, 0, st>>>(a);
  kivi_tail_kernel<<<static_cast<unsigned>(static_cast<int64_t>(batch) * num_kv_heads),
                     32, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? KV8_OK : KV8_ERR_CUDA;
}

int32_t kv8_kivi_paged_decode_attention(
    const void* q, const uint8_t* kivi_cache, const void* kivi_tail,
    const int32_t* block_tables, const int32_t* context_lens, int32_t batch,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, float softmax_scale, int32_t chunk_tokens,
    void* workspace, size_t workspace_bytes, void* out, int32_t out_dtype,
    void* stream) {
  if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 ||
      max_context_len < 0 || chunk_tokens < 0)
    return KV8_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return KV8_ERR_INVALID_ARG;
  if (out_dtype != KV8_OUT_BF16 && out_dtype != KV8_OUT_F32) return KV8_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || block_size != kBlockSize) return KV8_ERR_UNSUPPORTED;
  const int group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return KV8_ERR_UNSUPPORTED;
  if (chunk_tokens % block_size != 0) return KV8_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_context_len) >
      static_cast<int64_t>(max_blocks_per_seq) * block_size)
    return KV8_ERR_INVALID_ARG;
  if (num_blocks > INT64_MAX / (static_cast<int64_t>(num_kv_heads) * kRec))
    return KV8_ERR_UNSUPPORTED;
  if (batch == 0) return KV8_OK;
  if (!q || !kivi_cache || !kivi_tail || !block_tables || !context_lens || !out)
    return KV8_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kivi_cache, 16) || !aligned(kivi_tail, 16) ||
      !aligned(out, 16) || !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return KV8_ERR_INVALID_ARG;

  KiviDecode p;
  if (chunk_tokens == 0 || max_context_len <= chunk_tokens) {
    // one chunk covers every context
    const int32_t c = (max_context_len + kBlockSize - 1) / kBlockSize * kBlockSize;
    p.chunk_tokens = c < kBlockSize ? kBlockSize : c;
    p.max_chunks = 1;
  } else {
    p.chunk_tokens = chunk_tokens;
    p.max_chunks = (max_context_len + chunk_tokens - 1) / chunk_tokens;
  }
  p.ws_ml = nullptr;
  p.ws_o = nullptr;
  p.ws_ctr = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p.max_chunks > 1) {
    const size_t ml = workspace_ml_bytes(batch, num_q_heads, p.max_chunks);
    const size_t ob = workspace_o_bytes(batch, num_q_heads, p.max_chunks);
    if (!workspace || workspace_bytes < workspace_total_bytes(batch, num_q_heads, p.max_chunks) ||
        !aligned(workspace, 16))
      return KV8_ERR_WORKSPACE;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    p.ws_ml = reinterpret_cast<float*>(base);
    p.ws_o = reinterpret_cast<float*>(base + ml);
    p.ws_ctr = reinterpret_cast<uint32_t*>(base + ml + ob);
    if (cudaMemsetAsync(p.ws_ctr, 0, workspace_ctr_bytes(batch, num_q_heads), st) !=
        cudaSuccess)
      return KV8_ERR_CUDA;
  }
  if (!(softmax_scale > 0.0f))
    softmax_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(head_dim)));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.cache = kivi_cache;
  p.tail = static_cast<const __nv_bfloat16*>(kivi_tail);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.out = out;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.out_f32 = out_dtype == KV8_OUT_F32 ? 1 : 0;
  p.q_scale = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634074);
  const int per_item = group < 4 ? group : 4;
  p.subs = group / per_item;
  p.items = static_cast<int64_t>(p.max_chunks) * batch * num_kv_heads * p.subs;
  const int64_t blocks = (p.items + kWarps - 1) / kWarps;
  if (blocks > INT32_MAX) return KV8_ERR_UNSUPPORTED;
  const unsigned grid = static_cast<unsigned>(blocks);
  switch (per_item) {
    case 1: kivi_decode_kernel<1><<<grid, kWarps * 32, 0, st>>>(p); break;
    case 2: kivi_decode_kernel<2><<<grid, kWarps * 32, 0, st>>>(p); break;
    default: kivi_decode_kernel<4><<<grid, kWarps * 32, 0, st>>>(p); break;
  }
  return cudaGetLastError() == cudaSuccess ? KV8_OK : KV8_ERR_CUDA;
}

}  // extern "C"
