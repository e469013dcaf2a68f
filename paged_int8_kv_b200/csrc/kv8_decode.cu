// kv8_decode.cu -- split-K paged INT8 decode attention and the split reduce.
//
// What is computed [KV Cache 优化全景解析——从基础原理到工程实践, §2.1 and
// §3.3; KV-Cache 全栈优化系统, 主要特性]: for one new query token per
// sequence, every query head h of KV group kvh = h / G attends over the
// sequence's cached tokens, each dequantised on the fly (k_hat = code * ks,
// v_hat = code * vs), out = softmax(q k_hat^T / sqrt(d)) v_hat, with fp32
// accumulation [大模型推理加速：KV Cache与vLLM技术解析, §4.1].
//
// Work decomposition (one CTA per (context chunk, KV head, sequence)):
//   * The chunk's 16-token pages are dealt round-robin to NW warps.  Each
//     warp owns SPW shared-memory slots and streams its own pages through
//     them: lane 0 resolves the page through the block table
//     [KV Cache 优化全景解析, §4.2] and issues two TMA tensor copies (the
//     2 KB K page and the 2 KB V page, 128-byte swizzled so that the
//     column reads below are bank-conflict free) plus two 64-byte bulk
//     copies (the K and V scales) that complete on the slot's mbarrier.
//     There is no producer warp and no cross-warp handshake on the ring:
//     the warp that consumes a slot refills it.
//   * All G query heads of the KV group are computed together, so each K/V
//     byte is read from HBM exactly once per step.
//   * Per page, a warp computes the G x 16 scores with codes converted to
//     fp32 in registers, folds the token's K scale into the score, keeps a
//     base-2 online softmax (running max m and sum l per head), folds the
//     token's V scale into the probability and accumulates o += p * vc.
//   * At the end of the chunk the NW warp states are merged through shared
//     memory.  A sequence that fits one chunk writes the normalised output;
//     otherwise (m, l, o) go to the workspace and kv8_split_reduce merges
//     the chunks with a log-sum-exp.
#include "kv8_common.cuh"
#include "kv8_internal.h"

namespace kv8 {

__device__ uint32_t g_device_status = 0;

namespace {

constexpr int kD = kHeadDim;
constexpr int kBS = kBlockSize;
constexpr uint32_t kFull = 0xffffffffu;
constexpr uint32_t kPageTx = 2 * kPageBytes + 2 * kBS * sizeof(float);

// --------------------------------------------------------------------------
// Shared-memory plan of a decode CTA (base aligned to 1024 bytes):
//   per warp w: SPW slots of [K page 2048 B | V page 2048 B]   (tiles)
//   per warp w: SPW slots of [ks 64 B | vs 64 B]              (scales)
//   per warp w: SPW mbarriers
// After its last page a warp reuses its own tiles as its merge record:
//   o[G][128] fp32, m[G], l[G].
// --------------------------------------------------------------------------
template <int NW, int SPW>
struct SmemPlan {
  static constexpr int kTileBytes = NW * SPW * 2 * kPageBytes;
  static constexpr int kScaleBytes = NW * SPW * 2 * kBS * 4;
  static constexpr int kBarBytes = NW * SPW * 8;
  static constexpr int kBytes = kTileBytes + kScaleBytes + kBarBytes + 1024;
};

// Transposed butterfly reduction of G per-lane partial sums over a group of
// LPT consecutive lanes.  On return every lane holds the full sum for head
// lane_head<G, LPT>(dg); lanes of the same head hold identical values.
template <int G, int LPT>
__device__ __forceinline__ float reduce_heads(float (&v)[G], int lane) {
  int count = G;
#pragma unroll
  for (int m = LPT / 2; m >= 1; m >>= 1) {
    if (count > 1) {
      const int half = count / 2;
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < G / 2; ++i) {
        if (i < half) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(kFull, send, m);
        }
      }
      count = half;
    } else {
      v[0] += __shfl_xor_sync(kFull, v[0], m);
    }
  }
  return v[0];
}

template <int G, int LPT>
__device__ __forceinline__ int lane_head(int dg) {
  return dg / (LPT / G);
}

__device__ __forceinline__ void store_out(void* out, int64_t idx, float v,
                                          int out_f32) {
  if (out_f32)
    static_cast<float*>(out)[idx] = v;
  else
    static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
}

// Hardware base-2 exponential (MUFU), relative error ~2^-22; -inf -> 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^e for e in [-126, 127], built from the exponent bits.
__device__ __forceinline__ float pow2i(int e) {
  return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

// For x > 0 normal: the e with x = f * 2^e, f in [0.5, 1); x <= 2^-126 -> -125.
__device__ __forceinline__ int exp_frexp(float x) {
  const int be = static_cast<int>((__float_as_uint(x) >> 23) & 0xFF);
  return be == 0 ? -125 : be - 126;
}

// Log-sum-exp merge of one query head's C chunk partials into its output
// row: chunk c holds m_c (base-2 max), l_c (sum of 2^(s - m_c)) and o_c[d]
// (sum of 2^(s - m_c) v_hat[d]);
//   M = max_c m_c,  L = sum_c l_c 2^(m_c - M),
//   out[d] = sum_c o_c[d] 2^(m_c - M) / L.
// Called by every thread of a CTA of NW warps (it synchronises the CTA);
// `red` is NW*128 + 2 floats of shared memory.  Warp 0 finds M and L; then
// warp w sums chunks w, w + NW, ... for 4 dims per lane with float4 loads,
// and warp 0 adds the NW partial sums.  The fused merge of a split decode
// and the standalone reduce kernel both use it with the same NW, so they
// produce identical results.
template <int NW>
__device__ __forceinline__ void merge_head(const float* ml, const float* o,
                                           int nchunks, void* out,
                                           int64_t out_row, int out_f32,
                                           float* red) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    float mx = -INFINITY;
    for (int c = lane; c < nchunks; c += 32) mx = fmaxf(mx, __ldcg(&ml[2 * c]));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1)
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
    float ls = 0.0f;
    for (int c = lane; c < nchunks; c += 32) {
      const float mc = __ldcg(&ml[2 * c]);
      ls += (mc == -INFINITY) ? 0.0f : __ldcg(&ml[2 * c + 1]) * ex2(mc - mx);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) ls += __shfl_xor_sync(kFull, ls, m);
    if (lane == 0) {
      red[NW * kD] = mx;
      red[NW * kD + 1] = ls;
    }
  }
  __syncthreads();
  const float M = red[NW * kD];
  const float L = red[NW * kD + 1];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int c = warp; c < nchunks; c += NW) {
    const float mc = __ldcg(&ml[2 * c]);
    const float w = (mc == -INFINITY) ? 0.0f : ex2(mc - M);
    const float4 v =
        __ldcg(reinterpret_cast<const float4*>(o + static_cast<int64_t>(c) * kD) + lane);
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  *reinterpret_cast<float4*>(&red[warp * kD + 4 * lane]) = acc;
  __syncthreads();
  if (warp == 0) {
    float4 sum = *reinterpret_cast<const float4*>(&red[4 * lane]);
#pragma unroll
    for (int w = 1; w < NW; ++w) {
      const float4 t = *reinterpret_cast<const float4*>(&red[w * kD + 4 * lane]);
      sum.x += t.x;
      sum.y += t.y;
      sum.z += t.z;
      sum.w += t.w;
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    const int64_t base = out_row * kD + 4 * lane;
    store_out(out, base + 0, sum.x * inv, out_f32);
    store_out(out, base + 1, sum.y * inv, out_f32);
    store_out(out, base + 2, sum.z * inv, out_f32);
    store_out(out, base + 3, sum.w * inv, out_f32);
  }
  __syncthreads();
}

// --------------------------------------------------------------------------
// Page math.  A policy object holds one warp's running state over the pages
// it is dealt in a chunk:
//   init(qg, q_scale, lane)   q of the G heads of the group (bf16 [G][128])
//   page(tk, tv, ks, vs, nv)  fold in one 16-token page; tokens >= nv are
//                             masked (their bytes may be stale or poison)
//   reset()                   contribute nothing (after a failed wait)
//   record(rec, lane)         write this warp's o[G][128] (relative to its
//                             running max m, base 2), m[G] and l[G]
// --------------------------------------------------------------------------

// CUDA-core form: codes become exact fp32 in registers, fp32 FMA.
//   G <= 4: a lane covers 16 dims of one token (8 lanes per token, 4 tokens
//           per pass, 4 passes per page);
//   G == 8: 8 dims (16 lanes per token, 2 tokens per pass, 8 passes).
template <int G>
struct SimtMath {
  static constexpr int DPL = (G <= 4) ? 16 : 8;  // dims per lane
  static constexpr int LPT = kD / DPL;           // lanes per token
  static constexpr int TPP = 32 / LPT;           // tokens per pass
  static constexpr int NPASS = kBS / TPP;        // passes per page
  static constexpr int HSTRIDE = LPT / G;        // lanes per head after reduce

  int lane, tg, dg, hh;
  float2 q2[G][DPL / 2];
  float2 o2[G][DPL / 2];
  float m_run, l_run;

  __device__ __forceinline__ void init(const __nv_bfloat16* qg, float q_scale,
                                       int lane_) {
    lane = lane_;
    tg = lane / LPT;
    dg = lane % LPT;
    hh = lane_head<G, LPT>(dg);
    const __nv_bfloat16* qd = qg + dg * DPL;
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int i = 0; i < DPL / 8; ++i) {
        const uint4 raw = reinterpret_cast<const uint4*>(qd + h * kD)[i];
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          q2[h][i * 4 + j] =
              make_float2(__uint_as_float(w[j] << 16) * q_scale,
                          __uint_as_float(w[j] & 0xFFFF0000u) * q_scale);
      }
    }
    reset();
  }

  __device__ __forceinline__ void reset() {
    m_run = -INFINITY;
    l_run = 0.0f;
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < DPL / 2; ++i) o2[h][i] = make_float2(0.f, 0.f);
  }

  __device__ __forceinline__ void load_codes(const uint8_t* tile, int t,
                                             float2 (&f)[DPL / 2]) const {
    // swizzled 16-byte chunk holding dims [dg*DPL, dg*DPL + DPL)
    const int chunk16 = (dg * DPL) / 16;
    const uint8_t* row =
        tile + t * 128 + ((chunk16 ^ (t & 7)) << 4) + ((dg * DPL) & 15);
    if constexpr (DPL == 16) {
      const uint4 w = *reinterpret_cast<const uint4*>(row);
      i8x4_to_f32(w.x, f[0], f[1]);
      i8x4_to_f32(w.y, f[2], f[3]);
      i8x4_to_f32(w.z, f[4], f[5]);
      i8x4_to_f32(w.w, f[6], f[7]);
    } else {
      const uint2 w = *reinterpret_cast<const uint2*>(row);
      i8x4_to_f32(w.x, f[0], f[1]);
      i8x4_to_f32(w.y, f[2], f[3]);
    }
  }

  __device__ __forceinline__ void page(const uint8_t* tk, const uint8_t* tv,
                                       const float* ks, const float* vs,
                                       int nv) {
    float sc[NPASS];
#pragma unroll
    for (int ps = 0; ps < NPASS; ++ps) {
      const int t = ps * TPP + tg;
      float2 kf[DPL / 2];
      load_codes(tk, t, kf);
      float acc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i) a = ffma2(q2[h][i], kf[i], a);
        acc[h] = a.x + a.y;
      }
      const float dot = reduce_heads<G, LPT>(acc, lane);
      sc[ps] = t < nv ? dot * ks[t] : -INFINITY;
    }
    float mx = sc[0];
#pragma unroll
    for (int ps = 1; ps < NPASS; ++ps) mx = fmaxf(mx, sc[ps]);
#pragma unroll
    for (int m = LPT; m < 32; m <<= 1)
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
    const float m_new = fmaxf(m_run, mx);
    const bool live = m_new != -INFINITY;
    const float alpha = live ? exp2f(m_run - m_new) : 1.0f;
    float pv[NPASS];
    float psum = 0.0f;
#pragma unroll
    for (int ps = 0; ps < NPASS; ++ps) {
      const int t = ps * TPP + tg;
      const float pr = live ? exp2f(sc[ps] - m_new) : 0.0f;
      psum += pr;
      pv[ps] = t < nv ? pr * vs[t] : 0.0f;
    }
    l_run = l_run * alpha + psum;
    m_run = m_new;
    if (__any_sync(kFull, alpha != 1.0f)) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float a = __shfl_sync(kFull, alpha, h * HSTRIDE);
        const float2 a2 = make_float2(a, a);
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i) o2[h][i] = fmul2(o2[h][i], a2);
      }
    }
#pragma unroll
    for (int ps = 0; ps < NPASS; ++ps) {
      const int t = ps * TPP + tg;
      float2 vf[DPL / 2];
      load_codes(tv, t, vf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float ph = __shfl_sync(kFull, pv[ps], tg * LPT + h * HSTRIDE);
        const float2 p2 = make_float2(ph, ph);
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i) o2[h][i] = ffma2(p2, vf[i], o2[h][i]);
      }
    }
  }

  __device__ __forceinline__ void record(float* rec) {
#pragma unroll
    for (int m = LPT; m < 32; m <<= 1) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i) {
          o2[h][i].x += __shfl_xor_sync(kFull, o2[h][i].x, m);
          o2[h][i].y += __shfl_xor_sync(kFull, o2[h][i].y, m);
        }
    }
    float l_lane = (dg % HSTRIDE == 0) ? l_run : 0.0f;
#pragma unroll
    for (int m = LPT; m < 32; m <<= 1)
      l_lane += __shfl_xor_sync(kFull, l_lane, m);
    if (tg == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i)
          *reinterpret_cast<float2*>(&rec[h * kD + dg * DPL + 2 * i]) = o2[h][i];
      if (dg % HSTRIDE == 0) {
        rec[G * kD + hh] = m_run;
        rec[G * kD + G + hh] = l_lane;
      }
    }
  }
};

// Tensor-core form (mma.sync m16n8k16, fp16 operands, fp32 accumulation).
// Per 16-token page a warp computes
//   S^T[16 x 8]   = K_code[16 x 128] . q'^T[128 x 8]    rows = the 16 tokens
//   O^T[128 x 8] += V_code^T[128 x 16] . P''^T[16 x 8]   cols = query heads
// i.e. 8 k-steps for the scores and 8 m-tiles x (hi, lo) for the output;
// columns >= G carry zero q and are never stored.  Thread (r = lane/4,
// c = lane%4) owns, in both products, heads 2c and 2c+1: it holds their
// scores for tokens r and 8+r, keeps their running max, and holds their
// O^T columns, so the softmax bookkeeping never leaves the thread except
// on a (rare) change of the reference max.  P'' moves from the S^T layout
// to the B-operand layout of the p.v mma with two 8x8 movmatrix transposes
// per fp16 half.
// Exactness of the operands:
//   * codes -> fp16 exactly: the byte c+128 is placed under the fp16
//     exponent of 1024, giving 1152 + c exactly, then 1152 is subtracted;
//   * q is scaled per head by a power of two so that max|q'| lies in
//     [2^14, 2^15) and converted to fp16 (exact for bf16 values down to
//     2^-17 of that max); the power of two goes into the score factor;
//   * P'' = 2^(s - m) * vs_t * 2^-E is split into fp16 hi + lo (about 22
//     significant bits); E, a per-warp power of two that only grows, keeps
//     P'' inside the fp16 range (the accumulators are rescaled exactly);
//   * m and E are moved lazily (see page()), so most pages skip the
//     rescale of the accumulators.
// Index maps (any bijection works as long as both operands agree):
//   q.k: k index -> dim 32c + 4s + {0,2 | 1,3} in k-step s, so a thread
//        reads 32 contiguous code bytes of each of its tokens r and 8+r;
//   p.v: row r / r+8 of m-tile 2w+j -> dim 16r + 4w + 2j + {0 | 1}, so a
//        thread reads one 16-byte chunk of each of tokens 2c, 2c+1, 8+2c,
//        9+2c.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0,
                                         uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 8x8 transpose of 16-bit elements held in the mma fragment layout.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ float2 unpack_h2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  return __half22float2(h);
}

constexpr uint32_t kBias1152 = 0x64806480u;  // fp16 (1152, 1152)

// Exact fp16 codes of one K word: even = (byte0, byte2), odd = (byte1, byte3).
__device__ __forceinline__ void k_word_to_h2(uint32_t w, uint32_t& even,
                                             uint32_t& odd) {
  even = hsub2_u32((w & 0x00FF00FFu) ^ 0x64806480u, kBias1152);
  odd = hsub2_u32(prmt(w, 0x64646464u, 0x4341u) ^ 0x00800080u, kBias1152);
}

// Exact fp16 pair (byte j of a, byte j of b) from an interleaved word
// x = (a.bj, b.bj, a.bj', b.bj') biased by 0x80 per byte; sel picks j/j'.
__device__ __forceinline__ uint32_t v_pair(uint32_t x, uint32_t sel) {
  return hsub2_u32(prmt(x, 0x64646464u, sel), kBias1152);
}

__device__ __forceinline__ uint32_t word_of(const uint4& a, int i) {
  return i == 0 ? a.x : i == 1 ? a.y : i == 2 ? a.z : a.w;
}

template <int G>
struct MmaMath {
  static constexpr float kSlack = 8.0f;  // log2 units
  static constexpr int kVSlack = 4;
  int lane, r, c;
  uint2 qk[8];      // B fragments of q'^T (head r): k-step s
  float qf0, qf1;   // score factors of heads 2c, 2c+1
  float ot[8][4];   // O^T fragments: heads 2c, 2c+1 at two dims per m-tile
  float m0, m1;     // reference max of heads 2c, 2c+1 (base 2)
  float l0, l1;     // this thread's partial sums of heads 2c, 2c+1
  int e_run;        // P'' carries 2^-e_run (warp-uniform)
  float vlim;       // 2^(e_run + kVSlack)
  float fs;         // 2^-e_run

  __device__ __forceinline__ void init(const __nv_bfloat16* qg, float q_scale,
                                       int lane_) {
    lane = lane_;
    r = lane >> 2;
    c = lane & 3;
    float qv[32];
    if (r < G) {
      const uint4* src = reinterpret_cast<const uint4*>(qg + r * kD + 32 * c);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 raw = src[i];
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          qv[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
          qv[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) qv[i] = 0.0f;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(qv[i]));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    // q' = q * 2^sh with max|q'| in [2^14, 2^15); applied as two exact
    // power-of-two factors so that each stays representable
    const int sh = amax > 0.0f ? 15 - exp_frexp(amax) : 0;
    const float f1 = pow2i(sh / 2), f2 = pow2i(sh - sh / 2);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      qk[s].x = pack_h2(qv[4 * s + 0] * f1 * f2, qv[4 * s + 2] * f1 * f2);
      qk[s].y = pack_h2(qv[4 * s + 1] * f1 * f2, qv[4 * s + 3] * f1 * f2);
    }
    const float qf = q_scale * pow2i(-(sh / 2)) * pow2i(-(sh - sh / 2));
    // this thread's score columns are heads 2c and 2c+1 (quads 2c, 2c+1)
    qf0 = __shfl_sync(kFull, qf, 8 * c);
    qf1 = __shfl_sync(kFull, qf, 8 * c + 4);
    reset();
  }

  __device__ __forceinline__ void reset() {
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.0f;
    e_run = -126;
    vlim = 0.0f;
    fs = 1.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) ot[i][j] = 0.0f;
  }

  __device__ __forceinline__ void page(const uint8_t* tk, const uint8_t* tv,
                                       const float* ks, const float* vs,
                                       int nv) {
    // ---- S^T = K q'^T: rows r (token r) and r+8 (token 8+r)
    const uint8_t* ra = tk + r * 128;
    const uint8_t* rb = tk + (8 + r) * 128;
    const int sw = r & 7;  // (8 + r) & 7 == r & 7
    const uint4 ka0 = *reinterpret_cast<const uint4*>(ra + (((2 * c) ^ sw) << 4));
    const uint4 ka1 = *reinterpret_cast<const uint4*>(ra + (((2 * c + 1) ^ sw) << 4));
    const uint4 kb0 = *reinterpret_cast<const uint4*>(rb + (((2 * c) ^ sw) << 4));
    const uint4 kb1 = *reinterpret_cast<const uint4*>(rb + (((2 * c + 1) ^ sw) << 4));
    float st[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      uint32_t ea, oa, eb, ob;
      k_word_to_h2(word_of(s < 4 ? ka0 : ka1, s & 3), ea, oa);
      k_word_to_h2(word_of(s < 4 ? kb0 : kb1, s & 3), eb, ob);
      mma16816(st, ea, eb, oa, ob, qk[s].x, qk[s].y);
    }
    // st: [0] token r head 2c, [1] token r head 2c+1,
    //     [2] token 8+r head 2c, [3] token 8+r head 2c+1
    const bool va = r < nv, vb = 8 + r < nv;
    const float ksa = ks[r], ksb = ks[8 + r];
    const float vsa = va ? vs[r] : 0.0f, vsb = vb ? vs[8 + r] : 0.0f;
    float sc[4];
    sc[0] = va ? st[0] * qf0 * ksa : -INFINITY;
    sc[1] = va ? st[1] * qf1 * ksa : -INFINITY;
    sc[2] = vb ? st[2] * qf0 * ksb : -INFINITY;
    sc[3] = vb ? st[3] * qf1 * ksb : -INFINITY;

    // Lazy rescaling: the reference maxima (per head) and the exponent
    // e_run (per warp) move only when a score exceeds its reference by
    // more than kSlack or a V scale exceeds 2^(e_run + kVSlack); otherwise
    // probabilities up to 2^kSlack are accumulated against the stale
    // reference, which keeps every P'' below 2^(kSlack + kVSlack).
    const float lm0 = fmaxf(sc[0], sc[2]);
    const float lm1 = fmaxf(sc[1], sc[3]);
    const float lv = fmaxf(vsa, vsb);
    const bool move = lm0 > m0 + kSlack || lm1 > m1 + kSlack || lv > vlim;
    if (__any_sync(kFull, move)) {
      float x0 = lm0, x1 = lm1, vx = lv;
#pragma unroll
      for (int m = 4; m < 32; m <<= 1) {
        x0 = fmaxf(x0, __shfl_xor_sync(kFull, x0, m));
        x1 = fmaxf(x1, __shfl_xor_sync(kFull, x1, m));
        vx = fmaxf(vx, __shfl_xor_sync(kFull, vx, m));
      }
      const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
      // every lane sees the same 16 tokens' scales: e_new is warp-uniform
      const int e_new = vx > vlim ? exp_frexp(vx) : e_run;
      const float ef = pow2i(max(e_run - e_new, -126));
      const float a0 = (n0 == m0) ? 1.0f : ex2(m0 - n0);
      const float a1 = (n1 == m1) ? 1.0f : ex2(m1 - n1);
      l0 *= a0;
      l1 *= a1;
      m0 = n0;
      m1 = n1;
      e_run = e_new;
      vlim = pow2i(min(e_new + kVSlack, 127));
      fs = pow2i(-e_new);
      const float b0 = a0 * ef, b1 = a1 * ef;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ot[i][0] *= b0;
        ot[i][1] *= b1;
        ot[i][2] *= b0;
        ot[i][3] *= b1;
      }
    }
    const float u0 = m0 == -INFINITY ? 0.0f : m0;
    const float u1 = m1 == -INFINITY ? 0.0f : m1;
    const float p0 = ex2(sc[0] - u0), p1 = ex2(sc[1] - u1);
    const float p2 = ex2(sc[2] - u0), p3 = ex2(sc[3] - u1);
    l0 += p0 + p2;
    l1 += p1 + p3;
    const float wa = vsa * fs, wb = vsb * fs;
    const float q0 = p0 * wa, q1 = p1 * wa, q2 = p2 * wb, q3 = p3 * wb;
    // fp16 hi/lo in the S^T layout (rows = tokens, cols = heads) ...
    const uint32_t ha = pack_h2(q0, q1), hb = pack_h2(q2, q3);
    const float2 fa = unpack_h2(ha), fb = unpack_h2(hb);
    const uint32_t la = pack_h2(q0 - fa.x, q1 - fa.y);
    const uint32_t lb = pack_h2(q2 - fb.x, q3 - fb.y);
    // ... transposed to B fragments of P''^T: head r, tokens {2c, 2c+1}
    // (tokens 0..7 matrix) and {8+2c, 9+2c} (tokens 8..15 matrix)
    const uint32_t h0 = movmatrix_t(ha), h2 = movmatrix_t(hb);
    const uint32_t g0 = movmatrix_t(la), g2 = movmatrix_t(lb);

    // ---- O^T += V^T P''^T: tokens 2c, 2c+1, 8+2c, 9+2c, 16-byte chunk r
    const int t0 = 2 * c, t2 = 8 + 2 * c;
    const int cr0 = (r ^ (2 * c)) << 4;      // tokens 2c and 8+2c
    const int cr1 = (r ^ (2 * c + 1)) << 4;  // tokens 2c+1 and 9+2c
    const uint4 vA = *reinterpret_cast<const uint4*>(tv + t0 * 128 + cr0);
    const uint4 vB = *reinterpret_cast<const uint4*>(tv + (t0 + 1) * 128 + cr1);
    const uint4 vC = *reinterpret_cast<const uint4*>(tv + t2 * 128 + cr0);
    const uint4 vD = *reinterpret_cast<const uint4*>(tv + (t2 + 1) * 128 + cr1);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t A = word_of(vA, w), B = word_of(vB, w);
      const uint32_t C = word_of(vC, w), D = word_of(vD, w);
      const uint32_t X = prmt(A, B, 0x5140u) ^ 0x80808080u;  // bytes 0,1
      const uint32_t Y = prmt(A, B, 0x7362u) ^ 0x80808080u;  // bytes 2,3
      const uint32_t Z = prmt(C, D, 0x5140u) ^ 0x80808080u;
      const uint32_t U = prmt(C, D, 0x7362u) ^ 0x80808080u;
      // m-tile 2w: rows r / r+8 = byte 0 / byte 1
      {
        const uint32_t a0 = v_pair(X, 0x4140u), a1 = v_pair(X, 0x4342u);
        const uint32_t a2 = v_pair(Z, 0x4140u), a3 = v_pair(Z, 0x4342u);
        mma16816(ot[2 * w], a0, a1, a2, a3, h0, h2);
        mma16816(ot[2 * w], a0, a1, a2, a3, g0, g2);
      }
      // m-tile 2w+1: rows r / r+8 = byte 2 / byte 3
      {
        const uint32_t a0 = v_pair(Y, 0x4140u), a1 = v_pair(Y, 0x4342u);
        const uint32_t a2 = v_pair(U, 0x4140u), a3 = v_pair(U, 0x4342u);
        mma16816(ot[2 * w + 1], a0, a1, a2, a3, h0, h2);
        mma16816(ot[2 * w + 1], a0, a1, a2, a3, g0, g2);
      }
    }
  }

  __device__ __forceinline__ void record(float* rec) {
    float s0 = l0, s1 = l1;
#pragma unroll
    for (int m = 4; m < 32; m <<= 1) {
      s0 += __shfl_xor_sync(kFull, s0, m);
      s1 += __shfl_xor_sync(kFull, s1, m);
    }
    const float f = pow2i(e_run);
    const int h0 = 2 * c, h1 = 2 * c + 1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int w = i >> 1, j = i & 1;
      const int dA = 16 * r + 4 * w + 2 * j;  // row r
      const int dB = dA + 1;                  // row r + 8
      if (h0 < G) {
        rec[h0 * kD + dA] = ot[i][0] * f;
        rec[h0 * kD + dB] = ot[i][2] * f;
      }
      if (h1 < G) {
        rec[h1 * kD + dA] = ot[i][1] * f;
        rec[h1 * kD + dB] = ot[i][3] * f;
      }
    }
    if (r == 0) {
      if (h0 < G) {
        rec[G * kD + h0] = m0;
        rec[G * kD + G + h0] = s0;
      }
      if (h1 < G) {
        rec[G * kD + h1] = m1;
        rec[G * kD + G + h1] = s1;
      }
    }
  }
};

// --------------------------------------------------------------------------
// The decode kernel: pipeline, merge and write; the page math is `Math`.
// --------------------------------------------------------------------------
template <int G, int NW, int SPW, class Math>
__global__ void __launch_bounds__(NW * 32)
decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv) {
  using Plan = SmemPlan<NW, SPW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int chunk = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int n = p.context_lens[b];
  const int tok0 = chunk * p.chunk_tokens;
  if (tok0 >= n && !(n == 0 && chunk == 0)) return;
  const int tok1 = min(n, tok0 + p.chunk_tokens);
  const int npages = (tok1 - tok0 + kBS - 1) / kBS;
  const int nchunks = (n + p.chunk_tokens - 1) / p.chunk_tokens;
  const int my_pages = warp < npages ? (npages - warp + NW - 1) / NW : 0;

  uint8_t* tiles = smem + warp * SPW * 2 * kPageBytes;
  float* scl = reinterpret_cast<float*>(smem + Plan::kTileBytes) +
               warp * SPW * 2 * kBS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Plan::kTileBytes +
                                               Plan::kScaleBytes) +
                   warp * SPW;

  if (lane == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
#pragma unroll
    for (int s = 0; s < SPW; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // ---- page issue: block-table entries are fetched 32 at a time
  const int32_t* bt = p.block_tables +
                      static_cast<int64_t>(b) * p.max_blocks_per_seq +
                      tok0 / kBS + warp;
  int bt_reg = 0;
  auto issue = [&](int k) {
    if ((k & 31) == 0) {
      const int kk = k + lane;
      bt_reg = kk < my_pages ? bt[kk * NW] : 0;
    }
    const int blk = __shfl_sync(kFull, bt_reg, k & 31);
    if (lane == 0) {
      const int s = k % SPW;
      const int page = blk * p.num_kv_heads + kvh;
      mbar_arrive_expect_tx(&bars[s], kPageTx);
      uint8_t* tk = tiles + s * 2 * kPageBytes;
      tma_load_3d(tk, &tmk, 0, 0, page, &bars[s]);
      tma_load_3d(tk + kPageBytes, &tmv, 0, 0, page, &bars[s]);
      float* sc = scl + s * 2 * kBS;
      bulk_g2s(sc, p.k_scales + static_cast<int64_t>(page) * kBS,
               kBS * sizeof(float), &bars[s]);
      bulk_g2s(sc + kBS, p.v_scales + static_cast<int64_t>(page) * kBS,
               kBS * sizeof(float), &bars[s]);
    }
  };
  const int pre = my_pages < SPW ? my_pages : SPW;
  for (int k = 0; k < pre; ++k) issue(k);

  Math math;
  math.init(p.q + (static_cast<int64_t>(b) * p.num_q_heads + kvh * G) * kD,
            p.q_scale, lane);

  bool ok = true;
  int k = 0;
  for (; k < my_pages; ++k) {
    const int s = k % SPW;
    if (!mbar_wait(&bars[s], (k / SPW) & 1, &g_device_status)) {
      ok = false;
      break;
    }
    const uint8_t* tk = tiles + s * 2 * kPageBytes;
    const float* ks = scl + s * 2 * kBS;
    const int tbase = tok0 + (warp + k * NW) * kBS;
    math.page(tk, tk + kPageBytes, ks, ks + kBS, min(kBS, tok1 - tbase));
    __syncwarp();
    if (k + SPW < my_pages) issue(k + SPW);
  }
  if (!ok) {
    // A copy never landed: drain what is still in flight (bounded), then
    // contribute nothing to the merge.  The sticky status word reports it.
    for (int kk = k + 1; kk < my_pages && kk < k + SPW; ++kk)
      mbar_wait(&bars[kk % SPW], (kk / SPW) & 1, &g_device_status);
    math.reset();
  }

  // ---- warp record in this warp's own (now idle) tiles, then merge
  __syncwarp();
  math.record(reinterpret_cast<float*>(tiles));
  __syncthreads();

  const bool single = nchunks <= 1;
  for (int idx = threadIdx.x; idx < G * kD; idx += NW * 32) {
    const int h = idx / kD;
    const int d = idx % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* rw = reinterpret_cast<const float*>(smem + w * SPW * 2 * kPageBytes);
      M = fmaxf(M, rw[G * kD + h]);
    }
    float L = 0.0f, O = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* rw = reinterpret_cast<const float*>(smem + w * SPW * 2 * kPageBytes);
      const float mw = rw[G * kD + h];
      const float e = (mw == -INFINITY) ? 0.0f : ex2(mw - M);
      L += rw[G * kD + G + h] * e;
      O += rw[h * kD + d] * e;
    }
    const int hq = kvh * G + h;
    if (single) {
      const int64_t oi = (static_cast<int64_t>(b) * p.num_q_heads + hq) * kD + d;
      store_out(p.out, oi, L > 0.0f ? O / L : 0.0f, p.out_f32);
    } else {
      const int64_t ci =
          (static_cast<int64_t>(b) * p.num_q_heads + hq) * p.max_chunks + chunk;
      p.ws_o[ci * kD + d] = O;
      if (d == 0) {
        p.ws_ml[2 * ci] = M;
        p.ws_ml[2 * ci + 1] = L;
      }
    }
  }
  if (single) return;

  // ---- split: the last CTA of this (sequence, KV group) to finish merges
  // every chunk's partial (threadfence-then-ticket; no CTA ever waits).
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int ticket = atomicAdd(
        &p.ws_ctr[static_cast<int64_t>(b) * p.num_q_heads + kvh * G], 1u);
    s_last = ticket == static_cast<unsigned int>(nchunks - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  float* red = reinterpret_cast<float*>(smem);  // records no longer needed
  for (int h = 0; h < G; ++h) {
    const int64_t bh = static_cast<int64_t>(b) * p.num_q_heads + kvh * G + h;
    merge_head<NW>(p.ws_ml + bh * p.max_chunks * 2,
                   p.ws_o + bh * p.max_chunks * kD, nchunks, p.out, bh,
                   p.out_f32, red);
  }
}

// --------------------------------------------------------------------------
// Standalone split reduce: one CTA of kReduceNW warps per (b, hq), the same
// merge routine (and warp count) as the fused merge of the decode kernel.
// --------------------------------------------------------------------------
constexpr int kReduceNW = 4;

__global__ void __launch_bounds__(kReduceNW * 32)
split_reduce_kernel(const float* __restrict__ ws_ml,
                    const float* __restrict__ ws_o,
                    const int32_t* __restrict__ context_lens, int32_t num_q_heads,
                    int32_t chunk_tokens, int32_t max_chunks, void* out,
                    int32_t out_f32) {
  __shared__ __align__(16) float red[kReduceNW * kD + 2];
  const int bh = blockIdx.x;
  const int b = bh / num_q_heads;
  const int n = context_lens[b];
  const int nchunks = (n + chunk_tokens - 1) / chunk_tokens;
  if (nchunks <= 1) return;
  merge_head<kReduceNW>(ws_ml + static_cast<int64_t>(bh) * max_chunks * 2,
                        ws_o + static_cast<int64_t>(bh) * max_chunks * kD,
                        nchunks, out, bh, out_f32, red);
}

template <int G, int NW, int SPW, class Math>
int launch_decode_kernel(const DecodeParams& p, const CUtensorMap& tmk,
                         const CUtensorMap& tmv, cudaStream_t stream) {
  auto kern = decode_kernel<G, NW, SPW, Math>;
  constexpr int smem = SmemPlan<NW, SPW>::kBytes;
  static bool attr_done = false;  // per instantiation; benign race
  if (!attr_done) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return -1;
    attr_done = true;
  }
  dim3 grid(p.max_chunks, p.num_kv_heads, p.batch);
  kern<<<grid, NW * 32, smem, stream>>>(p, tmk, tmv);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int G>
int launch_group(const DecodeParams& p, const CUtensorMap& tmk,
                 const CUtensorMap& tmv, int32_t variant, cudaStream_t stream) {
  // CTA shape from a sweep on B200 over (warps, slots per warp) in
  // {1,2,4,8} x {2,3,4,6,8} on the four multi-sequence workloads: 4 warps
  // with 2 slots each (8 pages, 33 KB in flight per CTA; 4 CTAs per SM) was
  // fastest for the tensor-core form on all of them.
  if (variant == 1)
    return launch_decode_kernel<G, 4, 4, SimtMath<G>>(p, tmk, tmv, stream);
  static_assert(kReduceNW == 4, "fused and standalone merges must match");
  return launch_decode_kernel<G, 4, 2, MmaMath<G>>(p, tmk, tmv, stream);
}

}  // namespace

int read_device_status(uint32_t* value, int clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(value, g_device_status, sizeof(uint32_t)) !=
      cudaSuccess)
    return -1;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(uint32_t)) !=
        cudaSuccess)
      return -1;
  }
  return 0;
}

size_t workspace_ml_bytes(int32_t batch, int32_t num_q_heads,
                          int32_t max_chunks) {
  const size_t ml = static_cast<size_t>(batch) * num_q_heads * max_chunks * 2 *
                    sizeof(float);
  return (ml + 255) & ~size_t(255);
}

size_t workspace_o_bytes(int32_t batch, int32_t num_q_heads,
                         int32_t max_chunks) {
  return static_cast<size_t>(batch) * num_q_heads * max_chunks * kD *
         sizeof(float);
}

size_t workspace_ctr_bytes(int32_t batch, int32_t num_q_heads) {
  return static_cast<size_t>(batch) * num_q_heads * sizeof(uint32_t);
}

size_t workspace_total_bytes(int32_t batch, int32_t num_q_heads,
                             int32_t max_chunks) {
  return workspace_ml_bytes(batch, num_q_heads, max_chunks) +
         workspace_o_bytes(batch, num_q_heads, max_chunks) +
         workspace_ctr_bytes(batch, num_q_heads);
}

int launch_decode(const DecodeParams& p, const CUtensorMap& tmk,
                  const CUtensorMap& tmv, int32_t variant,
                  cudaStream_t stream) {
  const int g = p.num_q_heads / p.num_kv_heads;
  switch (g) {
    case 1: return launch_group<1>(p, tmk, tmv, variant, stream);
    case 2: return launch_group<2>(p, tmk, tmv, variant, stream);
    case 4: return launch_group<4>(p, tmk, tmv, variant, stream);
    case 8: return launch_group<8>(p, tmk, tmv, variant, stream);
    default: return -2;
  }
}

int launch_split_reduce(const float* ws_ml, const float* ws_o,
                        const int32_t* context_lens, int32_t batch,
                        int32_t num_q_heads, int32_t chunk_tokens,
                        int32_t max_chunks, void* out, int32_t out_f32,
                        cudaStream_t stream) {
  const int64_t nbh = static_cast<int64_t>(batch) * num_q_heads;
  if (nbh == 0) return 0;
  split_reduce_kernel<<<static_cast<unsigned>(nbh), kReduceNW * 32, 0, stream>>>(
      ws_ml, ws_o, context_lens, num_q_heads, chunk_tokens, max_chunks, out,
      out_f32);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace kv8
