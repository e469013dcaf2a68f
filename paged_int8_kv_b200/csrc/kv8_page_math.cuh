// kv8_page_math.cuh -- the per-page math of the warp-level decode forms,
// shared by the decode kernel and the shared-prefix kernel: each form is a
// policy object holding one warp's running attention state (online softmax
// and output accumulators for the G query heads of one KV group) over the
// 16-token pages it is dealt.
#pragma once

#include "../../include/kv8.h"
#include "kv8_common.cuh"
#include "kv8_internal.h"
#include "kv8_merge.cuh"

namespace kv8 {
namespace {

constexpr int kD = kHeadDim;
constexpr int kBS = kBlockSize;
constexpr uint32_t kFull = 0xffffffffu;

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

// Where a warp's finished chunk goes: the normalised output row (a context
// that fits one chunk) or the chunk's partial (m, l, o) in the workspace.
struct ChunkSink {
  void* out;
  float* ws_o;
  float* ws_ml;
  int64_t row0;  // b * H_q + first query head of the KV group
  int64_t ci0;   // partial index of the first head: row0 * max_chunks + chunk
  int max_chunks;
  bool single;
  int out_f32;

  __device__ __forceinline__ void put_o(int h, int d, float o, float l) const {
    if (single)
      store_out(out, (row0 + h) * kD + d, l > 0.0f ? o / l : 0.0f, out_f32);
    else
      ws_o[(ci0 + static_cast<int64_t>(h) * max_chunks) * kD + d] = o;
  }
  __device__ __forceinline__ void put_ml(int h, float m, float l) const {
    if (!single) {
      const int64_t ci = ci0 + static_cast<int64_t>(h) * max_chunks;
      ws_ml[2 * ci] = m;
      ws_ml[2 * ci + 1] = l;
    }
  }
};

// --------------------------------------------------------------------------
// Page math.  A policy object holds one warp's running state over the pages
// it is dealt in a chunk:
//   init(qg, q_scale, lane)   q of the G heads of the group (bf16 [G][128])
//   page(tk, tv, ks, vs, nv)  fold in one 16-token page; tokens >= nv are
//                             masked (their bytes may be stale or poison)
//   reset()                   contribute nothing (after a failed wait)
//   finish(sink)              hand this warp's o[G][128] (relative to its
//                             running max m, base 2), m[G] and l[G] to sink
// --------------------------------------------------------------------------

// CUDA-core form: codes become exact fp32 in registers, fp32 FMA.
//   G <= 4: a lane covers 16 dims of one token (8 lanes per token, 4 tokens
//           per pass, 4 passes per page);
//   G == 8: 8 dims (16 lanes per token, 2 tokens per pass, 8 passes).
template <int G>
struct SimtMath {
  static constexpr int kWarpsPerSM = 0;  // no register cap
  static constexpr int kScratchBytes = 0;
  static constexpr int kTmemCols = 0;
  static constexpr int kCodeBytes = 2048;  // one page of K (or V) codes
  static constexpr bool kSharedAddr = false;
  static constexpr int DPL = (G <= 4) ? 16 : 8;  // dims per lane
  static constexpr int LPT = kD / DPL;           // lanes per token
  static constexpr int TPP = 32 / LPT;           // tokens per pass
  static constexpr int NPASS = kBS / TPP;        // passes per page
  static constexpr int HSTRIDE = LPT / G;        // lanes per head after reduce

  int lane, tg, dg, hh;
  float2 q2[G][DPL / 2];

  __device__ __forceinline__ void attach(uint8_t*) {}
  __device__ __forceinline__ void attach_tmem(uint32_t) {}
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

  template <bool Full>
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

  __device__ __forceinline__ void finish(const ChunkSink& sk) {
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
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float lh = __shfl_sync(kFull, l_lane, h * HSTRIDE);
      if (tg == 0) {
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i) {
          sk.put_o(h, dg * DPL + 2 * i, o2[h][i].x, lh);
          sk.put_o(h, dg * DPL + 2 * i + 1, o2[h][i].y, lh);
        }
      }
    }
    if (tg == 0 && dg % HSTRIDE == 0) sk.put_ml(hh, m_run, l_lane);
  }
};

// Tensor-core form.  Per 16-token page a warp computes
//   S[16 x 16]    = Qd[16 x 128] . K_code^T[128 x 16]   (int8 mma, exact)
//   O^T[128 x 8] += V_code^T[128 x 16] . P''^T[16 x 8]   (fp16 mma, fp32 acc)
// * q.k: the rows of Qd are (query head, digit plane): q of head h is
//   rounded to Q = rint(q * 2^sh) with max|Q| in [2^29, 2^30) and written
//   as four balanced int8 digits Q = 2^24 d3 + 2^16 d2 + 2^8 d1 + d0; m-tile
//   0 holds (d3 | d2) and m-tile 1 (d1 | d0) of heads 0..7 in rows r / r+8.
//   The K codes enter as the B operand exactly as loaded (a thread's two
//   32-bit words of a token are one B fragment), the int32 products are
//   exact, and S = 2^-sh (2^16 (2^8 C3 + C2) + (2^8 C1 + C0)).  The only
//   approximation is the rounding of q to 30 bits of its head's max.
//   2 m-tiles x 2 n-tiles (tokens 0..7, 8..15) x 4 k-steps = 16 mma.
// * Thread (r = lane/4, c = lane%4) then holds head r's scores for tokens
//   2c, 2c+1, 8+2c, 9+2c: exactly its B fragment of P''^T for the p.v mma,
//   so the probabilities never move between lanes.
// * p.v: V codes -> fp16 exactly (the byte c+128 under the fp16 exponent of
//   1024 gives 1152 + c; 1152 is subtracted); P'' = 2^(s - m) vs_t 2^-E is
//   split into fp16 hi + lo (about 22 bits); 8 m-tiles x (hi, lo) = 16 mma.
//   The O^T columns are heads 2c, 2c+1.
// * Softmax: base 2, one running max and sum per head (quad r), moved
//   lazily: only when a score exceeds the reference by more than kSlack or
//   a V scale exceeds 2^(E + kVSlack) are the references moved and the
//   accumulators rescaled (exactly, by powers of two and one exp2).
// Index maps (any bijection works as long as both operands agree):
//   q.k: k index 4c+j / 16+4c+j -> dim 32c + 8s + j / 32c + 8s + 4 + j in
//        k-step s, so a thread reads 32 contiguous code bytes of each of its
//        tokens r and 8+r;
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

// Integer mma: D[16x8] (s32) += A[16x32] (s8, row) . B[32x8] (s8, col).
__device__ __forceinline__ void mma16832_s8(int (&d)[4], uint32_t a0,
                                            uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0,
                                            uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
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

// SharedV: p.v reads a fp16 copy of the V page from shared memory (pv_f16)
// instead of converting the int8 page (pv_codes); only the output dims map
// differs.
template <int G, bool SharedV = false>
struct MmaMath {
  static constexpr int kWarpsPerSM = 12;  // cap registers at 168 per thread
  static constexpr int kScratchBytes = 0;
  static constexpr int kTmemCols = 0;
  static constexpr int kCodeBytes = 2048;  // one page of K (or V) codes
  static constexpr bool kSharedAddr = false;
  static constexpr float kSlack = 8.0f;   // log2 units
  static constexpr int kVSlack = 4;
  int lane, r, c;
  uint4 qa[2][4];   // A fragments of Qd (head r): m-tile t, k-step s
  float qf;         // score factor of head r: 2^-sh * softmax_scale * log2(e)
  float ot[8][4];   // O^T fragments: heads 2c, 2c+1 at two dims per m-tile
  float m_run;      // reference max of head r (base 2)
  float l_run;      // this thread's partial sum of head r
  int e_run;        // P'' carries 2^-e_run (warp-uniform)
  float vlim;       // 2^(e_run + kVSlack)
  float fs;         // 2^-e_run

  __device__ __forceinline__ void attach(uint8_t*) {}
  __device__ __forceinline__ void attach_tmem(uint32_t) {}

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
    // max|q| * 2^sh in [2^29, 2^30), applied as two exact powers of two
    const int sh = amax > 0.0f ? 30 - exp_frexp(amax) : 0;
    const float f1 = pow2i(sh / 2), f2 = pow2i(sh - sh / 2);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t w0 = 0, w1 = 0, w2 = 0, w3 = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int Q = __float2int_rn(qv[8 * s + 4 * half + j] * f1 * f2);
          const int d0 = static_cast<int>(static_cast<int8_t>(Q & 0xFF));
          const int q1 = (Q - d0) >> 8;
          const int d1 = static_cast<int>(static_cast<int8_t>(q1 & 0xFF));
          const int q2 = (q1 - d1) >> 8;
          const int d2 = static_cast<int>(static_cast<int8_t>(q2 & 0xFF));
          const int d3 = (q2 - d2) >> 8;
          w0 |= (static_cast<uint32_t>(d0) & 0xFFu) << (8 * j);
          w1 |= (static_cast<uint32_t>(d1) & 0xFFu) << (8 * j);
          w2 |= (static_cast<uint32_t>(d2) & 0xFFu) << (8 * j);
          w3 |= (static_cast<uint32_t>(d3) & 0xFFu) << (8 * j);
        }
        // k = 4c..4c+3 (word 2s: a0/a1), k = 16+4c.. (word 2s+1: a2/a3)
        if (half == 0) {
          qa[0][s].x = w3; qa[0][s].y = w2;
          qa[1][s].x = w1; qa[1][s].y = w0;
        } else {
          qa[0][s].z = w3; qa[0][s].w = w2;
          qa[1][s].z = w1; qa[1][s].w = w0;
        }
      }
    }
    qf = q_scale * pow2i(-(sh / 2)) * pow2i(-(sh - sh / 2));
    reset();
  }

  __device__ __forceinline__ void reset() {
    m_run = -INFINITY;
    l_run = 0.0f;
    e_run = -126;
    vlim = 0.0f;
    fs = 1.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) ot[i][j] = 0.0f;
  }

  // q.k and the online softmax of one page; returns this thread's B
  // fragments of P''^T (hi: h0, h2; lo: g0, g2) for the p.v products
  template <bool Full>
  __device__ __forceinline__ void qk_softmax(const uint8_t* tk, const float* ks,
                                             const float* vs, int nv,
                                             uint32_t& h0, uint32_t& h2,
                                             uint32_t& g0, uint32_t& g2) {
    // ---- S = Qd K^T: n-tile 0 = tokens 0..7 (this thread feeds token r),
    //                  n-tile 1 = tokens 8..15 (token 8 + r)
    const uint8_t* ra = tk + r * 128;
    const uint8_t* rb = tk + (8 + r) * 128;
    const int sw = r & 7;  // (8 + r) & 7 == r & 7
    const uint4 ka0 = *reinterpret_cast<const uint4*>(ra + (((2 * c) ^ sw) << 4));
    const uint4 ka1 = *reinterpret_cast<const uint4*>(ra + (((2 * c + 1) ^ sw) << 4));
    const uint4 kb0 = *reinterpret_cast<const uint4*>(rb + (((2 * c) ^ sw) << 4));
    const uint4 kb1 = *reinterpret_cast<const uint4*>(rb + (((2 * c + 1) ^ sw) << 4));
    int acc[2][2][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[t][j][e] = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint4& ka = s < 2 ? ka0 : ka1;
      const uint4& kb = s < 2 ? kb0 : kb1;
      const uint32_t a0 = (s & 1) ? ka.z : ka.x, a1 = (s & 1) ? ka.w : ka.y;
      const uint32_t b0 = (s & 1) ? kb.z : kb.x, b1 = (s & 1) ? kb.w : kb.y;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        mma16832_s8(acc[t][0], qa[t][s].x, qa[t][s].y, qa[t][s].z, qa[t][s].w, a0, a1);
        mma16832_s8(acc[t][1], qa[t][s].x, qa[t][s].y, qa[t][s].z, qa[t][s].w, b0, b1);
      }
    }
    // head r, tokens 2c, 2c+1 (n-tile 0) and 8+2c, 9+2c (n-tile 1)
    float st[4];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int hi = acc[0][j][e] * 256 + acc[0][j][2 + e];  // d3, d2
        const int lo = acc[1][j][e] * 256 + acc[1][j][2 + e];  // d1, d0
        st[2 * j + e] = __int2float_rn(hi) * 65536.0f + __int2float_rn(lo);
      }
    const int t0 = 2 * c, t2 = 8 + 2 * c;
    const float2 ksa = *reinterpret_cast<const float2*>(ks + t0);
    const float2 ksb = *reinterpret_cast<const float2*>(ks + t2);
    const float2 vsa = *reinterpret_cast<const float2*>(vs + t0);
    const float2 vsb = *reinterpret_cast<const float2*>(vs + t2);
    const bool v0 = t0 < nv, v1 = t0 + 1 < nv, v2 = t2 < nv, v3 = t2 + 1 < nv;
    float sc[4];
    sc[0] = v0 ? st[0] * qf * ksa.x : -INFINITY;
    sc[1] = v1 ? st[1] * qf * ksa.y : -INFINITY;
    sc[2] = v2 ? st[2] * qf * ksb.x : -INFINITY;
    sc[3] = v3 ? st[3] * qf * ksb.y : -INFINITY;
    float vsv[4];
    vsv[0] = v0 ? vsa.x : 0.0f;
    vsv[1] = v1 ? vsa.y : 0.0f;
    vsv[2] = v2 ? vsb.x : 0.0f;
    vsv[3] = v3 ? vsb.y : 0.0f;

    const float lm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    const float lv = fmaxf(fmaxf(vsv[0], vsv[1]), fmaxf(vsv[2], vsv[3]));
    if (__any_sync(kFull, lm > m_run + kSlack || lv > vlim)) {
      float x = fmaxf(lm, __shfl_xor_sync(kFull, lm, 1));
      x = fmaxf(x, __shfl_xor_sync(kFull, x, 2));
      float vx = fmaxf(lv, __shfl_xor_sync(kFull, lv, 1));
      vx = fmaxf(vx, __shfl_xor_sync(kFull, vx, 2));
      const float n = fmaxf(m_run, x);
      // every quad sees all 16 tokens' scales: e_new is warp-uniform
      const int e_new = vx > vlim ? exp_frexp(vx) : e_run;
      const float a = (n == m_run) ? 1.0f : ex2(m_run - n);
      const float a_o = a * pow2i(max(e_run - e_new, -126));
      l_run *= a;
      m_run = n;
      e_run = e_new;
      vlim = pow2i(min(e_new + kVSlack, 127));
      fs = pow2i(-e_new);
      const float ae = __shfl_sync(kFull, a_o, 8 * c);      // head 2c
      const float ao = __shfl_sync(kFull, a_o, 8 * c + 4);  // head 2c+1
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ot[i][0] *= ae;
        ot[i][1] *= ao;
        ot[i][2] *= ae;
        ot[i][3] *= ao;
      }
    }
    const float mu = m_run == -INFINITY ? 0.0f : m_run;
    float pr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pr[i] = ex2(sc[i] - mu);
    l_run += (pr[0] + pr[1]) + (pr[2] + pr[3]);
    float pp[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pp[i] = pr[i] * (vsv[i] * fs);
    // B fragments of P''^T (head r): tokens {2c, 2c+1} and {8+2c, 9+2c}
    h0 = pack_h2(pp[0], pp[1]);
    h2 = pack_h2(pp[2], pp[3]);
    const float2 f0 = unpack_h2(h0);
    const float2 f2 = unpack_h2(h2);
    g0 = pack_h2(pp[0] - f0.x, pp[1] - f0.y);
    g2 = pack_h2(pp[2] - f2.x, pp[3] - f2.y);
  }

  // O^T += V^T P''^T from the int8 V page as TMA staged it: tokens 2c, 2c+1,
  // 8+2c, 9+2c, 16-byte chunk r, converted exactly to fp16 in registers
  __device__ __forceinline__ void pv_codes(const uint8_t* tv, uint32_t h0,
                                           uint32_t h2, uint32_t g0,
                                           uint32_t g2) {
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
      {  // m-tile 2w: rows r / r+8 = byte 0 / byte 1
        const uint32_t a0 = v_pair(X, 0x4140u), a1 = v_pair(X, 0x4342u);
        const uint32_t a2 = v_pair(Z, 0x4140u), a3 = v_pair(Z, 0x4342u);
        mma16816(ot[2 * w], a0, a1, a2, a3, h0, h2);
        mma16816(ot[2 * w], a0, a1, a2, a3, g0, g2);
      }
      {  // m-tile 2w+1: rows r / r+8 = byte 2 / byte 3
        const uint32_t a0 = v_pair(Y, 0x4140u), a1 = v_pair(Y, 0x4342u);
        const uint32_t a2 = v_pair(U, 0x4140u), a3 = v_pair(U, 0x4342u);
        mma16816(ot[2 * w + 1], a0, a1, a2, a3, h0, h2);
        mma16816(ot[2 * w + 1], a0, a1, a2, a3, g0, g2);
      }
    }
  }

  // O^T += V^T P''^T from a page already converted to fp16 in shared memory
  // (vh: [16 tokens][128 dims] fp16, 16-byte chunk j of token t stored at
  // chunk j ^ (t & 7)): m-tile i = dims 16i..16i+15, its A fragment one
  // transposing ldmatrix of four 8x8 tiles (tokens 0-7 / 8-15 x dims
  // 16i..+7 / 16i+8..+15)
  __device__ __forceinline__ void pv_f16(uint32_t vh, uint32_t h0, uint32_t h2,
                                         uint32_t g0, uint32_t g2) {
    const int q = lane >> 3, t = ((q >> 1) << 3) + (lane & 7);
    const uint32_t row = vh + t * 256;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int chunk = 2 * i + (q & 1);
      uint32_t a0, a1, a2, a3;
      asm volatile(
          "ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
          : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
          : "r"(row + ((chunk ^ (t & 7)) << 4))
          : "memory");
      mma16816(ot[i], a0, a1, a2, a3, h0, h2);
      mma16816(ot[i], a0, a1, a2, a3, g0, g2);
    }
  }

  template <bool Full>
  __device__ __forceinline__ void page(const uint8_t* tk, const uint8_t* tv,
                                       const float* ks, const float* vs,
                                       int nv) {
    uint32_t h0, h2, g0, g2;
    qk_softmax<Full>(tk, ks, vs, nv, h0, h2, g0, g2);
    pv_codes(tv, h0, h2, g0, g2);
  }

  __device__ __forceinline__ void finish(const ChunkSink& sk) {
    float l = l_run;
    l += __shfl_xor_sync(kFull, l, 1);
    l += __shfl_xor_sync(kFull, l, 2);
    // this thread's O^T columns are heads 2c (quad 2c) and 2c+1 (quad 2c+1)
    const float s0 = __shfl_sync(kFull, l, 8 * c);
    const float s1 = __shfl_sync(kFull, l, 8 * c + 4);
    const float m0 = __shfl_sync(kFull, m_run, 8 * c);
    const float m1 = __shfl_sync(kFull, m_run, 8 * c + 4);
    const float f = pow2i(e_run);
    const int h0 = 2 * c, h1 = 2 * c + 1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int w = i >> 1, j = i & 1;
      // pv_codes: rows r / r+8 of m-tile 2w+j are dims 16r+4w+2j+{0|1};
      // pv_f16: rows r / r+8 of m-tile i are dims 16i+r / 16i+r+8
      const int dA = SharedV ? 16 * i + r : 16 * r + 4 * w + 2 * j;  // row r
      const int dB = SharedV ? dA + 8 : dA + 1;                    // row r + 8
      if (h0 < G) {
        sk.put_o(h0, dA, ot[i][0] * f, s0);
        sk.put_o(h0, dB, ot[i][2] * f, s0);
      }
      if (h1 < G) {
        sk.put_o(h1, dA, ot[i][1] * f, s1);
        sk.put_o(h1, dB, ot[i][3] * f, s1);
      }
    }
    if (r == 0) {
      if (h0 < G) sk.put_ml(h0, m0, s0);
      if (h1 < G) sk.put_ml(h1, m1, s1);
    }
  }
};

// 32 consecutive 32-bit columns of this thread's tensor-memory lane (the
// warp's lane quarter), loaded / stored and waited for.
__device__ __forceinline__ void tm_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,"
      "%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,"
      "%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
        "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]),
        "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tm_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,"
      "%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,"
      "%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]),
      "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]),
      "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]), "f"(v[17]),
      "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]),
      "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]),
      "f"(v[30]), "f"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// s8 x u8 integer mma: D[16x8] (s32) += A[16x16] (s8, row) . B[16x8] (u8, col).
__device__ __forceinline__ void mma16816_s8u8(int (&d)[4], uint32_t a0,
                                              uint32_t a1, uint32_t b0) {
  asm("mma.sync.aligned.m16n8k16.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, "
      "{%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// Two 16 x 16 byte matrices from shared memory, each transposed into the A
// fragment of an m16n8k16 int8 mma: lanes 0..15 address the 16 source rows
// (16 bytes each) of matrix 0, lanes 16..31 those of matrix 1; thread
// (g = lane / 4, t = lane % 4) receives source rows 4t..4t+3 of column g
// (r0: matrix 0, r2: matrix 1) and of column g + 8 (r1, r3).
__device__ __forceinline__ void ldsm_x2_trans_b8(uint32_t addr, uint32_t& r0,
                                                 uint32_t& r1, uint32_t& r2,
                                                 uint32_t& r3) {
  asm volatile(
      "ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0, %1, %2, %3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr)
      : "memory");
}

// 16-byte shared-memory loads by 32-bit shared address (ordered like every
// other volatile access: never hoisted above the wait for the page).
__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Integer tensor-core form for groups of G <= 4 query heads: both products
// on int8 mma, no code is converted on the CUDA cores.
//   S[16 rows x 16 tok] = Qd[16 x 128] . K_code^T        (m16n8k32 s8, exact)
//   O^T[128 x 16 col]  += V_code^T[128 x 16 tok] . Pd^T   (m16n8k16 s8.u8)
// * Token <-> lane map: thread (r = lane/4, c = lane%4) ends up with the
//   scores of tokens 4c..4c+3; q.k n-tile j column n is token
//   4(n/2) + 2j + (n%2), and the p.v k index is the token itself.  Under the
//   TMA's 128-byte swizzle every shared-memory read below is then
//   bank-conflict free.
// * q.k rows: thread row r holds head hr = (r % 4) % G; its rows r and r+8
//   carry two of the four balanced int8 digit planes of q (Q = rint(q 2^sh),
//   max|Q| in [2^29, 2^30), Q = sum_p 2^(8p) d_p): planes 3 and 1 for r < 4,
//   2 and 0 for r >= 4.  Lanes L and L^16 hold the same head and add their
//   two partial scores, so both end with the full score; 8 mma per page.
//   The digits are the bytes of Q + 0x80808080, each minus 128: the unique
//   balanced base-256 representation.
// * p.v: P'' = 2^(s - m) vs 2^-e (lazy references as in MmaMath) is rounded
//   to the integer P = rint(P'' 2^kF) < 2^31, whose four bytes are exact
//   unsigned digit planes.  Column n of p.v n-tile t is (head hr(n), plane
//   2t + n/4); the V codes enter as the A operand straight from shared
//   memory through a transposing ldmatrix.  16 mma per page into int32
//   accumulators (|acc| < 127 * 255 * tokens: no overflow below 66K tokens
//   between drains).
// * The int32 accumulators are drained (converted, weighted 2^(8p - kF),
//   and added to fp32 partials kept in this warp's shared-memory scratch)
//   when the references move and at the end of an item.  The two lanes
//   c and c^2 hold complementary planes of the same outputs and are summed
//   at the end.
// InTmem: the drained fp32 partials live in 32 tensor-memory columns of the
// warp's lane quarter instead of 4 KB of the warp's shared memory (which is
// then free for page slots).
template <int G, bool InTmem = false>
struct I8Math {
  static_assert(G == 1 || G == 2 || G == 4, "groups of 1, 2 or 4 heads");
  static constexpr int kWarpsPerSM = 12;  // cap registers at 168 per thread
  static constexpr int kScratchBytes = InTmem ? 0 : 32 * 32 * 4;  // fp32 [32][lane]
  static constexpr int kTmemCols = InTmem ? 32 : 0;
  static constexpr int kCodeBytes = 2048;  // one page of K (or V) codes
  static constexpr float kSlack = 6.0f;   // log2 units
  static constexpr int kVSlack = 2;
  static constexpr int kF = 23;  // P'' < 2^(kSlack + kVSlack): P < 2^31
  // lowest V-scale exponent tracked, so that 2^(kF - e) stays a normal
  // float; V scales below 2^kMinE keep fewer bits of P (they are zero in
  // any practical cache)
  static constexpr int kMinE = kF - 127;
  int lane, r, c, up;
  uint32_t qa[4][4];  // A fragments of Qd per k-step: rows r / r+8, k halves
  float qf;           // score factor of head hr: 2^-sh * softmax_scale * log2(e)
  int acc[8][2][4];   // p.v int32 accumulators: m-tile, n-tile, fragment
  float* of;          // this warp's drained fp32 partials, [32][lane]
  uint32_t otm;       // ... or their tensor-memory address (InTmem)
  float m_run, l_run;
  int e_run;
  float vlim;         // 2^(e_run + kVSlack)
  float fsF;          // 2^(kF - e_run)
  uint32_t psel;      // prmt selector of this thread's two P planes
  bool started;       // the accumulators or the partials hold something
  bool of_live;       // the partials hold something

  __device__ __forceinline__ void attach(uint8_t* scratch) {
    of = reinterpret_cast<float*>(scratch);
  }
  __device__ __forceinline__ void attach_tmem(uint32_t taddr) { otm = taddr; }

  __device__ __forceinline__ void init(const __nv_bfloat16* qg, float q_scale,
                                       int lane_) {
    lane = lane_;
    r = lane >> 2;
    c = lane & 3;
    up = r >> 2;
    const int h = (r & 3) % G;
    float qv[32];
    const uint4* src = reinterpret_cast<const uint4*>(qg + h * kD + 32 * c);
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
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(qv[i]));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    const int sh = amax > 0.0f ? 30 - exp_frexp(amax) : 0;
    const float f1 = pow2i(sh / 2), f2 = pow2i(sh - sh / 2);
    // bytes (planes) this thread row keeps: rows r -> pa, rows r+8 -> pb
    const uint32_t pa = up ? 2u : 3u, pb = up ? 0u : 1u;
    const uint32_t sel = pa | ((4u + pa) << 4) | (pb << 8) | ((4u + pb) << 12);
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // dims 32c + 4i .. 32c + 4i + 3
      uint32_t u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        u[j] = static_cast<uint32_t>(__float2int_rn(qv[4 * i + j] * f1 * f2)) +
               0x80808080u;
      const uint32_t x = prmt(u[0], u[1], sel);
      const uint32_t y = prmt(u[2], u[3], sel);
      const uint32_t wa = prmt(x, y, 0x5410u) ^ 0x80808080u;
      const uint32_t wb = prmt(x, y, 0x7632u) ^ 0x80808080u;
      // k-step s = i / 2 covers dims 32c + 8s .. + 7: a0/a1 the first four
      // (rows r / r+8), a2/a3 the next four
      if (i & 1) {
        qa[i >> 1][2] = wa;
        qa[i >> 1][3] = wb;
      } else {
        qa[i >> 1][0] = wa;
        qa[i >> 1][1] = wb;
      }
    }
    qf = q_scale * pow2i(-(sh / 2)) * pow2i(-(sh - sh / 2));
    psel = static_cast<uint32_t>(up) | ((4u + up) << 4) | ((2u + up) << 8) |
           ((6u + up) << 12);
    reset();
  }

  __device__ __forceinline__ void zero_acc() {
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[m][t][e] = 0;
  }

  __device__ __forceinline__ void reset() {
    m_run = -INFINITY;
    l_run = 0.0f;
    e_run = kMinE;
    vlim = 0.0f;
    fsF = pow2i(kF - kMinE);
    started = false;
    of_live = false;
    zero_acc();
  }

  // partials += planes of the accumulators (weighted), then *= scale of the
  // output column's head (aA: column 2c, aB: column 2c+1); accumulators := 0
  __device__ __forceinline__ void drain(float aA, float aB) {
    const float w0 = pow2i(8 * (c >> 1) - kF);
    const float w1 = pow2i(16 + 8 * (c >> 1) - kF);
    if constexpr (InTmem) {
      float o[32];
      if (of_live) {
        tm_ld32(otm, o);
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = 0.0f;
      }
#pragma unroll
      for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int k = m * 4 + e;
          const float v = __int2float_rn(acc[m][0][e]) * w0 +
                           __int2float_rn(acc[m][1][e]) * w1;
          o[k] = (o[k] + v) * ((e & 1) ? aB : aA);
        }
      tm_st32(otm, o);
    } else {
#pragma unroll
      for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int k = m * 4 + e;
          const float v = __int2float_rn(acc[m][0][e]) * w0 +
                           __int2float_rn(acc[m][1][e]) * w1;
          const float old = of_live ? of[k * 32 + lane] : 0.0f;
          of[k * 32 + lane] = (old + v) * ((e & 1) ? aB : aA);
        }
    }
    of_live = true;
    zero_acc();
  }

  static constexpr bool kSharedAddr = true;

  template <bool Full>
  __device__ __forceinline__ void page(const uint8_t* tk, const uint8_t* tv,
                                       const float* ks, const float* vs,
                                       int nv) {
    page_s<Full>(smem_u32(tk), smem_u32(tv), smem_u32(ks), smem_u32(vs), nv);
  }

  // page() on 32-bit shared addresses (tk, tv: the K and V pages; ks, vs:
  // their 16 scales)
  template <bool Full>
  __device__ __forceinline__ void page_s(uint32_t tk, uint32_t tv, uint32_t ks,
                                         uint32_t vs, int nv) {
    // ---- S = Qd K^T.  n-tile j, column n = r: token 4(r/2) + 2j + r%2
    const uint32_t ta = 4 * (r >> 1) + (r & 1), tb = ta + 2;
    const uint32_t ra = tk + ta * 128, rb = tk + tb * 128;
    const uint32_t sw = ta & 7, swb = tb & 7, c2 = 2 * c;
    const uint4 ka0 = lds_u4(ra + ((c2 ^ sw) << 4));
    const uint4 ka1 = lds_u4(ra + (((c2 + 1) ^ sw) << 4));
    const uint4 kb0 = lds_u4(rb + ((c2 ^ swb) << 4));
    const uint4 kb1 = lds_u4(rb + (((c2 + 1) ^ swb) << 4));
    int sacc[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[j][e] = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint4& ka = s < 2 ? ka0 : ka1;
      const uint4& kb = s < 2 ? kb0 : kb1;
      mma16832_s8(sacc[0], qa[s][0], qa[s][1], qa[s][2], qa[s][3],
                  (s & 1) ? ka.z : ka.x, (s & 1) ? ka.w : ka.y);
      mma16832_s8(sacc[1], qa[s][0], qa[s][1], qa[s][2], qa[s][3],
                  (s & 1) ? kb.z : kb.x, (s & 1) ? kb.w : kb.y);
    }
    // rows r / r+8 hold planes (3, 1) for up == 0 and (2, 0) for up == 1
    const float wa = up ? 65536.0f : 16777216.0f;
    const float wb = up ? 1.0f : 256.0f;
    float st[4];  // tokens 4c + i, i = 2j + e
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float part = __fmaf_rn(__int2float_rn(sacc[j][e]), wa,
                                     __int2float_rn(sacc[j][2 + e]) * wb);
        st[2 * j + e] = part + __shfl_xor_sync(kFull, part, 16);
      }
    const float4 ks4 = lds_f4(ks + 16 * c);
    const float4 vs4 = lds_f4(vs + 16 * c);
    const float ksv[4] = {ks4.x, ks4.y, ks4.z, ks4.w};
    const float vsr[4] = {vs4.x, vs4.y, vs4.z, vs4.w};
    float sc[4], vsv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (Full) {
        sc[i] = st[i] * qf * ksv[i];
        vsv[i] = vsr[i];
      } else {
        const bool ok = 4 * c + i < nv;
        sc[i] = ok ? st[i] * qf * ksv[i] : -INFINITY;
        vsv[i] = ok ? vsr[i] : 0.0f;
      }
    }
    const float lm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    const float lv = fmaxf(fmaxf(vsv[0], vsv[1]), fmaxf(vsv[2], vsv[3]));
    if (__any_sync(kFull, lm > m_run + kSlack || lv > vlim)) {
      float x = fmaxf(lm, __shfl_xor_sync(kFull, lm, 1));
      x = fmaxf(x, __shfl_xor_sync(kFull, x, 2));
      float vx = fmaxf(lv, __shfl_xor_sync(kFull, lv, 1));
      vx = fmaxf(vx, __shfl_xor_sync(kFull, vx, 2));
      const float n = fmaxf(m_run, x);
      // every quad sees all 16 tokens' scales: e_new is warp-uniform
      const int e_new = vx > vlim ? max(exp_frexp(vx), kMinE) : e_run;
      const float a = (n == m_run) ? 1.0f : ex2(m_run - n);
      const float a_o = a * pow2i(max(e_run - e_new, -126));
      if (started) {
        const int hA = ((2 * c) & 3) % G, hB = ((2 * c + 1) & 3) % G;
        const float aA = __shfl_sync(kFull, a_o, 4 * hA);
        const float aB = __shfl_sync(kFull, a_o, 4 * hB);
        drain(aA, aB);
      }
      l_run *= a;
      m_run = n;
      e_run = e_new;
      vlim = pow2i(min(e_new + kVSlack, 127));
      fsF = pow2i(kF - e_new);
    }
    const float mu = m_run == -INFINITY ? 0.0f : m_run;
    float pr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pr[i] = ex2(sc[i] - mu);
    l_run += (pr[0] + pr[1]) + (pr[2] + pr[3]);
    uint32_t pi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pi[i] = __float2uint_rn(pr[i] * (vsv[i] * fsF));
    // B fragments: bytes = tokens 4c..4c+3, planes up (n-tile 0), 2+up (1)
    const uint32_t x = prmt(pi[0], pi[1], psel);
    const uint32_t y = prmt(pi[2], pi[3], psel);
    const uint32_t b0 = prmt(x, y, 0x5410u);
    const uint32_t b1 = prmt(x, y, 0x7632u);

    // ---- O^T += V^T Pd^T: ldmatrix rows = tokens 0..15 (lanes 0..15 and
    //      16..31 address the same tokens in m-tiles 2w and 2w+1)
    const uint32_t vbase = tv + (lane & 15) * 128;
    const int vsw = lane & 7, vmt = lane >> 4;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t a0, a1, a2, a3;
      ldsm_x2_trans_b8(vbase + (((2 * w + vmt) ^ vsw) << 4), a0, a1, a2, a3);
      mma16816_s8u8(acc[2 * w][0], a0, a1, b0);
      mma16816_s8u8(acc[2 * w][1], a0, a1, b1);
      mma16816_s8u8(acc[2 * w + 1][0], a2, a3, b0);
      mma16816_s8u8(acc[2 * w + 1][1], a2, a3, b1);
    }
    started = true;
  }

  __device__ __forceinline__ void finish(const ChunkSink& sk) {
    if (started) drain(1.0f, 1.0f);
    float l = l_run;
    l += __shfl_xor_sync(kFull, l, 1);
    l += __shfl_xor_sync(kFull, l, 2);
    const int nA = 2 * c, nB = 2 * c + 1;  // output columns of this thread
    const int hA = (nA & 3) % G, hB = (nB & 3) % G;
    const float sA = __shfl_sync(kFull, l, 4 * hA);
    const float sB = __shfl_sync(kFull, l, 4 * hB);
    const float mA = __shfl_sync(kFull, m_run, 4 * hA);
    const float mB = __shfl_sync(kFull, m_run, 4 * hB);
    const float f = pow2i(e_run);
    const bool wA = c < 2 && nA < G, wB = c < 2 && nB < G;
    float o[32];
    if constexpr (InTmem) {
      if (of_live) {
        tm_ld32(otm, o);
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = 0.0f;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) o[k] = of_live ? of[k * 32 + lane] : 0.0f;
    }
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = m * 4 + e;
        float v = o[k];
        v += __shfl_xor_sync(kFull, v, 2);  // the complementary planes
        const int d = 16 * m + r + ((e & 2) ? 8 : 0);
        if (e & 1) {
          if (wB) sk.put_o(nB, d, v * f, sB);
        } else {
          if (wA) sk.put_o(nA, d, v * f, sA);
        }
      }
    if (r == 0) {
      if (wA) sk.put_ml(nA, mA, sA);
      if (wB) sk.put_ml(nB, mB, sB);
    }
  }
};

// s8 x u8 integer mma, K = 32: D[16x8] (s32) += A[16x32] (s8) . B[32x8] (u8).
__device__ __forceinline__ void mma16832_s8u8(int (&d)[4], uint32_t a0,
                                              uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// u8 x u8 integer mma, K = 16: D[16x8] (s32) += A[16x16] (u8) . B[16x8] (u8).
__device__ __forceinline__ void mma16816_u8u8(int (&d)[4], uint32_t a0,
                                              uint32_t a1, uint32_t b0) {
  asm("mma.sync.aligned.m16n8k16.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, "
      "{%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// The INT4 form (groups of G <= 4 heads) over the INT4 cache: K and V codes
// are excess-8 nibbles u = c + 8, two per byte (dims 2i / 2i+1 in the low /
// high nibble of byte i); a page is 16 tokens x 64 bytes, staged by TMA as
// 8 rows of 128 bytes (tokens 2R and 2R+1 in row R) with the 128-byte
// swizzle.  The arithmetic is I8Math's, with the nibbles fed to the tensor
// cores as unsigned bytes and the bias removed exactly in integers:
// * q.k: sum_j d_j u_j = sum_j d_j c_j + 8 sum_j d_j, so every plane's
//   accumulator starts at -8 sum_j d_j (the plane's digit sum over the 128
//   dims).  A thread's 16 bytes of a token (dims 32c..32c+31) unpack into
//   even-dim words (mask) and odd-dim words (shift + mask); k-step s pairs
//   the even and odd words of dims 32c + 8s .. + 7, and q's digit planes
//   are laid out the same way.
// * p.v: one transposing ldmatrix of the packed V page gives, per 16-byte
//   column chunk q (dims 32q..32q+31), the even-dim m-tile (low nibbles)
//   and the odd-dim m-tile (high nibbles); sum_t P_t u_t - 8 sum_t P_t is
//   taken per digit plane, the planes' digit sums tracked with dp4a and
//   subtracted (times 8) from the int32 accumulators when they are drained.
template <int G>
struct I4Math {
  static_assert(G == 1 || G == 2 || G == 4, "groups of 1, 2 or 4 heads");
  static constexpr int kWarpsPerSM = 12;
  static constexpr int kScratchBytes = 0;
  static constexpr int kTmemCols = 32;
  static constexpr int kCodeBytes = 1024;  // one page of K (or V) nibbles
  static constexpr float kSlack = 6.0f;
  static constexpr int kVSlack = 2;
  static constexpr int kF = 23;
  static constexpr int kMinE = kF - 127;
  int lane, r, c, up;
  uint32_t qa[4][4];
  int dsa, dsb;       // digit sums of planes (rows r, r+8) over the head's dims
  float qf;
  int acc[8][2][4];
  int psum[2];        // this thread's P digit sums (n-tiles 0, 1) since the last drain
  uint32_t otm;
  float m_run, l_run;
  int e_run;
  float vlim, fsF;
  uint32_t psel;
  bool started, of_live;

  __device__ __forceinline__ void attach(uint8_t*) {}
  __device__ __forceinline__ void attach_tmem(uint32_t taddr) { otm = taddr; }

  __device__ __forceinline__ void init(const __nv_bfloat16* qg, float q_scale,
                                       int lane_) {
    lane = lane_;
    r = lane >> 2;
    c = lane & 3;
    up = r >> 2;
    const int h = (r & 3) % G;
    float qv[32];
    const uint4* src = reinterpret_cast<const uint4*>(qg + h * kD + 32 * c);
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
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(qv[i]));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    const int sh = amax > 0.0f ? 30 - exp_frexp(amax) : 0;
    const float f1 = pow2i(sh / 2), f2 = pow2i(sh - sh / 2);
    const uint32_t pa = up ? 2u : 3u, pb = up ? 0u : 1u;
    const uint32_t sel = pa | ((4u + pa) << 4) | (pb << 8) | ((4u + pb) << 12);
    int sa = 0, sb = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // k-step s = i / 2; i even: dims 32c + 8s + {0,2,4,6}, odd: + {1,3,5,7}
      const int s = i >> 1, odd = i & 1;
      uint32_t u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        u[j] = static_cast<uint32_t>(
                   __float2int_rn(qv[8 * s + 2 * j + odd] * f1 * f2)) +
               0x80808080u;
      const uint32_t x = prmt(u[0], u[1], sel);
      const uint32_t y = prmt(u[2], u[3], sel);
      const uint32_t wa = prmt(x, y, 0x5410u) ^ 0x80808080u;
      const uint32_t wb = prmt(x, y, 0x7632u) ^ 0x80808080u;
      sa = __dp4a(static_cast<int>(wa), 0x01010101, sa);
      sb = __dp4a(static_cast<int>(wb), 0x01010101, sb);
      if (odd) {
        qa[s][2] = wa;
        qa[s][3] = wb;
      } else {
        qa[s][0] = wa;
        qa[s][1] = wb;
      }
    }
    sa += __shfl_xor_sync(kFull, sa, 1);
    sa += __shfl_xor_sync(kFull, sa, 2);
    sb += __shfl_xor_sync(kFull, sb, 1);
    sb += __shfl_xor_sync(kFull, sb, 2);
    dsa = sa;
    dsb = sb;
    qf = q_scale * pow2i(-(sh / 2)) * pow2i(-(sh - sh / 2));
    psel = static_cast<uint32_t>(up) | ((4u + up) << 4) | ((2u + up) << 8) |
           ((6u + up) << 12);
    reset();
  }

  __device__ __forceinline__ void zero_acc() {
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[m][t][e] = 0;
    psum[0] = psum[1] = 0;
  }

  __device__ __forceinline__ void reset() {
    m_run = -INFINITY;
    l_run = 0.0f;
    e_run = kMinE;
    vlim = 0.0f;
    fsF = pow2i(kF - kMinE);
    started = false;
    of_live = false;
    zero_acc();
  }

  // remove the V bias (8 x the column's digit sum) from the accumulators
  __device__ __forceinline__ void unbias() {
    int s0 = psum[0], s1 = psum[1];
    s0 += __shfl_xor_sync(kFull, s0, 1);
    s0 += __shfl_xor_sync(kFull, s0, 2);
    s1 += __shfl_xor_sync(kFull, s1, 1);
    s1 += __shfl_xor_sync(kFull, s1, 2);
    // column n of n-tile t is thread row n's plane: columns 2c, 2c+1 here
    const int a0 = __shfl_sync(kFull, s0, 4 * (2 * c)), a1 = __shfl_sync(kFull, s0, 4 * (2 * c + 1));
    const int b0 = __shfl_sync(kFull, s1, 4 * (2 * c)), b1 = __shfl_sync(kFull, s1, 4 * (2 * c + 1));
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[m][0][e] -= 8 * ((e & 1) ? a1 : a0);
        acc[m][1][e] -= 8 * ((e & 1) ? b1 : b0);
      }
  }

  __device__ __forceinline__ void drain(float aA, float aB) {
    unbias();
    const float w0 = pow2i(8 * (c >> 1) - kF);
    const float w1 = pow2i(16 + 8 * (c >> 1) - kF);
    float o[32];
    if (of_live) {
      tm_ld32(otm, o);
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) o[k] = 0.0f;
    }
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = m * 4 + e;
        const float v = __int2float_rn(acc[m][0][e]) * w0 +
                         __int2float_rn(acc[m][1][e]) * w1;
        o[k] = (o[k] + v) * ((e & 1) ? aB : aA);
      }
    tm_st32(otm, o);
    of_live = true;
    zero_acc();
  }

  static constexpr bool kSharedAddr = true;

  template <bool Full>
  __device__ __forceinline__ void page(const uint8_t* tk, const uint8_t* tv,
                                       const float* ks, const float* vs,
                                       int nv) {
    page_s<Full>(smem_u32(tk), smem_u32(tv), smem_u32(ks), smem_u32(vs), nv);
  }

  // page() on 32-bit shared addresses (tk, tv: the K and V pages; ks, vs:
  // their 16 scales)
  template <bool Full>
  __device__ __forceinline__ void page_s(uint32_t tk, uint32_t tv, uint32_t ks,
                                         uint32_t vs, int nv) {
    // ---- S = Qd K^T: n-tile j, column n = r: token 4(r/2) + 2j + r%2;
    //      this thread's 16 bytes of a token t: row t/2, chunk 4(t%2) + c
    const uint32_t ta = 4 * (r >> 1) + (r & 1), tb = ta + 2;
    const uint4 pka =
        lds_u4(tk + (ta >> 1) * 128 + (((4 * (ta & 1) + c) ^ ((ta >> 1) & 7)) << 4));
    const uint4 pkb =
        lds_u4(tk + (tb >> 1) * 128 + (((4 * (tb & 1) + c) ^ ((tb >> 1) & 7)) << 4));
    int sacc[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      sacc[j][0] = sacc[j][1] = -8 * dsa;
      sacc[j][2] = sacc[j][3] = -8 * dsb;
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint32_t wa = word_of(pka, s), wb = word_of(pkb, s);
      mma16832_s8u8(sacc[0], qa[s][0], qa[s][1], qa[s][2], qa[s][3],
                    wa & 0x0F0F0F0Fu, (wa >> 4) & 0x0F0F0F0Fu);
      mma16832_s8u8(sacc[1], qa[s][0], qa[s][1], qa[s][2], qa[s][3],
                    wb & 0x0F0F0F0Fu, (wb >> 4) & 0x0F0F0F0Fu);
    }
    const float wa = up ? 65536.0f : 16777216.0f;
    const float wb = up ? 1.0f : 256.0f;
    float st[4];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float part = __fmaf_rn(__int2float_rn(sacc[j][e]), wa,
                                     __int2float_rn(sacc[j][2 + e]) * wb);
        st[2 * j + e] = part + __shfl_xor_sync(kFull, part, 16);
      }
    const float4 ks4 = lds_f4(ks + 16 * c);
    const float4 vs4 = lds_f4(vs + 16 * c);
    const float ksv[4] = {ks4.x, ks4.y, ks4.z, ks4.w};
    const float vsr[4] = {vs4.x, vs4.y, vs4.z, vs4.w};
    float sc[4], vsv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (Full) {
        sc[i] = st[i] * qf * ksv[i];
        vsv[i] = vsr[i];
      } else {
        const bool ok = 4 * c + i < nv;
        sc[i] = ok ? st[i] * qf * ksv[i] : -INFINITY;
        vsv[i] = ok ? vsr[i] : 0.0f;
      }
    }
    const float lm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    const float lv = fmaxf(fmaxf(vsv[0], vsv[1]), fmaxf(vsv[2], vsv[3]));
    if (__any_sync(kFull, lm > m_run + kSlack || lv > vlim)) {
      float x = fmaxf(lm, __shfl_xor_sync(kFull, lm, 1));
      x = fmaxf(x, __shfl_xor_sync(kFull, x, 2));
      float vx = fmaxf(lv, __shfl_xor_sync(kFull, lv, 1));
      vx = fmaxf(vx, __shfl_xor_sync(kFull, vx, 2));
      const float n = fmaxf(m_run, x);
      const int e_new = vx > vlim ? max(exp_frexp(vx), kMinE) : e_run;
      const float a = (n == m_run) ? 1.0f : ex2(m_run - n);
      const float a_o = a * pow2i(max(e_run - e_new, -126));
      if (started) {
        const int hA = ((2 * c) & 3) % G, hB = ((2 * c + 1) & 3) % G;
        const float aA = __shfl_sync(kFull, a_o, 4 * hA);
        const float aB = __shfl_sync(kFull, a_o, 4 * hB);
        drain(aA, aB);
      }
      l_run *= a;
      m_run = n;
      e_run = e_new;
      vlim = pow2i(min(e_new + kVSlack, 127));
      fsF = pow2i(kF - e_new);
    }
    const float mu = m_run == -INFINITY ? 0.0f : m_run;
    float pr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pr[i] = ex2(sc[i] - mu);
    l_run += (pr[0] + pr[1]) + (pr[2] + pr[3]);
    uint32_t pi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pi[i] = __float2uint_rn(pr[i] * (vsv[i] * fsF));
    const uint32_t x = prmt(pi[0], pi[1], psel);
    const uint32_t y = prmt(pi[2], pi[3], psel);
    const uint32_t b0 = prmt(x, y, 0x5410u);
    const uint32_t b1 = prmt(x, y, 0x7632u);
    psum[0] = static_cast<int>(__dp4a(b0, 0x01010101u, static_cast<unsigned>(psum[0])));
    psum[1] = static_cast<int>(__dp4a(b1, 0x01010101u, static_cast<unsigned>(psum[1])));

    // ---- O^T += V^T Pd^T: ldmatrix rows = tokens 0..15; lanes 0..15 take
    //      column chunk 2w, lanes 16..31 chunk 2w+1 (dims 32q..32q+31)
    const int vt = lane & 15, vq = lane >> 4;
    const uint32_t vrow = tv + (vt >> 1) * 128;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int q = 2 * w + vq;
      uint32_t r0, r1, r2, r3;
      ldsm_x2_trans_b8(vrow + (((4 * (vt & 1) + q) ^ ((vt >> 1) & 7)) << 4), r0, r1, r2, r3);
      // chunk 2w: m-tiles 4w (even dims) and 4w+1 (odd); chunk 2w+1: 4w+2, 4w+3
      const uint32_t e0 = r0 & 0x0F0F0F0Fu, e1 = r1 & 0x0F0F0F0Fu;
      const uint32_t o0 = (r0 >> 4) & 0x0F0F0F0Fu, o1 = (r1 >> 4) & 0x0F0F0F0Fu;
      const uint32_t e2 = r2 & 0x0F0F0F0Fu, e3 = r3 & 0x0F0F0F0Fu;
      const uint32_t o2 = (r2 >> 4) & 0x0F0F0F0Fu, o3 = (r3 >> 4) & 0x0F0F0F0Fu;
      mma16816_u8u8(acc[4 * w][0], e0, e1, b0);
      mma16816_u8u8(acc[4 * w][1], e0, e1, b1);
      mma16816_u8u8(acc[4 * w + 1][0], o0, o1, b0);
      mma16816_u8u8(acc[4 * w + 1][1], o0, o1, b1);
      mma16816_u8u8(acc[4 * w + 2][0], e2, e3, b0);
      mma16816_u8u8(acc[4 * w + 2][1], e2, e3, b1);
      mma16816_u8u8(acc[4 * w + 3][0], o2, o3, b0);
      mma16816_u8u8(acc[4 * w + 3][1], o2, o3, b1);
    }
    started = true;
  }

  __device__ __forceinline__ void finish(const ChunkSink& sk) {
    if (started) drain(1.0f, 1.0f);
    float l = l_run;
    l += __shfl_xor_sync(kFull, l, 1);
    l += __shfl_xor_sync(kFull, l, 2);
    const int nA = 2 * c, nB = 2 * c + 1;
    const int hA = (nA & 3) % G, hB = (nB & 3) % G;
    const float sA = __shfl_sync(kFull, l, 4 * hA);
    const float sB = __shfl_sync(kFull, l, 4 * hB);
    const float mA = __shfl_sync(kFull, m_run, 4 * hA);
    const float mB = __shfl_sync(kFull, m_run, 4 * hB);
    const float f = pow2i(e_run);
    const bool wA = c < 2 && nA < G, wB = c < 2 && nB < G;
    float o[32];
    if (of_live) {
      tm_ld32(otm, o);
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) o[k] = 0.0f;
    }
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = m * 4 + e;
        float v = o[k];
        v += __shfl_xor_sync(kFull, v, 2);
        // m-tile m: chunk q = m / 2 (dims 32q..), odd dims when m is odd;
        // rows r / r+8 are bytes r / r+8 of the chunk
        const int d = 32 * (m >> 1) + 2 * r + ((e & 2) ? 16 : 0) + (m & 1);
        if (e & 1) {
          if (wB) sk.put_o(nB, d, v * f, sB);
        } else {
          if (wA) sk.put_o(nA, d, v * f, sA);
        }
      }
    if (r == 0) {
      if (wA) sk.put_ml(nA, mA, sA);
      if (wB) sk.put_ml(nB, mB, sB);
    }
  }
};
}  // namespace
}  // namespace kv8
