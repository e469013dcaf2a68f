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

// --------------------------------------------------------------------------
// CUDA-core (FP32 FMA) page math.
//   G <= 4: a lane covers 16 dims of one token (8 lanes per token,
//           4 tokens per pass, 4 passes per page);
//   G == 8: 8 dims (16 lanes per token, 2 tokens per pass, 8 passes).
// --------------------------------------------------------------------------
template <int G, int NW, int SPW>
__global__ void __launch_bounds__(NW * 32)
decode_simt_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv) {
  constexpr int DPL = (G <= 4) ? 16 : 8;  // dims per lane
  constexpr int LPT = kD / DPL;           // lanes per token
  constexpr int TPP = 32 / LPT;           // tokens per pass
  constexpr int NPASS = kBS / TPP;        // passes per page
  constexpr int HSTRIDE = LPT / G;        // lanes per head after reduction
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

  // ---- per-lane constants
  const int tg = lane / LPT;   // token within a pass
  const int dg = lane % LPT;   // dim group
  const int hh = lane_head<G, LPT>(dg);

  // q for the G heads of this group, this lane's DPL dims, pre-scaled by
  // softmax_scale * log2(e) so that scores come out in base-2 units.
  float2 q2[G][DPL / 2];
  {
    const __nv_bfloat16* qg =
        p.q + (static_cast<int64_t>(b) * p.num_q_heads + kvh * G) * kD +
        dg * DPL;
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int i = 0; i < DPL / 8; ++i) {
        const uint4 raw = reinterpret_cast<const uint4*>(qg + h * kD)[i];
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          q2[h][i * 4 + j] =
              make_float2(__uint_as_float(w[j] << 16) * p.q_scale,
                          __uint_as_float(w[j] & 0xFFFF0000u) * p.q_scale);
        }
      }
    }
  }

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
      fence_proxy_async_smem();
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

  // ---- running softmax state (per lane: head hh) and output accumulators
  float m_run = -INFINITY;
  float l_run = 0.0f;
  float2 o2[G][DPL / 2];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int i = 0; i < DPL / 2; ++i) o2[h][i] = make_float2(0.f, 0.f);

  bool ok = true;
  int k = 0;
  for (; k < my_pages; ++k) {
    const int s = k % SPW;
    if (!mbar_wait(&bars[s], (k / SPW) & 1, &g_device_status)) {
      ok = false;
      break;
    }
    const uint8_t* tk = tiles + s * 2 * kPageBytes;
    const uint8_t* tv = tk + kPageBytes;
    const float* ks = scl + s * 2 * kBS;
    const float* vs = ks + kBS;
    const int tbase = tok0 + (warp + k * NW) * kBS;

    // ---- scores for this lane's tokens (head hh)
    float sc[NPASS];
#pragma unroll
    for (int ps = 0; ps < NPASS; ++ps) {
      const int t = ps * TPP + tg;
      // swizzled 16-byte chunk holding dims [dg*DPL, dg*DPL + DPL)
      const int chunk16 = (dg * DPL) / 16;
      const uint8_t* row = tk + t * 128 + ((chunk16 ^ (t & 7)) << 4) +
                           ((dg * DPL) & 15);
      float2 kf[DPL / 2];
      if constexpr (DPL == 16) {
        const uint4 w = *reinterpret_cast<const uint4*>(row);
        i8x4_to_f32(w.x, kf[0], kf[1]);
        i8x4_to_f32(w.y, kf[2], kf[3]);
        i8x4_to_f32(w.z, kf[4], kf[5]);
        i8x4_to_f32(w.w, kf[6], kf[7]);
      } else {
        const uint2 w = *reinterpret_cast<const uint2*>(row);
        i8x4_to_f32(w.x, kf[0], kf[1]);
        i8x4_to_f32(w.y, kf[2], kf[3]);
      }
      float acc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i) a = ffma2(q2[h][i], kf[i], a);
        acc[h] = a.x + a.y;
      }
      const float dot = reduce_heads<G, LPT>(acc, lane);
      const bool valid = tbase + t < tok1;
      sc[ps] = valid ? dot * ks[t] : -INFINITY;
    }

    // ---- online softmax update (per head; heads live in lane groups)
    float mx = sc[0];
#pragma unroll
    for (int ps = 1; ps < NPASS; ++ps) mx = fmaxf(mx, sc[ps]);
#pragma unroll
    for (int m = LPT; m < 32; m <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
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
      pv[ps] = (tbase + t < tok1) ? pr * vs[t] : 0.0f;
    }
    l_run = l_run * alpha + psum;
    m_run = m_new;

    // ---- rescale the accumulators when some head's max moved
    if (__any_sync(kFull, alpha != 1.0f)) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float a = __shfl_sync(kFull, alpha, h * HSTRIDE);
        const float2 a2 = make_float2(a, a);
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i) o2[h][i] = fmul2(o2[h][i], a2);
      }
    }

    // ---- o += p * v_code for this lane's tokens and dims
#pragma unroll
    for (int ps = 0; ps < NPASS; ++ps) {
      const int t = ps * TPP + tg;
      const int chunk16 = (dg * DPL) / 16;
      const uint8_t* row = tv + t * 128 + ((chunk16 ^ (t & 7)) << 4) +
                           ((dg * DPL) & 15);
      float2 vf[DPL / 2];
      if constexpr (DPL == 16) {
        const uint4 w = *reinterpret_cast<const uint4*>(row);
        i8x4_to_f32(w.x, vf[0], vf[1]);
        i8x4_to_f32(w.y, vf[2], vf[3]);
        i8x4_to_f32(w.z, vf[4], vf[5]);
        i8x4_to_f32(w.w, vf[6], vf[7]);
      } else {
        const uint2 w = *reinterpret_cast<const uint2*>(row);
        i8x4_to_f32(w.x, vf[0], vf[1]);
        i8x4_to_f32(w.y, vf[2], vf[3]);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float ph = __shfl_sync(kFull, pv[ps], tg * LPT + h * HSTRIDE);
        const float2 p2 = make_float2(ph, ph);
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i) o2[h][i] = ffma2(p2, vf[i], o2[h][i]);
      }
    }

    __syncwarp();
    if (k + SPW < my_pages) issue(k + SPW);
  }

  if (!ok) {
    // A copy never landed: drain what is still in flight (bounded), then
    // contribute nothing to the merge.  The sticky status word reports it.
    for (int kk = k + 1; kk < my_pages && kk < k + SPW; ++kk)
      mbar_wait(&bars[kk % SPW], (kk / SPW) & 1, &g_device_status);
    m_run = -INFINITY;
    l_run = 0.0f;
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < DPL / 2; ++i) o2[h][i] = make_float2(0.f, 0.f);
  }

  // ---- fold the TPP token groups of this warp together
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
  for (int m = LPT; m < 32; m <<= 1) l_lane += __shfl_xor_sync(kFull, l_lane, m);

  // ---- warp merge record in this warp's own (now idle) tiles
  __syncwarp();
  float* rec = reinterpret_cast<float*>(tiles);
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
  __syncthreads();

  // ---- merge the NW warp records and write
  const bool single = nchunks <= 1;
  for (int idx = threadIdx.x; idx < G * kD; idx += NW * 32) {
    const int h = idx / kD;
    const int d = idx % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* r = reinterpret_cast<const float*>(smem + w * SPW * 2 * kPageBytes);
      M = fmaxf(M, r[G * kD + h]);
    }
    float L = 0.0f, O = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* r = reinterpret_cast<const float*>(smem + w * SPW * 2 * kPageBytes);
      const float mw = r[G * kD + h];
      const float e = (mw == -INFINITY) ? 0.0f : exp2f(mw - M);
      L += r[G * kD + G + h] * e;
      O += r[h * kD + d] * e;
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
}

// --------------------------------------------------------------------------
// Split reduce: one CTA of 128 threads (one per output dim) per (b, hq).
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
split_reduce_kernel(const float* __restrict__ ws_ml,
                    const float* __restrict__ ws_o,
                    const int32_t* __restrict__ context_lens, int32_t num_q_heads,
                    int32_t chunk_tokens, int32_t max_chunks, void* out,
                    int32_t out_f32) {
  const int bh = blockIdx.x;
  const int b = bh / num_q_heads;
  const int n = context_lens[b];
  const int nchunks = (n + chunk_tokens - 1) / chunk_tokens;
  if (nchunks <= 1) return;
  const int d = threadIdx.x;
  const float* ml = ws_ml + static_cast<int64_t>(bh) * max_chunks * 2;
  const float* o = ws_o + static_cast<int64_t>(bh) * max_chunks * kD;
  float M = -INFINITY;
  for (int c = 0; c < nchunks; ++c) M = fmaxf(M, ml[2 * c]);
  float L = 0.0f, O = 0.0f;
  for (int c = 0; c < nchunks; ++c) {
    const float mc = ml[2 * c];
    const float e = (mc == -INFINITY) ? 0.0f : exp2f(mc - M);
    L += ml[2 * c + 1] * e;
    O += o[static_cast<int64_t>(c) * kD + d] * e;
  }
  store_out(out, static_cast<int64_t>(bh) * kD + d, L > 0.0f ? O / L : 0.0f,
            out_f32);
}

template <int G, int NW, int SPW>
int launch_simt(const DecodeParams& p, const CUtensorMap& tmk,
                const CUtensorMap& tmv, cudaStream_t stream) {
  auto kern = decode_simt_kernel<G, NW, SPW>;
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

size_t workspace_total_bytes(int32_t batch, int32_t num_q_heads,
                             int32_t max_chunks) {
  return workspace_ml_bytes(batch, num_q_heads, max_chunks) +
         static_cast<size_t>(batch) * num_q_heads * max_chunks * kD *
             sizeof(float);
}

int launch_decode(const DecodeParams& p, const CUtensorMap& tmk,
                  const CUtensorMap& tmv, int32_t variant,
                  cudaStream_t stream) {
  (void)variant;
  const int g = p.num_q_heads / p.num_kv_heads;
  switch (g) {
    case 1: return launch_simt<1, 4, 4>(p, tmk, tmv, stream);
    case 2: return launch_simt<2, 4, 4>(p, tmk, tmv, stream);
    case 4: return launch_simt<4, 4, 4>(p, tmk, tmv, stream);
    case 8: return launch_simt<8, 4, 4>(p, tmk, tmv, stream);
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
  split_reduce_kernel<<<static_cast<unsigned>(nbh), kD, 0, stream>>>(
      ws_ml, ws_o, context_lens, num_q_heads, chunk_tokens, max_chunks, out,
      out_f32);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace kv8
