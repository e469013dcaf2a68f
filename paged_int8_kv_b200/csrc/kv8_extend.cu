// kv8_extend.cu -- extend (prefill) attention over the paged INT8 cache on
// the 5th-generation tensor cores.
//
// What is computed [KV Cache 优化全景解析——从基础原理到工程实践, §2.1, §2.2,
// §11.2; KV-Cache 全栈优化系统, 主要特性]: the n_b new query rows of each
// sequence b (its last n_b cached positions, appended before the call) attend
// causally over the dequantised cache, row i at position
// p = context_lens[b] - n_b + i seeing tokens 0..p:
//     out = softmax(q K_hat^T / sqrt(d)) V_hat,  K_hat = code ks, V_hat = code vs.
//
// Tiles.  A work item is (sequence, KV head, query tile): 128 rows, each a
// (position, head) pair of the KV head's G query heads (128 / G positions).
// Keys come in tiles of 128 tokens (8 pages).  Both products are dense
// 128 x 128 x 128 contractions on tcgen05 (kind::f16, fp32 accumulators in
// tensor memory):
//   S[128 rows][128 keys]  = Q16 . K16^T    Q16: q rows scaled by an exact
//                                           power of two into fp16; K16: the
//                                           K codes, exact in fp16
//   O[128 rows][128 dims] += P16 . V16      P16: 2^(s - m) vs 2^-E in fp16;
//                                           V16: the V codes, exact in fp16
// The K scale is applied to S and the V scale folded into P, per key.
//
// CTA (12 warps, one per SM, persistent over items; the producer, issuer
// and converter roles and the key-tile softmax live in kv8_tc.cuh, shared
// with the shared-prefix kernel):
//   warp 0      TMA producer: each key tile's 8 K pages, 8 V pages and their
//               scales into a 2-stage ring;
//   warp 1      MMA issuer (one thread): S of tile j+1 is issued before O of
//               tile j, so the tensor cores compute the next scores while
//               the softmax warps work;
//   warps 2-3   converters: int8 codes -> fp16 operand tiles (128-byte
//               swizzle) in shared memory, scales copied aside;
//   warps 4-11  softmax, two warps per tensor-memory lane quarter, one row
//               per thread, each of the pair taking 64 key columns and 64
//               output dims of its rows: loads the item's q rows, reads S,
//               masks causally, meets its partner once per tile for the
//               row's maxima, keeps a base-2 online softmax with lazy moves
//               of the reference max m and of the V-scale exponent E
//               (rescaling O in tensor memory only then), writes P16, and at
//               the end normalises and stores O.
// Roles hand over through mbarriers only; every wait is bounded in time and
// records a status bit on timeout.
#include <cuda_fp16.h>

#include "../../include/kv8.h"
#include "kv8_common.cuh"
#include "kv8_internal.h"
#include "kv8_tc.cuh"

namespace kv8 {

__device__ uint32_t g_ext_status = 0;

namespace {

struct ExtParams {
  const __nv_bfloat16* q;       // [q_total][Hq][128]
  const float* k_scales;
  const float* v_scales;
  const int32_t* block_tables;  // [B][MBS]
  const int32_t* context_lens;  // [B]
  const int32_t* q_start;       // [B+1]
  void* out;                    // [q_total][Hq][128]
  int32_t batch, num_q_heads, num_kv_heads, max_blocks_per_seq;
  int32_t q_tiles;              // ceil(max_q_len / positions per tile)
  int32_t out_f32;
  float q_scale;                // softmax_scale * log2(e)
};

struct ExtItem {
  int b, kvh, qt;
  int t_ctx, n_new, i0, npos;  // context, new rows, first row, rows here
  int nkt;                     // key tiles
};

// Item idx = (qt * H_kv + kvh) * B + b; false if the query tile is empty.
__device__ __forceinline__ bool eitem_load(const ExtParams& p, int64_t idx,
                                           int P, ExtItem& it) {
  it.b = static_cast<int>(idx % p.batch);
  const int64_t r = idx / p.batch;
  it.kvh = static_cast<int>(r % p.num_kv_heads);
  it.qt = static_cast<int>(r / p.num_kv_heads);
  const int qs = p.q_start[it.b];
  it.n_new = p.q_start[it.b + 1] - qs;
  it.i0 = it.qt * P;
  if (it.i0 >= it.n_new) return false;
  it.t_ctx = p.context_lens[it.b];
  it.npos = min(P, it.n_new - it.i0);
  const int keys = it.t_ctx - it.n_new + it.i0 + it.npos;  // last row's view
  it.nkt = (keys + kKT - 1) / kKT;
  return true;
}

// The extend items as the producer, issuer and converter roles see them.
struct ExtItems {
  const ExtParams& p;
  int P;
  __device__ __forceinline__ int64_t size() const {
    return static_cast<int64_t>(p.q_tiles) * p.num_kv_heads * p.batch;
  }
  __device__ __forceinline__ bool load(int64_t idx, TileItem& t, int) const {
    ExtItem it;
    if (!eitem_load(p, idx, P, it)) return false;
    const int keys = it.t_ctx - it.n_new + it.i0 + it.npos;  // last row's view
    t.tab = static_cast<int64_t>(it.b) * p.max_blocks_per_seq;
    t.kvh = it.kvh;
    t.npages = (keys + kBS - 1) / kBS;
    t.nkt = it.nkt;
    return true;
  }
};

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
extend_kernel(const ExtParams p, const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv) {
  constexpr int P = kRows / G;  // positions per item
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ExtPlan::kBar);
  const uint32_t tmem = tc_setup(smem, &tmk, &tmv, warp);

  const int64_t n_items =
      static_cast<int64_t>(p.q_tiles) * p.num_kv_heads * p.batch;
  bool failed = false;

  const ExtItems items{p, P};
  if (warp == 0) {
    tc_produce(items, p.block_tables, p.num_kv_heads, p.k_scales, p.v_scales,
               &tmk, &tmv, smem, bars, failed, &g_ext_status, lane);
  } else if (warp == 1) {
    tc_issue(items, smem, bars, tmem, failed, &g_ext_status, lane);
  } else if (warp < 4) {
    tc_convert(items, smem, bars, failed, &g_ext_status, threadIdx.x - 64, lane);
  } else {
    // ================================================= softmax (8 warps)
    // rows r = 32 qd + lane (tensor-memory lane quarter qd); half hf takes
    // key columns and output dims 64 hf .. 64 hf + 63
    const int sw = warp - 4, qd = sw & 3, hf = sw >> 2;
    const int r = 32 * qd + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * qd) << 16);
    const int pos = r / G, head = r % G;
    uint32_t u = 0, xk = 0;
    for (int64_t idx = blockIdx.x; idx < n_items; idx += gridDim.x) {
      ExtItem it;
      if (!eitem_load(p, idx, P, it)) continue;
      const bool live = pos < it.npos;
      const int64_t qrow =
          static_cast<int64_t>(p.q_start[it.b] + it.i0 + pos) * p.num_q_heads +
          it.kvh * G + head;
      const float qf =
          tc_stage_q(smem, p.q + qrow * kD, live, r, hf, qd, p.q_scale, xk);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_Q_FULL]);
      {
        // the next item's q row (this half: 128 bytes) into L1 while this
        // item's tiles run, so its staging does not wait on L2
        ExtItem nx;
        if (idx + gridDim.x < n_items && eitem_load(p, idx + gridDim.x, P, nx) &&
            pos < nx.npos) {
          const int64_t nrow =
              static_cast<int64_t>(p.q_start[nx.b] + nx.i0 + pos) * p.num_q_heads +
              nx.kvh * G + head;
          asm volatile("prefetch.global.L1 [%0];" ::"l"(
              reinterpret_cast<const char*>(p.q + nrow * kD) + 128 * hf));
        }
      }

      // ---- key tiles
      const int key_lim = it.t_ctx - it.n_new + it.i0 + pos + 1;  // keys < this
      const RowSoftmax rs =
          tc_row_tiles(smem, bars, trow, r, hf, qd, lane, live, key_lim, qf,
                       it.nkt, u, xk, failed, &g_ext_status);
      u += it.nkt;
      const float l = rs.l + pair_xch(smem, xk, hf, r, qd, make_float2(rs.l, 0.0f)).x;
      // ---- output: wait for the last O product, normalise, store this
      // half's dims
      ewait(&bars[B_O_DONE], (u - 1) & 1, failed, &g_ext_status);
      __syncwarp();
      tc_fence_after();
      const float f = pow2i(rs.e) / (l > 0.0f ? l : 1.0f);
#pragma unroll 1
      for (int c = 0; c < kHalf / 32; ++c) {
        float o[32];
        const int d0 = kHalf * hf + 32 * c;
        __syncwarp();  // the stores below diverge by row; reconverge first
        tmem_ld32(trow + kColO + d0, o);
        if (live) {
          if (p.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) +
                                                    qrow * kD + d0);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(o[4 * i] * f, o[4 * i + 1] * f,
                                   o[4 * i + 2] * f, o[4 * i + 3] * f);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(
                static_cast<__nv_bfloat16*>(p.out) + qrow * kD + d0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint32_t w[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(
                    o[8 * i + 2 * k] * f, o[8 * i + 2 * k + 1] * f);
                w[k] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      tc_fence_before();
    }
  }

  tc_teardown(tmem, warp);
}

template <int G>
int launch_extend_group(const ExtParams& p, const CUtensorMap& tmk,
                        const CUtensorMap& tmv, cudaStream_t stream) {
  auto kern = extend_kernel<G>;
  constexpr int smem = ExtPlan::kBytes;
  static LaunchFacts table[kMaxDevices];
  LaunchFacts* f = facts_for_current_device(table);
  if (!f) return -1;
  int sms = f->sms.load(std::memory_order_acquire);
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return -1;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
        cudaSuccess)
      return -1;
    f->resident.store(1, std::memory_order_release);
    f->sms.store(sms, std::memory_order_release);
  }
  const int64_t n_items =
      static_cast<int64_t>(p.q_tiles) * p.num_kv_heads * p.batch;
  if (n_items == 0) return 0;
  int64_t ctas = sms;
  if (ctas > n_items) ctas = n_items;
  kern<<<static_cast<unsigned>(ctas), kThreads, smem, stream>>>(p, tmk, tmv);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

int launch_extend(const void* q, const float* k_scales, const float* v_scales,
                  const int32_t* block_tables, const int32_t* context_lens,
                  const int32_t* q_start, int32_t batch, int32_t num_q_heads,
                  int32_t num_kv_heads, int32_t max_blocks_per_seq,
                  int32_t max_q_len, float softmax_scale, void* out,
                  int32_t out_f32, const CUtensorMap& tmk,
                  const CUtensorMap& tmv, cudaStream_t stream) {
  const int g = num_q_heads / num_kv_heads;
  ExtParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_scales = k_scales;
  p.v_scales = v_scales;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.q_start = q_start;
  p.out = out;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.out_f32 = out_f32;
  p.q_scale = static_cast<float>(static_cast<double>(softmax_scale) *
                                 1.4426950408889634074);
  const int P = kRows / g;
  p.q_tiles = (max_q_len + P - 1) / P;
  switch (g) {
    case 1: return launch_extend_group<1>(p, tmk, tmv, stream);
    case 2: return launch_extend_group<2>(p, tmk, tmv, stream);
    case 4: return launch_extend_group<4>(p, tmk, tmv, stream);
    case 8: return launch_extend_group<8>(p, tmk, tmv, stream);
    default: return -2;
  }
}

int read_ext_status(uint32_t* value, int clear) {
  if (cudaMemcpyFromSymbol(value, g_ext_status, sizeof(uint32_t)) != cudaSuccess)
    return -1;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_ext_status, &zero, sizeof(uint32_t)) != cudaSuccess)
      return -1;
  }
  return 0;
}

}  // namespace kv8
