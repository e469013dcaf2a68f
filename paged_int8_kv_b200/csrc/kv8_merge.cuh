// kv8_merge.cuh -- device helpers shared by the decode kernels and the
// standalone split reduce: output store, base-2 exponential, power-of-two
// helpers and the log-sum-exp merge of chunk partials.  Every translation
// unit that merges partials uses this one routine, so a fused merge and the
// standalone reduce give bit-identical rows.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "kv8_internal.h"

namespace kv8 {
namespace {

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
// row, by one warp: chunk c holds m_c (base-2 max), l_c (sum of
// 2^(s - m_c)) and o_c[d] (sum of 2^(s - m_c) v_hat[d]); an empty slot
// (m_c = -inf: no token, or a slot whose chunk another slot's partial
// covers) contributes nothing and its o_c is not read;
//   M = max_c m_c,  L = sum_c l_c 2^(m_c - M),
//   out[d] = sum_c o_c[d] 2^(m_c - M) / L.
// Lanes split the chunks for M and L, then each lane accumulates 4 dims over
// all chunks with float4 loads.  The fused merge of a split decode and the
// standalone reduce kernel both call it, so they give identical results.
__device__ __forceinline__ void merge_head_warp(const float* ml, const float* o,
                                                int nchunks, void* out,
                                                int64_t out_row, int out_f32) {
  const int lane = threadIdx.x & 31;
  float mx = -INFINITY;
  for (int c = lane; c < nchunks; c += 32) mx = fmaxf(mx, __ldcg(&ml[2 * c]));
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
  float ls = 0.0f;
  for (int c = lane; c < nchunks; c += 32) {
    const float mc = __ldcg(&ml[2 * c]);
    ls += (mc == -INFINITY) ? 0.0f : __ldcg(&ml[2 * c + 1]) * ex2(mc - mx);
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, m);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
  for (int c = 0; c < nchunks; ++c) {
    const float mc = __ldcg(&ml[2 * c]);
    if (mc == -INFINITY) continue;  // an empty slot: its o is not read
    const float w = ex2(mc - mx);
    const float4 v =
        __ldcg(reinterpret_cast<const float4*>(o + static_cast<int64_t>(c) * kHeadDim) + lane);
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  const float inv = ls > 0.0f ? 1.0f / ls : 0.0f;
  const int64_t base = out_row * kHeadDim + 4 * lane;
  store_out(out, base + 0, acc.x * inv, out_f32);
  store_out(out, base + 1, acc.y * inv, out_f32);
  store_out(out, base + 2, acc.z * inv, out_f32);
  store_out(out, base + 3, acc.w * inv, out_f32);
}

// merge_head_warp for the G consecutive query heads row0 .. row0 + G - 1
// of a KV group (partials at ws_ml + row * max_chunks * 2, ws_o + row *
// max_chunks * kHeadDim): the same arithmetic, in the same order, per head
// (so the results equal G calls of merge_head_warp bit for bit), with the
// heads' loads of each chunk issued together so that G times more of them
// are in flight.
template <int G>
__device__ __forceinline__ void merge_group_warp(const float* ws_ml,
                                                 const float* ws_o,
                                                 int64_t row0, int max_chunks,
                                                 int nchunks, void* out,
                                                 int out_f32) {
  const int lane = threadIdx.x & 31;
  float mx[G], ls[G];
#pragma unroll
  for (int h = 0; h < G; ++h) mx[h] = -INFINITY;
  for (int c = lane; c < nchunks; c += 32)
#pragma unroll
    for (int h = 0; h < G; ++h)
      mx[h] = fmaxf(mx[h], __ldcg(&ws_ml[((row0 + h) * max_chunks + c) * 2]));
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1)
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], m));
    ls[h] = 0.0f;
  }
  for (int c = lane; c < nchunks; c += 32)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float* ml = ws_ml + ((row0 + h) * max_chunks + c) * 2;
      const float mc = __ldcg(&ml[0]);
      ls[h] += (mc == -INFINITY) ? 0.0f : __ldcg(&ml[1]) * ex2(mc - mx[h]);
    }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) ls[h] += __shfl_xor_sync(0xffffffffu, ls[h], m);
  float4 acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
  for (int c = 0; c < nchunks; ++c) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const int64_t ci = (row0 + h) * max_chunks + c;
      const float mc = __ldcg(&ws_ml[2 * ci]);
      if (mc == -INFINITY) continue;  // an empty slot: its o is not read
      const float w = ex2(mc - mx[h]);
      const float4 v =
          __ldcg(reinterpret_cast<const float4*>(ws_o + ci * kHeadDim) + lane);
      acc[h].x += w * v.x;
      acc[h].y += w * v.y;
      acc[h].z += w * v.z;
      acc[h].w += w * v.w;
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float inv = ls[h] > 0.0f ? 1.0f / ls[h] : 0.0f;
    const int64_t base = (row0 + h) * kHeadDim + 4 * lane;
    store_out(out, base + 0, acc[h].x * inv, out_f32);
    store_out(out, base + 1, acc[h].y * inv, out_f32);
    store_out(out, base + 2, acc[h].z * inv, out_f32);
    store_out(out, base + 3, acc[h].w * inv, out_f32);
  }
}

}  // namespace
}  // namespace kv8
