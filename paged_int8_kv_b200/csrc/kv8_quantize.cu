// kv8_quantize.cu -- per-(token, KV head) dynamic INT8 quantisation of new
// K/V rows, scattered into the paged cache through a slot mapping.
//
// Method [KV-Cache 全栈优化系统, 主要特性]: K/V are quantised per token to
// INT8 when written.  Group = one KV head's head_dim = 128 values
// [大模型推理加速：KV Cache与vLLM技术解析, §4.1].  Scale s = fl32(max|x|/127),
// code = clamp(rint(fl32(x/s)), -127, 127), both divisions IEEE round to
// nearest (no reciprocal multiply), rint ties to even, so the codes are
// bit-identical to a plain CPU implementation.
//
// Mapping: one warp per (token, KV head, K-or-V) row of 128 bf16 (256 B):
// each lane reads 4 values (8 B), the warp reduces the max with shuffles,
// each lane writes its 4 codes as one 32-bit word (a 128-B coalesced row)
// and lane 0 writes the scale.  The work is HBM-bound and tiny per decode
// step (batch x H_kv x 2 rows).
#include "kv8_common.cuh"
#include "kv8_internal.h"

namespace kv8 {

namespace {

constexpr int kD = 128;
constexpr int kBS = 16;

// Levels each side of zero: 127 for INT8 codes, 7 for INT4 codes.
template <int Bits>
__device__ __forceinline__ int quant_one(float x, float s) {
  constexpr float kL = Bits == 8 ? 127.0f : 7.0f;
  if (s == 0.0f) return 0;
  float r = rintf(__fdiv_rn(x, s));
  r = fminf(fmaxf(r, -kL), kL);
  return static_cast<int>(r);
}

// Bits == 8: int8 codes, one 128-byte row per (token, KV head).
// Bits == 4: the INT4 variant [nano-KvLLM, §2.2: historical tokens' K/V in
// 4 bits]: s = fl32(max|x|/7), codes clamped to +-7 and stored as the
// nibble code + 8, dims 2i / 2i+1 in the low / high nibble of byte i; one
// 64-byte row per (token, KV head).
template <int Bits>
__global__ void __launch_bounds__(256)
quantize_append_kernel(const __nv_bfloat16* __restrict__ k_new,
                       const __nv_bfloat16* __restrict__ v_new,
                       const int64_t* __restrict__ slot_mapping,
                       int64_t n_rows,  // n_tokens * H_kv * 2
                       int32_t num_kv_heads, int8_t* __restrict__ k_cache,
                       int8_t* __restrict__ v_cache,
                       float* __restrict__ k_scales,
                       float* __restrict__ v_scales) {
  constexpr float kL = Bits == 8 ? 127.0f : 7.0f;
  constexpr int kRowBytes = kD * Bits / 8;
  const int lane = threadIdx.x & 31;
  const int64_t warps_total =
      static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) +
                     (threadIdx.x >> 5);
       row < n_rows; row += warps_total) {
    const int which = static_cast<int>(row & 1);  // 0 = K, 1 = V
    const int64_t th = row >> 1;                 // token * H_kv + head
    const int64_t tok = th / num_kv_heads;
    const int h = static_cast<int>(th - tok * num_kv_heads);
    const int64_t slot = slot_mapping[tok];
    if (slot < 0) continue;  // padding token
    const __nv_bfloat16* src = (which ? v_new : k_new) + th * kD;
    const uint2 raw = reinterpret_cast<const uint2*>(src)[lane];
    float x[4];
    x[0] = __uint_as_float(raw.x << 16);
    x[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    x[2] = __uint_as_float(raw.y << 16);
    x[3] = __uint_as_float(raw.y & 0xFFFF0000u);
    float a = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])),
                    fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1)
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, m));
    const float s = (a == 0.0f) ? 0.0f : __fdiv_rn(a, kL);
    const int64_t blk = slot / kBS;
    const int64_t off = slot - blk * kBS;
    const int64_t base = (blk * num_kv_heads + h) * kBS + off;
    int8_t* dst = (which ? v_cache : k_cache) + base * kRowBytes;
    if constexpr (Bits == 8) {
      uint32_t packed = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        packed |= (static_cast<uint32_t>(quant_one<8>(x[i], s)) & 0xFFu) << (8 * i);
      reinterpret_cast<uint32_t*>(dst)[lane] = packed;
    } else {
      uint32_t packed = 0;  // dims 4 lane .. 4 lane + 3 -> two bytes
#pragma unroll
      for (int i = 0; i < 4; ++i)
        packed |= static_cast<uint32_t>(quant_one<4>(x[i], s) + 8) << (4 * i);
      reinterpret_cast<uint16_t*>(dst)[lane] = static_cast<uint16_t>(packed);
    }
    if (lane == 0) (which ? v_scales : k_scales)[base] = s;
  }
}

}  // namespace

int launch_quantize_append(const void* k_new, const void* v_new,
                           const int64_t* slot_mapping, int64_t n_tokens,
                           int32_t num_kv_heads, int8_t* k_cache,
                           int8_t* v_cache, float* k_scales, float* v_scales,
                           cudaStream_t stream, int32_t bits) {
  const int64_t n_rows = n_tokens * num_kv_heads * 2;
  const int threads = 256;
  const int64_t warps_per_block = threads / 32;
  int64_t blocks = (n_rows + warps_per_block - 1) / warps_per_block;
  if (blocks > 148 * 64) blocks = 148 * 64;  // grid-stride beyond this
  auto kern = bits == 4 ? quantize_append_kernel<4> : quantize_append_kernel<8>;
  kern<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(k_new),
      static_cast<const __nv_bfloat16*>(v_new), slot_mapping, n_rows,
      num_kv_heads, k_cache, v_cache, k_scales, v_scales);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace kv8
