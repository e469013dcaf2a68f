// kv8_common.cuh -- small sm_100a building blocks shared by the kv8 kernels:
// mbarrier phases with bounded waits, TMA bulk and tensor copies into shared
// memory, and a sticky device status word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kv8 {

// Sticky device status bits: a kernel ORs them into a status word owned by
// its translation unit (kv8_read_device_status() reads and clears it).  A
// wait that gives up sets KV8_DEV_WAIT_TIMEOUT and the kernel skips the rest
// of its work instead of hanging.
enum : uint32_t {
  KV8_DEV_WAIT_TIMEOUT = 1u,
  // a shared-prefix group listed a member whose context is shorter than the
  // group's prefix; that member's shared chunks were skipped
  KV8_DEV_BAD_PREFIX = 2u,
};

// Upper bound on mbarrier polls before a wait gives up (each poll may also
// suspend the thread for a short hardware-chosen time): far above any real
// latency of a 4 KB copy, a second or so in the worst case.  The test-hook
// build (KV8_TEST_HOOKS) gives up after a few milliseconds instead, so that
// its test of the give-up path is short.
#ifdef KV8_TEST_HOOKS
constexpr uint32_t kMaxWaitPolls = 1u << 12;
#else
constexpr uint32_t kMaxWaitPolls = 1u << 24;
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) writes to the same addresses.
// Order this thread's earlier generic-proxy global writes before its later
// async-proxy (TMA) reads of the same addresses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar,
                                                      uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of `bar` to complete.  Returns false (and
// raises the sticky timeout bit) if it never does.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint32_t* status) {
  for (uint32_t i = 0; i < kMaxWaitPolls; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
  }
  atomicOr(status, KV8_DEV_WAIT_TIMEOUT);
  return false;
}

// 1-D bulk copy global -> shared, completing `bytes` of transaction on `bar`.
// src, dst 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src,
                                         uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// The same operations on 32-bit shared addresses (no address conversion at
// each call).
__device__ __forceinline__ void mbar_arrive_expect_tx_s(uint32_t bar,
                                                        uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                   bar),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_wait_s(uint32_t bar, uint32_t parity,
                                            uint32_t* status) {
  for (uint32_t i = 0; i < kMaxWaitPolls; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  atomicOr(status, KV8_DEV_WAIT_TIMEOUT);
  return false;
}
__device__ __forceinline__ void bulk_g2s_s(uint32_t dst, const void* src,
                                           uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_s(uint32_t dst, const CUtensorMap* map,
                                              int32_t c0, int32_t c1, int32_t c2,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_"
      "tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// 3-D tiled tensor copy global -> shared through a tensor map (no multicast).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map,
                                            int32_t c0, int32_t c1, int32_t c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_"
      "tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2),
      "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map))
               : "memory");
}

// Packed fp32x2 fused multiply-add (sm_100 f32x2 ALU form).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(*reinterpret_cast<uint64_t*>(&d))
      : "l"(*reinterpret_cast<uint64_t*>(&a)),
        "l"(*reinterpret_cast<uint64_t*>(&b)),
        "l"(*reinterpret_cast<uint64_t*>(&c)));
  return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(*reinterpret_cast<uint64_t*>(&d))
      : "l"(*reinterpret_cast<uint64_t*>(&a)),
        "l"(*reinterpret_cast<uint64_t*>(&b)));
  return d;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(*reinterpret_cast<uint64_t*>(&d))
      : "l"(*reinterpret_cast<uint64_t*>(&a)),
        "l"(*reinterpret_cast<uint64_t*>(&b)));
  return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Four signed int8 codes (one 32-bit word) -> four exact fp32 values.
// Each byte is biased to unsigned (c + 128) and placed in the low mantissa
// bits of 2^23, which makes the float 2^23 + 128 + c exactly; subtracting
// 2^23 + 128 leaves c exactly.  Pairs come out as (byte0, byte1) and
// (byte2, byte3).
__device__ __forceinline__ void i8x4_to_f32(uint32_t w, float2& lo, float2& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const float2 nbias = make_float2(-8388736.0f, -8388736.0f);  // -(2^23+128)
  float2 a, b;
  a.x = __uint_as_float(prmt(u, 0x4B000000u, 0x7650u));
  a.y = __uint_as_float(prmt(u, 0x4B000000u, 0x7651u));
  b.x = __uint_as_float(prmt(u, 0x4B000000u, 0x7652u));
  b.y = __uint_as_float(prmt(u, 0x4B000000u, 0x7653u));
  lo = fadd2(a, nbias);
  hi = fadd2(b, nbias);
}

}  // namespace kv8
