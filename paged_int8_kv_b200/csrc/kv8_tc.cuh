// kv8_tc.cuh -- the 5th-generation tensor-core pieces shared by the kernels
// that attend many query rows to 128-key tiles of the paged INT8 cache (the
// extend kernel and the shared-prefix kernel): the shared-memory plan, the
// role barriers, tcgen05 descriptors and instructions, tensor-memory loads
// and stores, the bounded wait and the int8 -> fp16 operand conversion.
#pragma once

#include <cuda_fp16.h>

#include "../../include/kv8.h"
#include "kv8_common.cuh"
#include "kv8_internal.h"
#include "kv8_merge.cuh"

namespace kv8 {
namespace {

constexpr int kD = kHeadDim;
constexpr int kBS = kBlockSize;
constexpr uint32_t kFull = 0xffffffffu;
constexpr int kKT = 128;              // keys per tile
constexpr int kTilePages = kKT / kBS;  // 8
constexpr int kRows = 128;            // query rows per item (MMA M)
// warps: 0 TMA producer, 1 MMA issuer, 2-3 converters, 4-11 softmax (two
// per tensor-memory lane quarter: warp 4 + q and 8 + q hold the same 32 rows,
// one the key columns / output dims 0..63, the other 64..127)
constexpr int kThreads = 384;
constexpr int kHalf = 64;             // columns per softmax thread
constexpr int kTmemCols = 512;        // S[2] (256) + O (128), power of two
constexpr uint32_t kColS = 0, kColO = 256;
constexpr float kSlack = 8.0f;        // scores may pass m by 2^8 before m moves
constexpr int kVSlack = 2;            // V scales may pass 2^E by 2^2
constexpr int kOpBytes = kRows * kD * 2;  // one fp16 operand tile: 32 KB

// Shared memory, offsets from a 1024-byte aligned base.
struct ExtPlan {
  static constexpr int kStage = 0;                          // [2][K 16K | V 16K]
  static constexpr int kK16 = kStage + 2 * 2 * kTilePages * kPageBytes;
  static constexpr int kV16 = kK16 + kOpBytes;
  static constexpr int kQ16 = kV16 + kOpBytes;
  static constexpr int kP16 = kQ16 + kOpBytes;
  static constexpr int kStageScl = kP16 + kOpBytes;         // [2][ks 128 | vs 128]
  static constexpr int kScl = kStageScl + 2 * 2 * kKT * 4;  // [4][ks 128 | vs 128]
  // the two softmax halves of a row exchange per-row values here:
  // [2 tile parities][2 halves][128 rows] float2
  static constexpr int kXch = kScl + 4 * 2 * kKT * 4;
  static constexpr int kBar = kXch + 2 * 2 * kRows * 8;
  // st_full[2] st_empty[2] k16_full k16_empty v16_full v16_empty s_full[2]
  // s_empty[2] p_full o_done q_full
  static constexpr int kBarCount = 15;
  static constexpr int kTslot = kBar + kBarCount * 8;
  static constexpr int kBytes = kTslot + 16 + 1024;
};
enum {
  B_ST_FULL = 0, B_ST_EMPTY = 2, B_K16_FULL = 4, B_K16_EMPTY, B_V16_FULL,
  B_V16_EMPTY, B_S_FULL = 8, B_S_EMPTY = 10, B_P_FULL = 12, B_O_DONE,
  B_Q_FULL
};

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo,
                                              uint32_t sbo) {
  // start, leading / stride byte offsets (16-byte units), descriptor
  // version 1, 128-byte swizzle (layout type 2)
  return static_cast<uint64_t>((addr >> 4) & 0x3FFF) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32) |
         (static_cast<uint64_t>(1) << 46) | (static_cast<uint64_t>(2) << 61);
}

// kind::f16 instruction descriptor: fp32 accumulator, fp16 A and B, A
// K-major, B K-major (b_mn = 0) or MN-major (b_mn = 1), M x N.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int b_mn) {
  return (1u << 4) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
      "[%0];" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
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

// Shared-memory loads by 32-bit address; volatile, so a run of them stays
// interleaved with the arithmetic that consumes it (no hoisting of all loads
// ahead, which would need a register each).
__device__ __forceinline__ uint4 lds_u4v(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ float lds_f1v(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// 32 columns into r without waiting (tmem_wait32 makes them readable).
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
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
}
// Wait for this thread's tensor-memory loads; r's registers are operands,
// so no use of them is scheduled before the wait.
__device__ __forceinline__ void tmem_wait32(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]),
        "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]),
        "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
        "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
        "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
        "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
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

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait (about a second); a thread that timed out once stops waiting
// (its results are then meaningless and the sticky status bit says so), so
// the kernel still ends.
constexpr uint64_t kWaitNs = 1000000000ull;
__device__ __forceinline__ void ewait(uint64_t* bar, uint32_t parity,
                                      bool& failed, uint32_t* status) {
  if (failed) return;
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return;
    if (global_ns() - t0 > kWaitNs) break;
  }
  atomicOr(status, KV8_DEV_WAIT_TIMEOUT);
  failed = true;
}

// Byte offset of 16-byte chunk c (8 fp16, 0..15 over 128 elements) of row r
// in a 128 x 128 fp16 operand tile: two 64-element panels of 128 rows x
// 128 bytes, 8-row groups 1024 bytes apart, chunks 128-byte swizzled.
__device__ __forceinline__ uint32_t op_off(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * (kRows * 128) + (r >> 3) * 1024 +
                               (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// 16 int8 codes -> 16 exact fp16 (two 16-byte chunks): c + 128 under the
// fp16 exponent of 1024, minus 1152.
__device__ __forceinline__ void codes16_to_f16(uint4 w, uint4& lo, uint4& hi) {
  const uint32_t x[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u,
                         w.z ^ 0x80808080u, w.w ^ 0x80808080u};
  uint32_t h[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t a, b;
    asm("prmt.b32 %0, %1, %2, 0x4140;" : "=r"(a) : "r"(x[i]), "r"(0x64646464u));
    asm("prmt.b32 %0, %1, %2, 0x4342;" : "=r"(b) : "r"(x[i]), "r"(0x64646464u));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(h[2 * i]) : "r"(a), "r"(0x64806480u));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(h[2 * i + 1]) : "r"(b), "r"(0x64806480u));
  }
  lo = make_uint4(h[0], h[1], h[2], h[3]);
  hi = make_uint4(h[4], h[5], h[6], h[7]);
}

// ---------------------------------------------------------------------------
// Roles shared by the kernels built on this plan.  Each kernel describes its
// items through an item source with
//   int64_t size() const                       items in the launch
//   bool load(int64_t idx, TileItem&, int lane) const
//                                              false: the item is empty;
//                                              warp-collective, and every
//                                              role takes the same decision
// and runs these roles over items blockIdx.x, + gridDim.x, ... in order.
// ---------------------------------------------------------------------------
struct TileItem {
  int64_t tab;  // block_tables offset of the item's first key page
  int kvh;      // KV head
  int npages;   // key pages the item reads
  int nkt;      // key tiles of kKT keys (the last one may be partial)
};

// Warp 0: stream each key tile's pages (K, V codes and their scales) into
// the two-stage ring.
template <class Items>
__device__ __forceinline__ void tc_produce(const Items& items,
                                           const int32_t* block_tables,
                                           int num_kv_heads, const float* k_scales,
                                           const float* v_scales,
                                           const CUtensorMap* tmk,
                                           const CUtensorMap* tmv, uint8_t* smem,
                                           uint64_t* bars, bool& failed,
                                           uint32_t* status, int lane) {
  uint32_t u = 0;  // key tiles issued
  const int64_t n = items.size();
  for (int64_t idx = blockIdx.x; idx < n; idx += gridDim.x) {
    TileItem it;
    if (!items.load(idx, it, lane)) continue;
    for (int j = 0; j < it.nkt; ++j, ++u) {
      const int s = u & 1;
      ewait(&bars[B_ST_EMPTY + s], ((u >> 1) & 1) ^ 1, failed, status);
      const int pg = j * kTilePages + lane;  // lanes 0..7: this tile's pages
      const bool live = lane < kTilePages && pg < it.npages;
      const int blk = live ? block_tables[it.tab + pg] : 0;
      const uint32_t nlive = __popc(__ballot_sync(kFull, live));
      if (lane == 0)
        mbar_arrive_expect_tx(&bars[B_ST_FULL + s],
                              nlive * (2 * kPageBytes + 2 * kBS * 4));
      __syncwarp();
      if (live) {
        uint8_t* st = smem + ExtPlan::kStage + s * 2 * kTilePages * kPageBytes;
        float* sc = reinterpret_cast<float*>(smem + ExtPlan::kStageScl) + s * 2 * kKT;
        const int page = blk * num_kv_heads + it.kvh;
        tma_load_3d(st + lane * kPageBytes, tmk, 0, 0, page, &bars[B_ST_FULL + s]);
        tma_load_3d(st + (kTilePages + lane) * kPageBytes, tmv, 0, 0, page,
                    &bars[B_ST_FULL + s]);
        bulk_g2s(sc + lane * kBS, k_scales + static_cast<int64_t>(page) * kBS,
                 kBS * 4, &bars[B_ST_FULL + s]);
        bulk_g2s(sc + kKT + lane * kBS, v_scales + static_cast<int64_t>(page) * kBS,
                 kBS * 4, &bars[B_ST_FULL + s]);
      }
      __syncwarp();
    }
  }
}

// Warp 1: the MMA issuer (one thread issues): S of tile j+1 is issued before
// O of tile j, so the tensor cores compute the next scores while the
// softmax warps work.  Waits for the softmax's q rows of each item (B_Q_FULL).
template <class Items>
__device__ __forceinline__ void tc_issue(const Items& items, uint8_t* smem,
                                         uint64_t* bars, uint32_t tmem,
                                         bool& failed, uint32_t* status,
                                         int lane) {
  const uint32_t id_qk = idesc_f16(kRows, kKT, 0);
  const uint32_t id_pv = idesc_f16(kRows, kD, 1);
  const uint32_t q16 = smem_u32(smem + ExtPlan::kQ16);
  const uint32_t k16 = smem_u32(smem + ExtPlan::kK16);
  const uint32_t v16 = smem_u32(smem + ExtPlan::kV16);
  const uint32_t p16 = smem_u32(smem + ExtPlan::kP16);
  uint32_t u = 0, nitem = 0;
  auto issue_qk = [&](uint32_t t) {  // S[t & 1] = Q16 K16^T
    ewait(&bars[B_K16_FULL], t & 1, failed, status);
    ewait(&bars[B_S_EMPTY + (t & 1)], ((t >> 1) & 1) ^ 1, failed, status);
    tc_fence_after();
    if (lane == 0) {
      for (int ks = 0; ks < kD / 16; ++ks) {
        const uint32_t off = (ks >> 2) * (kRows * 128) + (ks & 3) * 32;
        mma_f16(tmem + kColS + (t & 1) * kKT, smem_desc(q16 + off, 16, 1024),
                smem_desc(k16 + off, 16, 1024), id_qk, ks > 0);
      }
      mma_commit(&bars[B_K16_EMPTY]);
      mma_commit(&bars[B_S_FULL + (t & 1)]);
    }
    __syncwarp();
  };
  auto issue_pv = [&](uint32_t t, bool first) {  // O += P16 V16
    ewait(&bars[B_P_FULL], t & 1, failed, status);
    ewait(&bars[B_V16_FULL], t & 1, failed, status);
    tc_fence_after();
    if (lane == 0) {
      for (int ks = 0; ks < kKT / 16; ++ks) {
        const uint32_t aoff = (ks >> 2) * (kRows * 128) + (ks & 3) * 32;
        // V16 is MN-major: 16 keys = two 8-key row groups of 1024 bytes; the
        // two 64-dim panels are kRows * 128 bytes apart
        const uint32_t boff = ks * 2048;
        mma_f16(tmem + kColO, smem_desc(p16 + aoff, 16, 1024),
                smem_desc(v16 + boff, kKT * 128, 1024), id_pv,
                (first && ks == 0) ? 0u : 1u);
      }
      mma_commit(&bars[B_V16_EMPTY]);
      mma_commit(&bars[B_O_DONE]);
    }
    __syncwarp();
  };
  const int64_t n = items.size();
  for (int64_t idx = blockIdx.x; idx < n; idx += gridDim.x) {
    TileItem it;
    if (!items.load(idx, it, lane)) continue;
    ewait(&bars[B_Q_FULL], nitem & 1, failed, status);
    ++nitem;
    issue_qk(u);
    for (int j = 0; j < it.nkt; ++j) {
      if (j + 1 < it.nkt) issue_qk(u + j + 1);
      issue_pv(u + j, j == 0);
    }
    u += it.nkt;
  }
}

// Warps 2-3 (ct = 0..63): int8 codes -> fp16 operand tiles (128-byte swizzle)
// in shared memory, the tile's scales set aside in a 4-deep ring.
template <class Items>
__device__ __forceinline__ void tc_convert(const Items& items, uint8_t* smem,
                                           uint64_t* bars, bool& failed,
                                           uint32_t* status, int ct, int lane) {
  uint32_t u = 0;
  const int64_t n = items.size();
  for (int64_t idx = blockIdx.x; idx < n; idx += gridDim.x) {
    TileItem it;
    if (!items.load(idx, it, lane)) continue;
    for (int j = 0; j < it.nkt; ++j, ++u) {
      const int s = u & 1;
      ewait(&bars[B_ST_FULL + s], (u >> 1) & 1, failed, status);
      const uint8_t* st = smem + ExtPlan::kStage + s * 2 * kTilePages * kPageBytes;
      // scales aside (4-deep ring: tile u's are read by the softmax of u)
      {
        const float4* src = reinterpret_cast<const float4*>(
            smem + ExtPlan::kStageScl + s * 2 * kKT * 4);
        float4* dst = reinterpret_cast<float4*>(smem + ExtPlan::kScl +
                                                (u & 3) * 2 * kKT * 4);
        dst[ct] = src[ct];
      }
      // K then V: key t = ct and ct + 64; 8 code chunks of 16 per key
      for (int kv = 0; kv < 2; ++kv) {
        ewait(&bars[kv ? B_V16_EMPTY : B_K16_EMPTY], (u & 1) ^ 1, failed, status);
        uint8_t* dst = smem + (kv ? ExtPlan::kV16 : ExtPlan::kK16);
        const uint8_t* src = st + kv * kTilePages * kPageBytes;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          const int t = ct + 64 * h;
          const uint32_t row =
              smem_u32(src) + (t >> 4) * kPageBytes + (t & 15) * 128;
#pragma unroll
          for (int j8 = 0; j8 < 8; ++j8) {
            const uint4 w = lds_u4v(row + ((j8 ^ (t & 7)) << 4));
            uint4 lo, hi;
            codes16_to_f16(w, lo, hi);
            *reinterpret_cast<uint4*>(dst + op_off(t, 2 * j8)) = lo;
            *reinterpret_cast<uint4*>(dst + op_off(t, 2 * j8 + 1)) = hi;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kv ? B_V16_FULL : B_K16_FULL]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_ST_EMPTY + s]);
    }
  }
}

// The two softmax warps of a lane quarter (qd = 0..3) meet at named
// barrier 1 + qd.
__device__ __forceinline__ void pair_sync(int qd) {
  asm volatile("bar.sync %0, 64;" ::"r"(1 + qd) : "memory");
}

// Exchange one float2 per row with the other half of the row's pair: write
// mine, meet, read the other's.  Consecutive exchanges (counted by xk)
// alternate between two slots, so a fast half cannot overwrite a value the
// slow half has not read yet (that needs it past the next meeting).
__device__ __forceinline__ float2 pair_xch(uint8_t* smem, uint32_t& xk, int hf,
                                           int r, int qd, float2 mine) {
  float2* x =
      reinterpret_cast<float2*>(smem + ExtPlan::kXch) + (xk & 1) * 2 * kRows;
  ++xk;
  x[hf * kRows + r] = mine;
  pair_sync(qd);
  return x[(1 - hf) * kRows + r];
}

// A softmax thread's half (dims 64 hf .. 64 hf + 63) of query row r, staged
// for the q.k product: q (bf16 [128]; read only when live) times an exact
// power of two into fp16 (max |q| 2^sh in [2^14, 2^15), the row's max taken
// over both halves: exact), written to row r of the Q16 operand.  Returns
// the factor that turns an S entry back into a base-2 score.
__device__ __forceinline__ float tc_stage_q(uint8_t* smem, const __nv_bfloat16* qptr,
                                            bool live, int r, int hf, int qd,
                                            float q_scale, uint32_t& xk) {
  uint8_t* q16 = smem + ExtPlan::kQ16;
  const uint4* qsrc = reinterpret_cast<const uint4*>(qptr) + 8 * hf;
  uint4 w[8];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    w[i] = live ? qsrc[i] : make_uint4(0, 0, 0, 0);
    const uint32_t ww[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(ww[k] << 16)),
                               fabsf(__uint_as_float(ww[k] & 0xFFFF0000u))));
  }
  amax = fmaxf(amax, pair_xch(smem, xk, hf, r, qd, make_float2(amax, 0.0f)).x);
  const int sh = amax > 0.0f ? 15 - exp_frexp(amax) : 0;
  const float f1 = pow2i(sh / 2), f2 = pow2i(sh - sh / 2);
  // the previous item's products are done (its o_done was awaited)
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t ww[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
    uint32_t h[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __half2 v = __floats2half2_rn(
          __uint_as_float(ww[k] << 16) * f1 * f2,
          __uint_as_float(ww[k] & 0xFFFF0000u) * f1 * f2);
      h[k] = *reinterpret_cast<const uint32_t*>(&v);
    }
    *reinterpret_cast<uint4*>(q16 + op_off(r, 8 * hf + c)) =
        make_uint4(h[0], h[1], h[2], h[3]);
  }
  return q_scale * pow2i(-(sh / 2)) * pow2i(-(sh - sh / 2));
}

// Running softmax state of one row, base 2: max m, V-scale exponent e (the
// same in both halves of the row) and this half's share of the sum l.
struct RowSoftmax {
  float m, l;
  int e;
};

// A softmax thread's pass over its item's nkt key tiles (tiles u .. u+nkt-1
// of the CTA), for key columns (and output dims) 64 hf .. 64 hf + 63 of row
// r: reads its half of S from tensor memory, masks keys >= key_lim (all keys
// when the row is not live), takes the row's maxima with the other half,
// keeps the lazy online softmax, rescales its half of O in tensor memory
// when the references move, and writes its half of P16 for the O product.
__device__ __forceinline__ RowSoftmax tc_row_tiles(uint8_t* smem, uint64_t* bars,
                                                   uint32_t trow, int r, int hf,
                                                   int qd, int lane, bool live,
                                                   int key_lim, float qf, int nkt,
                                                   uint32_t u, uint32_t& xk,
                                                   bool& failed, uint32_t* status) {
  uint8_t* p16 = smem + ExtPlan::kP16;
  float m_run = -INFINITY, l_run = 0.0f;
  int e_run = -126;
  float vlim = 0.0f, fs = 1.0f;
  const int c0 = kHalf * hf;  // this half's first key column
  for (int j = 0; j < nkt; ++j) {
    const uint32_t t = u + j;
    ewait(&bars[B_S_FULL + (t & 1)], (t >> 1) & 1, failed, status);
    __syncwarp();  // converged for the warp-collective tensor-memory loads
    tc_fence_after();
    // both loads in flight together, then one wait; the registers are
    // reused in place as the half tile's scores
    uint32_t sr[kHalf];
    {
      using Block = uint32_t[32];
      Block* blk = reinterpret_cast<Block*>(sr);
      const uint32_t sa = trow + kColS + (t & 1) * kKT + c0;
      tmem_ld32_async(sa, blk[0]);
      tmem_ld32_async(sa + 32, blk[1]);
      tmem_wait32(blk[0]);
      tmem_wait32(blk[1]);
    }
    float* sv = reinterpret_cast<float*>(sr);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[B_S_EMPTY + (t & 1)]);
    // scores and the half tile's maxima, then the row's with the other half
    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    float vx4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    // the tile's K and V scales (the same for every row): shared-memory
    // loads by 32-bit address
    const uint32_t ks_s =
        smem_u32(smem + ExtPlan::kScl) + (t & 3) * 2 * kKT * 4 + 4 * c0;
    const uint32_t vs_s = ks_s + kKT * 4;
    const int lim = live ? key_lim - j * kKT - c0 : 0;  // columns c < lim visible
    // every row of the warp sees all 64 columns (all but the diagonal and
    // the last tiles): no masking
    const bool all_visible = __all_sync(kFull, lim >= kHalf);
    if (all_visible) {
#pragma unroll
      for (int c = 0; c < kHalf; ++c) {
        sv[c] = sv[c] * qf * lds_f1v(ks_s + 4 * c);
        mx4[c & 3] = fmaxf(mx4[c & 3], sv[c]);
        vx4[c & 3] = fmaxf(vx4[c & 3], lds_f1v(vs_s + 4 * c));
      }
    } else {
#pragma unroll
      for (int c = 0; c < kHalf; ++c) {
        const bool ok = c < lim;
        sv[c] = ok ? sv[c] * qf * lds_f1v(ks_s + 4 * c) : -INFINITY;
        mx4[c & 3] = fmaxf(mx4[c & 3], sv[c]);
        vx4[c & 3] = fmaxf(vx4[c & 3], ok ? lds_f1v(vs_s + 4 * c) : 0.0f);
      }
    }
    float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
    float vx = fmaxf(fmaxf(vx4[0], vx4[1]), fmaxf(vx4[2], vx4[3]));
    {
      const float2 o = pair_xch(smem, xk, hf, r, qd, make_float2(mx, vx));
      mx = fmaxf(mx, o.x);
      vx = fmaxf(vx, o.y);
    }
    // both halves see the same maxima and take the same decisions
    float a_o = 1.0f;
    bool moved = false;
    if (mx > m_run + kSlack || vx > vlim) {
      const float n = fmaxf(m_run, mx);
      const int e_new = vx > vlim ? exp_frexp(vx) : e_run;
      const float a = (n == m_run) ? 1.0f : ex2(m_run - n);
      a_o = a * pow2i(max(e_run - e_new, -126));
      l_run *= a;
      m_run = n;
      e_run = e_new;
      vlim = pow2i(min(e_new + kVSlack, 127));
      fs = pow2i(-e_new);
      moved = true;
    }
    const float mu = m_run == -INFINITY ? 0.0f : m_run;
    // probabilities first (packed fp16 in registers), so that the
    // exponentials overlap the previous O product on the tensor cores
    uint32_t ph[kHalf / 2];
    float ls4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (all_visible) {
#pragma unroll
      for (int c = 0; c < kHalf / 2; ++c) {
        const float p0 = ex2(sv[2 * c] - mu), p1 = ex2(sv[2 * c + 1] - mu);
        ls4[(2 * c) & 3] += p0;
        ls4[(2 * c + 1) & 3] += p1;
        const __half2 hv = __floats2half2_rn(p0 * (lds_f1v(vs_s + 8 * c) * fs),
                                             p1 * (lds_f1v(vs_s + 8 * c + 4) * fs));
        ph[c] = *reinterpret_cast<const uint32_t*>(&hv);
      }
    } else {
#pragma unroll
      for (int c = 0; c < kHalf / 2; ++c) {
        const float p0 = ex2(sv[2 * c] - mu), p1 = ex2(sv[2 * c + 1] - mu);
        ls4[(2 * c) & 3] += p0;
        ls4[(2 * c + 1) & 3] += p1;
        const float v0 = sv[2 * c] == -INFINITY ? 0.0f : lds_f1v(vs_s + 8 * c);
        const float v1 = sv[2 * c + 1] == -INFINITY ? 0.0f : lds_f1v(vs_s + 8 * c + 4);
        const __half2 hv = __floats2half2_rn(p0 * (v0 * fs), p1 * (v1 * fs));
        ph[c] = *reinterpret_cast<const uint32_t*>(&hv);
      }
    }
    const float lsum = (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
    // P16 is free and O is up to date once the previous O product is done
    if (t >= 1) ewait(&bars[B_O_DONE], (t - 1) & 1, failed, status);
    __syncwarp();
    tc_fence_after();
    // rescale this half of O in tensor memory where the row's references
    // moved; the tensor-memory loads and stores are warp-collective, so the
    // whole warp takes the branch (rows that did not move multiply by 1)
    const bool rescale = moved && j > 0;
    if (__any_sync(kFull, rescale)) {
      const float f = rescale ? a_o : 1.0f;
#pragma unroll 1
      for (int c = 0; c < kHalf / 32; ++c) {
        float o[32];
        __syncwarp();
        tmem_ld32(trow + kColO + c0 + 32 * c, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= f;
        tmem_st32(trow + kColO + c0 + 32 * c, o);
      }
    }
#pragma unroll
    for (int c = 0; c < kHalf / 8; ++c)
      *reinterpret_cast<uint4*>(p16 + op_off(r, c0 / 8 + c)) =
          make_uint4(ph[4 * c], ph[4 * c + 1], ph[4 * c + 2], ph[4 * c + 3]);
    l_run += lsum;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[B_P_FULL]);
  }
  return RowSoftmax{m_run, l_run, e_run};
}

// Barriers and tensor memory of a CTA (all threads): returns the base
// tensor-memory address (512 columns, allocated by warp 1).
__device__ __forceinline__ uint32_t tc_setup(uint8_t* smem, const CUtensorMap* tmk,
                                             const CUtensorMap* tmv, int warp) {
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ExtPlan::kBar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + ExtPlan::kTslot);
  if (threadIdx.x == 0) {
    prefetch_tensormap(tmk);
    prefetch_tensormap(tmv);
    const uint32_t counts[ExtPlan::kBarCount] = {1, 1, 2, 2, 2, 1, 2, 1,
                                                 1, 1, 8, 8, 8, 1, 8};
    for (int i = 0; i < ExtPlan::kBarCount; ++i) mbar_init(&bars[i], counts[i]);
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile(
        "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
            smem_u32(tslot)),
        "r"(kTmemCols)
        : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::
                     : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *tslot;
}

// Every role is done issuing; wait for the CTA's tensor-core work and copies
// (all of them were awaited by their consumers) before freeing the columns.
__device__ __forceinline__ void tc_teardown(uint32_t tmem, int warp) {
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
}

}  // namespace
}  // namespace kv8
