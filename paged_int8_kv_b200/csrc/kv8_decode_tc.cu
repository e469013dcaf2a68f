// kv8_decode_tc.cu -- paged INT8 decode attention on the 5th-generation
// tensor cores (tcgen05.mma kind::i8, int32 accumulators in tensor memory).
//
// Computes what decode_kernel in kv8_decode.cu computes
// [KV Cache 优化全景解析——从基础原理到工程实践, §2.1, §3.3, §4.2;
// KV-Cache 全栈优化系统, 主要特性]: per (sequence, KV head, context chunk),
// softmax(q K_hat^T / sqrt(d)) V_hat over the chunk's tokens, with
// K_hat = code * ks and V_hat = code * vs, as split-K partials merged by
// log-sum-exp.  Both products run as exact integer matrix products on
// tcgen05, so no INT8 code is ever converted on the CUDA cores:
//
//   S[128 tok][N]  = Kc[128 tok][128 dim] . Qd^T   K codes as TMA stages
//                                                  them (K-major, 128-B
//                                                  swizzle)
//   O[128 dim][N] += Vc^T[128 dim][128 tok] . Pd^T V codes as TMA stages
//                                                  them, read MN-major
//
// N = 4 digit planes x GP head columns (GP = max(G, 4)).  Qd holds each
// head's q rounded to 30 bits of its largest element and split into four
// balanced int8 digits; Pd holds, per token and head, P'' = 2^(s - m) vs 2^-E
// rounded to 2^-24 and split the same way.  The planes are recombined in
// fp32 when read from tensor memory.
//
// A CTA is persistent over work items (sequence, KV head, chunk) numbered
// chunk-major; a chunk is taken in groups of 8 pages (128 tokens) that cycle
// through NB shared-memory buffers.  Warp roles (8 warps):
//   producer (1)   TMA of each group's K and V pages and both scale rows;
//   q planes (1)   the q digit planes of each item, up to two items ahead
//                  of q.k, from q loaded one item before that;
//   issuer (1)     one thread issues q.k and p.v from a non-blocking event
//                  loop (p.v first); completion is signalled by
//                  tcgen05.commit on mbarriers;
//   softmax (4)    thread t takes token t of a group: reads S from tensor
//                  memory, runs the base-2 online softmax with lazy moves of
//                  the reference max m and of the V-scale exponent E, writes
//                  the P'' planes; drains O (thread t = dim t) into fp32
//                  registers when m or E move, and at the end of the item
//                  after the next item's first group is handed over (O has
//                  two tensor-memory slots, by item parity);
//   epilogue (1)   per split item, the merge ticket and, for the last chunk,
//                  the log-sum-exp merge.
// Roles hand over through mbarriers (and one shared counter for the
// epilogue) only.  Every wait is bounded in time and records a status bit
// on timeout.
#include "kv8_common.cuh"
#include "kv8_internal.h"
#include "kv8_merge.cuh"

namespace kv8 {

__device__ uint32_t g_tc_status = 0;

namespace {

constexpr int kD = kHeadDim;
constexpr int kBS = kBlockSize;
constexpr uint32_t kFull = 0xffffffffu;
constexpr int kGroupPages = 8;               // pages per group
constexpr int kGroupTok = kGroupPages * kBS;  // 128 tokens = MMA M
constexpr int kConsumers = 128;
constexpr int kThreads = kConsumers + 128;  // + producer, issuer, epilogue, q planes
constexpr int kTmemCols = 128;
constexpr float kSlack = 4.0f;   // scores may pass m by 2^4 before m moves
constexpr int kVSlack = 2;       // V scales may pass 2^E by 2^2
constexpr int kPFrac = 24;       // P'' is kept in units of 2^-24
constexpr int kMaxAccGroups = 256;  // int32 headroom of the O accumulator

// Shared memory of one CTA, offsets from a 1024-byte aligned base.
template <int NB, int N>
struct TcPlan {
  static constexpr int kK = 0;                                     // [NB][8][2048]
  static constexpr int kV = kK + NB * kGroupPages * kPageBytes;    // [NB][8][2048]
  static constexpr int kKs = kV + NB * kGroupPages * kPageBytes;   // [NB][128] f32
  static constexpr int kVs = kKs + NB * kGroupTok * 4;             // [NB][128] f32
  static constexpr int kQd = kVs + NB * kGroupTok * 4;             // [2][N x 128 B]
  static constexpr int kPd = kQd + 2 * N * kD;                     // [2][N x 128 B]
  static constexpr int kQf = kPd + 2 * N * kD;                     // [2][8] f32
  static constexpr int kPacc = kQf + 64;                           // [2] u32
  static constexpr int kRed = kPacc + 16;                          // 176 f32
  static constexpr int kBar = kRed + 176 * 4;                      // mbarriers
  static constexpr int kBarCount = 2 * NB + 14;
  static constexpr int kEnd = kBar + kBarCount * 8 + 16;           // + tmem slot
  static constexpr int kBytes = kEnd + 1024;                       // align slack
};

// tcgen05 shared-memory matrix descriptor: start, leading and stride byte
// offsets (16-byte units), descriptor version 1, layout (2 = 128-B swizzle,
// 0 = no swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo,
                                              uint32_t sbo, uint32_t layout) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFF) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32) |
         (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(layout & 7) << 61);
}

// kind::i8 instruction descriptor: s32 accumulator, signed int8 A and B,
// B K-major, A K-major (a_mn = 0) or MN-major (a_mn = 1), M x N.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N, int a_mn) {
  return (2u << 4) | (1u << 7) | (1u << 10) |
         (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a, uint64_t b,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives on `bar` once every tcgen05 operation this thread issued before
// has completed.
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
// Generic-proxy shared-memory writes made visible to the tensor cores.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier 1 over the 4 consumer warps (the producer never joins it).
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
__device__ __forceinline__ bool consumers_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// 16 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,"
      "%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
        "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]),
        "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, uint32_t (&r)[N]) {
  __syncwarp();
  tmem_ld16(taddr, r);
  if constexpr (N == 32) tmem_ld16(taddr + 16, r + 16);
  tmem_wait_ld();
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of `bar` for at most about kWaitNs; on timeout
// raise the sticky status bit and return false.
constexpr uint64_t kWaitNs = 1000000000ull;
__device__ __forceinline__ bool mbar_wait_ns(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitNs) break;
  }
  atomicOr(&g_tc_status, KV8_DEV_WAIT_TIMEOUT);
  return false;
}

// Bounded wait.  A thread that has timed out once stops waiting (its results
// are then meaningless, and the sticky status bit says so), so the kernel
// still ends within a few seconds.
__device__ __forceinline__ void wait_or_fail(uint64_t* bar, uint32_t parity,
                                             bool& failed) {
  if (failed) return;
  if (!mbar_wait_ns(bar, parity)) failed = true;
}

// Byte offset of (row n, k) in a K-major operand tile without swizzle of
// N rows x 128 k-bytes: 8-row x 16-byte core matrices; row groups of 8 are
// 128 bytes apart, 16-byte k-chunks N/8 * 128 bytes apart.
template <int N>
__device__ __forceinline__ int kmaj_off(int n, int k) {
  return ((k >> 4) * (N >> 3) + (n >> 3)) * 128 + (n & 7) * 16 + (k & 15);
}

// 2^e as two factors, each a normal float, for |e| <= 250.
__device__ __forceinline__ float2 pow2pair(int e) {
  const int e1 = e / 2, e2 = e - e1;
  return make_float2(pow2i(e1), pow2i(e2));
}

// Balanced base-256 digits of v, |v| <= 2^30:
// v = 2^24 d3 + 2^16 d2 + 2^8 d1 + d0, d0..d2 in [-128, 127].
__device__ __forceinline__ void digits4(int v, int (&d)[4]) {
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    d[i] = static_cast<int>(static_cast<int8_t>(v & 0xFF));
    v = (v - d[i]) >> 8;
  }
  d[3] = v;
}

// sum_pl 2^(8 pl) C_pl of the four int32 plane sums of head column h.
template <int GP>
__device__ __forceinline__ float planes_to_f32(const uint32_t* c, int h) {
  const int hi = static_cast<int>(c[3 * GP + h]) * 256 + static_cast<int>(c[2 * GP + h]);
  const int lo = static_cast<int>(c[GP + h]) * 256 + static_cast<int>(c[h]);
  return __int2float_rn(hi) * 65536.0f + __int2float_rn(lo);
}

struct TcItem {
  int b, kvh, chunk, n, tok0, tok1, npages, nchunks;
};

// Walks this CTA's items, item i = (chunk * H_kv + kvh) * B + b for
// i = blockIdx.x + k * gridDim.x, by mixed-radix addition of the stride (no
// division per item), with the context length of the next candidate loaded
// one item ahead so that moving on does not wait on global memory.  Items
// whose chunk starts past the context are skipped; an empty context keeps
// chunk 0, which writes zeros.
struct TcCursor {
  TcItem it;                 // current item; it.chunk >= max_chunks when done
  int nb, nkvh, nchunk, nn;  // next candidate and its context length
  int sb, skh, sc;           // gridDim.x as (chunk, kvh, b) digits
  const DecodeParams* p;

  __device__ __forceinline__ void step(int& c, int& h, int& b) const {
    b += sb;
    h += skh;
    c += sc;
    if (b >= p->batch) {
      b -= p->batch;
      ++h;
    }
    if (h >= p->num_kv_heads) {
      h -= p->num_kv_heads;
      ++c;
    }
  }
  __device__ __forceinline__ bool make(int c, int h, int b, int n) {
    it.chunk = c;
    it.kvh = h;
    it.b = b;
    it.n = n;
    it.tok0 = c * p->chunk_tokens;
    if (it.tok0 >= n && !(n == 0 && c == 0)) return false;
    it.tok1 = min(n, it.tok0 + p->chunk_tokens);
    it.npages = (it.tok1 - it.tok0 + kBS - 1) / kBS;
    it.nchunks = (n + p->chunk_tokens - 1) / p->chunk_tokens;
    return true;
  }
  __device__ __forceinline__ void prefetch() {
    nchunk = it.chunk;
    nkvh = it.kvh;
    nb = it.b;
    step(nchunk, nkvh, nb);
    if (nchunk < p->max_chunks) nn = __ldg(&p->context_lens[nb]);
  }
  __device__ __forceinline__ void seek(int c, int h, int b, int n) {
    while (c < p->max_chunks && !make(c, h, b, n)) {
      step(c, h, b);
      if (c < p->max_chunks) n = __ldg(&p->context_lens[b]);
    }
    it.chunk = c;
    it.kvh = h;
    it.b = b;
    if (c < p->max_chunks) prefetch();
  }
  __device__ __forceinline__ void start(const DecodeParams& params) {
    p = &params;
    const int64_t bh = static_cast<int64_t>(p->batch) * p->num_kv_heads;
    const int64_t g = gridDim.x, i = blockIdx.x;
    sb = static_cast<int>(g % p->batch);
    skh = static_cast<int>((g / p->batch) % p->num_kv_heads);
    sc = static_cast<int>(g / bh);
    const int b = static_cast<int>(i % p->batch);
    const int h = static_cast<int>((i / p->batch) % p->num_kv_heads);
    const int c = static_cast<int>(i / bh);
    seek(c, h, b, c < p->max_chunks ? __ldg(&p->context_lens[b]) : 0);
  }
  __device__ __forceinline__ bool valid() const { return it.chunk < p->max_chunks; }
  __device__ __forceinline__ void next() { seek(nchunk, nkvh, nb, nn); }
};

// Maximum of v over the full warp (one warp-wide reduction instruction).
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Waits for phase `parity` of `bar` for about `ns` nanoseconds at most (the
// thread is suspended meanwhile); true once the phase has completed.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity,
                                                   uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Non-blocking probe of phase `parity` of `bar`.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Count of softmax warps that have written an item's partials: each warp
// adds 1 with release semantics; the epilogue warp reads it with acquire.
__device__ __forceinline__ void done_add(uint32_t* ctr) {
  asm volatile("red.release.cta.shared::cta.add.u32 [%0], 1;" ::"r"(smem_u32(ctr))
               : "memory");
}
__device__ __forceinline__ uint32_t done_get(const uint32_t* ctr) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];"
               : "=r"(v)
               : "r"(smem_u32(ctr))
               : "memory");
  return v;
}

// Lane 0 of each consumer warp arrives once the whole warp is done (the
// consumer-side barriers count 4 arrivals).
__device__ __forceinline__ void warp_arrive(uint64_t* bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

template <int G, int NB>
__global__ void __launch_bounds__(kThreads, 2)
decode_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                 const __grid_constant__ CUtensorMap tmv) {
  constexpr int GP = G < 4 ? 4 : G;  // head columns per digit plane
  constexpr int N = 4 * GP;          // 16 or 32
  static_assert(N == 16 || N == 32, "digit-plane layout");
  constexpr uint32_t kIdS = idesc_i8(128, N, 0);
  constexpr uint32_t kIdO = idesc_i8(128, N, 1);
  constexpr uint32_t kLbo = (N / 8) * 128;  // B operand: k-chunk stride
  using Plan = TcPlan<NB, N>;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kbuf = smem + Plan::kK;
  uint8_t* vbuf = smem + Plan::kV;
  float* ksb = reinterpret_cast<float*>(smem + Plan::kKs);
  float* vsb = reinterpret_cast<float*>(smem + Plan::kVs);
  uint8_t* qd = smem + Plan::kQd;  // [2][N x 128]
  uint8_t* pd = smem + Plan::kPd;  // [2][N x 128]
  float* qfs = reinterpret_cast<float*>(smem + Plan::kQf);     // [2][8]
  uint32_t* pacc = reinterpret_cast<uint32_t*>(smem + Plan::kPacc);  // [2]
  float* red = reinterpret_cast<float*>(smem + Plan::kRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Plan::kBar);
  uint64_t* full = bars;                 // [NB] producer -> TMA bytes landed
  uint64_t* empty = bars + NB;           // [NB] p.v done: buffer free
  uint64_t* sfull = bars + 2 * NB;       // [2] q.k done: S slot readable
  uint64_t* sempty = bars + 2 * NB + 2;  // [2] consumers read S slot
  uint64_t* pfull = bars + 2 * NB + 4;   // [2] consumers wrote Pd slot
  uint64_t* pempty = bars + 2 * NB + 6;  // [2] p.v done: Pd slot free, O final
  uint64_t* qready = bars + 2 * NB + 8;  // [2] issuer wrote Qd / qf slot
  uint64_t* qfree = bars + 2 * NB + 10;  // [2] consumers read qf slot
  uint64_t* qempty = bars + 2 * NB + 12; // [2] last q.k of the item done
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + Plan::kBarCount);
  __shared__ uint32_t s_done;  // softmax-warp completions of split items

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    // arrivals per phase: 1 (TMA expect_tx or tcgen05.commit), 4 (one per
    // softmax warp) or 32 (every issuer lane)
    constexpr uint8_t kCount[7] = {1, 4, 4, 1, 32, 4, 1};
    for (int i = 0; i < Plan::kBarCount; ++i)
      mbar_init(&bars[i], i < 2 * NB ? 1u : kCount[(i - 2 * NB) >> 1]);
    fence_mbar_init();
    s_done = 0;
  }
  if (warp == 0) {
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
  const uint32_t tmem = *tslot;
  // tensor memory: S slots at columns [0, N) and [N, 2N); O slots (by item
  // parity) at [2N, 3N) and [3N, 4N)

  TcCursor cur;
  cur.start(p);

  bool failed = false;
  uint32_t ngrp = 0;  // groups of this CTA so far (same count in every role)

  if (warp == 4) {
    // ======================================================= producer
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
    for (; cur.valid(); cur.next()) {
      const TcItem& it = cur.it;
      const int32_t* bt = p.block_tables +
                          static_cast<int64_t>(it.b) * p.max_blocks_per_seq +
                          it.tok0 / kBS;
      for (int g0 = 0; g0 < it.npages; g0 += kGroupPages, ++ngrp) {
        const int np = min(kGroupPages, it.npages - g0);
        const int b = static_cast<int>(ngrp % NB);
        const uint32_t use = ngrp / NB;
        int blk = 0;
        if (lane < np) blk = __ldg(&bt[g0 + lane]);
        if (use > 0) wait_or_fail(&empty[b], (use - 1) & 1, failed);
        __syncwarp();
        if (lane == 0)
          mbar_arrive_expect_tx(&full[b], np * (2 * kPageBytes + 2 * kBS * 4));
        __syncwarp();
        if (lane < np) {
          const int page = blk * p.num_kv_heads + it.kvh;
          const int slot = b * kGroupPages + lane;
          tma_load_3d(kbuf + slot * kPageBytes, &tmk, 0, 0, page, &full[b]);
          tma_load_3d(vbuf + slot * kPageBytes, &tmv, 0, 0, page, &full[b]);
          bulk_g2s(ksb + slot * kBS, p.k_scales + static_cast<int64_t>(page) * kBS,
                   kBS * 4, &full[b]);
          bulk_g2s(vsb + slot * kBS, p.v_scales + static_cast<int64_t>(page) * kBS,
                   kBS * 4, &full[b]);
        }
      }
    }
    // no copy may still be landing when the CTA exits
    for (uint32_t k = ngrp > NB ? ngrp - NB : 0; k < ngrp; ++k)
      mbar_wait_ns(&full[k % NB], (k / NB) & 1);
  } else if (warp == 5) {
    // ======================================================= MMA issuer
    uint32_t obits = 0;  // O slot (item parity) of group g at bit g % 32
    auto issue_pv = [&](uint32_t g) {  // pfull of g observed
      const int s = g & 1;
      const uint32_t tO = tmem + (2 + ((obits >> (g & 31)) & 1u)) * N;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t acc = pacc[s];
        const uint32_t a0 = smem_u32(vbuf + (g % NB) * kGroupPages * kPageBytes);
        const uint32_t b0 = smem_u32(pd + s * N * kD);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_i8(tO, smem_desc(a0 + 4096 * k, 16, 1024, 2),
                 smem_desc(b0 + k * 2 * kLbo, kLbo, 128, 0), kIdO,
                 (k > 0 || acc) ? 1u : 0u);
        mma_commit(&pempty[s]);
        mma_commit(&empty[g % NB]);
      }
      __syncwarp();
    };
    // Event loop over two kinds of work, p.v first: p.v of the oldest group
    // whose P'' planes are written, then q.k of the next group whose pages
    // have landed (S slot free, q planes built).  Nothing here blocks; an
    // idle spell longer than the wait limit ends the loop with the timeout
    // bit set.
    while (cur.valid() && cur.it.npages == 0) cur.next();
    int qk_groups = cur.valid() ? (cur.it.npages + kGroupPages - 1) / kGroupPages : 0;
    int qk_j = 0;          // next group within the q.k item
    uint32_t nitem = 0;    // index of the q.k item among items with groups
    uint32_t gv = 0;       // next group for p.v (ngrp counts q.k issued)
    uint64_t t_idle = 0;
    uint32_t spins = 0;
    for (;;) {
      const bool qk_left = cur.valid();
      if (!qk_left && gv == ngrp) break;
      bool ready = false;
      if (gv < ngrp) {
        if (lane == 0) ready = mbar_test_wait(&pfull[gv & 1], (gv >> 1) & 1);
        if (__shfl_sync(kFull, ready ? 1 : 0, 0)) {
          issue_pv(gv);
          ++gv;
          spins = 0;
          continue;
        }
      }
      if (qk_left) {
        const int s = ngrp & 1;
        if (lane == 0)
          ready = mbar_test_wait(&qready[nitem & 1], (nitem >> 1) & 1) &&
                  mbar_test_wait(&full[ngrp % NB], (ngrp / NB) & 1) &&
                  (ngrp < 2 || mbar_test_wait(&sempty[s], ((ngrp >> 1) - 1) & 1));
        if (__shfl_sync(kFull, ready ? 1 : 0, 0)) {
          tc_fence_after();
          const int qs = nitem & 1;
          if (lane == 0) {
            const uint32_t a0 = smem_u32(kbuf + (ngrp % NB) * kGroupPages * kPageBytes);
            const uint32_t b0 = smem_u32(qd + qs * N * kD);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_i8(tmem + s * N, smem_desc(a0 + 32 * k, 16, 1024, 2),
                     smem_desc(b0 + k * 2 * kLbo, kLbo, 128, 0), kIdS, k > 0);
            mma_commit(&sfull[s]);
            if (qk_j == qk_groups - 1) mma_commit(&qempty[qs]);
          }
          __syncwarp();
          obits = (obits & ~(1u << (ngrp & 31))) | ((nitem & 1u) << (ngrp & 31));
          ++ngrp;
          if (++qk_j == qk_groups) {
            qk_j = 0;
            ++nitem;
            do {
              cur.next();
            } while (cur.valid() && cur.it.npages == 0);
            qk_groups = cur.valid() ? (cur.it.npages + kGroupPages - 1) / kGroupPages : 0;
          }
          spins = 0;
          continue;
        }
      }
      // idle: sleep briefly on the barrier most likely to complete next
      if (lane == 0) {
        if (gv < ngrp)
          mbar_try_wait_hint(&pfull[gv & 1], (gv >> 1) & 1, 256);
        else if (qk_left)
          mbar_try_wait_hint(&full[ngrp % NB], (ngrp / NB) & 1, 256);
      }
      __syncwarp();
      if (spins == 0) t_idle = global_ns();
      if ((++spins & 15) == 0 && global_ns() - t_idle > kWaitNs) {
        if (lane == 0) atomicOr(&g_tc_status, KV8_DEV_WAIT_TIMEOUT);
        break;
      }
    }
    if (ngrp >= 1) {
      // every MMA has completed before tensor memory is released
      mbar_wait_ns(&pempty[(ngrp - 1) & 1], ((ngrp - 1) >> 1) & 1);
    }
  } else if (warp == 7) {
    // ===================================================== q planes
    // Builds the q digit planes of each item with groups, up to two items
    // ahead of q.k, from q loaded one item before that.
    // lane l holds dims 4l..4l+3 of each head
    auto load_q = [&](const TcItem& it, float (&qv)[GP][4]) {
      const int64_t row0 = static_cast<int64_t>(it.b) * p.num_q_heads + it.kvh * G;
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        uint2 w = make_uint2(0u, 0u);
        if (h < G)
          w = __ldg(reinterpret_cast<const uint2*>(p.q + (row0 + h) * kD) + lane);
        qv[h][0] = __uint_as_float(w.x << 16);
        qv[h][1] = __uint_as_float(w.x & 0xFFFF0000u);
        qv[h][2] = __uint_as_float(w.y << 16);
        qv[h][3] = __uint_as_float(w.y & 0xFFFF0000u);
      }
    };
    TcCursor& qcur = cur;
    while (qcur.valid() && qcur.it.npages == 0) qcur.next();
    float qn[GP][4];
    if (qcur.valid()) load_q(qcur.it, qn);
    uint32_t nq = 0;  // items whose planes are built
    auto build_q = [&]() {  // its slot observed free
      const int qs = nq & 1;
      // Q = rint(q 2^sh) with max |Q| in [2^29, 2^30)
      uint8_t* qdst = qd + qs * N * kD;
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        const float a = warp_max(fmaxf(fmaxf(fabsf(qn[h][0]), fabsf(qn[h][1])),
                                       fmaxf(fabsf(qn[h][2]), fabsf(qn[h][3]))));
        const int sh = a > 0.0f ? 30 - exp_frexp(a) : 0;
        const float2 f = pow2pair(sh);
        uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          int d[4];
          digits4(__float2int_rn(qn[h][i] * f.x * f.y), d);
#pragma unroll
          for (int pl = 0; pl < 4; ++pl)
            w[pl] |= (static_cast<uint32_t>(d[pl]) & 0xFFu) << (8 * i);
        }
#pragma unroll
        for (int pl = 0; pl < 4; ++pl)
          *reinterpret_cast<uint32_t*>(qdst + kmaj_off<N>(pl * GP + h, 4 * lane)) = w[pl];
        if (lane == 0) {
          const float2 g2 = pow2pair(-sh);
          qfs[qs * 8 + h] = p.q_scale * g2.x * g2.y;
        }
      }
      fence_async_smem();
      mbar_arrive(&qready[qs]);
      __syncwarp();
      ++nq;
      do {
        qcur.next();
      } while (qcur.valid() && qcur.it.npages == 0);
      if (qcur.valid()) load_q(qcur.it, qn);
    };
    while (qcur.valid()) {
      const int qs = nq & 1;
      if (nq >= 2) {  // slot free: its item has read qf and finished its q.k
        wait_or_fail(&qfree[qs], ((nq >> 1) - 1) & 1, failed);
        wait_or_fail(&qempty[qs], ((nq >> 1) - 1) & 1, failed);
      }
      build_q();
    }
  } else if (warp == 6) {
    // ===================================================== epilogue
    // Per split item, once the four softmax warps have written its partials:
    // take the (sequence, KV group) ticket; the last of its chunks merges
    // the G heads.  The softmax warps never wait for this warp.
    uint32_t nsplit = 0;
    for (; cur.valid(); cur.next()) {
      const TcItem& it = cur.it;
      if (it.nchunks <= 1) continue;
      ++nsplit;
      if (!failed) {
        const uint64_t t0 = global_ns();
        while (done_get(&s_done) < 4 * nsplit) {
          __nanosleep(64);
          if (global_ns() - t0 > kWaitNs) {
            if (lane == 0) atomicOr(&g_tc_status, KV8_DEV_WAIT_TIMEOUT);
            failed = true;
            break;
          }
        }
      }
      const int64_t row0 = static_cast<int64_t>(it.b) * p.num_q_heads + it.kvh * G;
      uint32_t ticket = 0;
      if (lane == 0) {
        __threadfence();
        ticket = atomicAdd(&p.ws_ctr[row0], 1u);
      }
      ticket = __shfl_sync(kFull, ticket, 0);
      if (ticket == static_cast<uint32_t>(it.nchunks - 1)) {
        __threadfence();
        for (int h = 0; h < G; ++h)
          merge_head_warp(p.ws_ml + (row0 + h) * p.max_chunks * 2,
                          p.ws_o + (row0 + h) * p.max_chunks * kD, it.nchunks,
                          p.out, row0 + h, p.out_f32);
      }
    }
  } else {
    // ===================================================== consumers
    const int t = tid;  // token of a group in the softmax, dim in the output
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    uint32_t nitem = 0, nout = 0;
    // The previous item's O (tensor-memory slot by item parity) is drained
    // and its output written only after this item's first group has been
    // handed to the tensor cores, so its last p.v is never waited for.
    // (m and l of the pending item, the same in every thread, stay in the
    // shared l-sum area of its parity: l at [0, 32), m at [32, 40))
    bool pn_on = false, pn_drain = false, pn_single = false;
    int64_t pn_row0 = 0;
    int pn_chunk = 0, pn_e = 0;
    uint32_t pn_g = 0, pn_slot = 0;
    const float* pn_red = red;
    float pn_o[GP];
    auto drain_into = [&](uint32_t oslot, uint32_t glast, float (&acc)[GP]) {
      // O (int32 planes) of the p.v up to group glast, added into acc
      wait_or_fail(&pempty[glast & 1], (glast >> 1) & 1, failed);
      tc_fence_after();
      uint32_t orr[N];
      tmem_ld_row(tmem + (2 + oslot) * N + lane_base, orr);
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        const float v =
            (__int2float_rn(static_cast<int>(orr[3 * GP + h])) * 256.0f +
             __int2float_rn(static_cast<int>(orr[2 * GP + h]))) * 65536.0f +
            (__int2float_rn(static_cast<int>(orr[GP + h])) * 256.0f +
             __int2float_rn(static_cast<int>(orr[h])));
        acc[h] += v;
      }
    };
    auto finish_pending = [&]() {
      if (!pn_on) return;
      if (pn_drain) drain_into(pn_slot, pn_g, pn_o);
      const float2 os = pow2pair(pn_e - kPFrac);  // O = acc 2^(E - 24)
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float o = pn_o[h] * os.x * os.y;
        const float L = (pn_red[h] + pn_red[8 + h]) + (pn_red[16 + h] + pn_red[24 + h]);
        if (pn_single) {
          store_out(p.out, (pn_row0 + h) * kD + t, L > 0.0f ? o / L : 0.0f, p.out_f32);
        } else {
          const int64_t ci = (pn_row0 + h) * p.max_chunks + pn_chunk;
          p.ws_o[ci * kD + t] = o;
          if (t == 0) {
            p.ws_ml[2 * ci] = pn_red[32 + h];
            p.ws_ml[2 * ci + 1] = L;
          }
        }
      }
      if (!pn_single) {  // partials written: hand the item to the epilogue warp
        __syncwarp();
        if (lane == 0) done_add(&s_done);
      }
      pn_on = false;
    };
    for (; cur.valid(); cur.next()) {
      const TcItem it = cur.it;
      const int64_t row0 = static_cast<int64_t>(it.b) * p.num_q_heads + it.kvh * G;
      const int ngroups = (it.npages + kGroupPages - 1) / kGroupPages;
      const uint32_t oslot = nitem & 1;
      float qf[GP];
      if (ngroups > 0) {
        const int qs = nitem & 1;
        wait_or_fail(&qready[qs], (nitem >> 1) & 1, failed);
#pragma unroll
        for (int h = 0; h < GP; ++h) qf[h] = qfs[qs * 8 + h];
        warp_arrive(&qfree[qs], lane);
        ++nitem;
      }
      float m_ref[GP], l_part[GP], o_acc[GP];
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        m_ref[h] = -INFINITY;
        l_part[h] = 0.0f;
        o_acc[h] = 0.0f;
      }
      int e_run = -126;
      float vlim = 0.0f;
      bool o_fresh = true;  // next p.v overwrites O
      int o_groups = 0;     // groups accumulated in O since the last drain

      for (int g = 0; g < ngroups; ++g, ++ngrp) {
        const int s = ngrp & 1;
        const int cb = static_cast<int>(ngrp % NB);
        const int nv = it.tok1 - (it.tok0 + g * kGroupTok);  // valid tokens
        // ---- scores of this group
        wait_or_fail(&sfull[s], (ngrp >> 1) & 1, failed);
        wait_or_fail(&full[cb], (ngrp / NB) & 1, failed);
        tc_fence_after();
        uint32_t sr[N];
        tmem_ld_row(tmem + s * N + lane_base, sr);
        tc_fence_before();
        warp_arrive(&sempty[s], lane);
        const bool valid = t < nv;
        const float ks = ksb[cb * kGroupTok + t];
        const float vs = valid ? vsb[cb * kGroupTok + t] : 0.0f;
        float sc[GP];
#pragma unroll
        for (int h = 0; h < GP; ++h)
          sc[h] = (valid && h < G) ? planes_to_f32<GP>(sr, h) * qf[h] * ks : -INFINITY;
        // ---- lazy move of m and E, decided for the whole CTA
        bool mv = vs > vlim || o_groups >= kMaxAccGroups;
#pragma unroll
        for (int h = 0; h < GP; ++h) mv = mv || sc[h] > m_ref[h] + kSlack;
        if (consumers_any(mv)) {
#pragma unroll
          for (int h = 0; h < GP; ++h) {
            const float x = warp_max(sc[h]);
            if (lane == 0) red[32 + warp * 8 + h] = x;
          }
          float vx = warp_max(vs);
          if (lane == 0) red[64 + warp] = vx;
          if (!o_fresh) {  // O so far into o_acc at the old references
            drain_into(oslot, ngrp - 1, o_acc);
            o_fresh = true;
            o_groups = 0;
          }
          consumers_sync();
          vx = fmaxf(fmaxf(red[64], red[65]), fmaxf(red[66], red[67]));
          const int e_new = vx > vlim ? exp_frexp(vx) : e_run;  // vs < 2^E
          const float2 ef = pow2pair(e_run - e_new);
#pragma unroll
          for (int h = 0; h < GP; ++h) {
            const float x = fmaxf(fmaxf(red[32 + h], red[40 + h]), fmaxf(red[48 + h], red[56 + h]));
            const float nm = fmaxf(m_ref[h], x);
            const float alpha = (nm == m_ref[h]) ? 1.0f : ex2(m_ref[h] - nm);
            m_ref[h] = nm;
            l_part[h] *= alpha;
            o_acc[h] *= alpha * ef.x * ef.y;
          }
          e_run = e_new;
          vlim = e_new + kVSlack >= 128 ? INFINITY : pow2i(e_new + kVSlack);
        }
        // ---- probabilities and the P'' digit planes
        const float2 fe = pow2pair(kPFrac - e_run);
        const float vn = vs * fe.x * fe.y;  // vs 2^(24 - E) <= 2^26
        if (ngrp >= 2) wait_or_fail(&pempty[s], ((ngrp >> 1) - 1) & 1, failed);
        uint8_t* pds = pd + s * N * kD;
#pragma unroll
        for (int h = 0; h < GP; ++h) {
          const float pr = ex2(sc[h] - (m_ref[h] == -INFINITY ? 0.0f : m_ref[h]));
          l_part[h] += pr;
          int d[4];
          digits4(__float2int_rn(pr * vn), d);
#pragma unroll
          for (int pl = 0; pl < 4; ++pl)
            pds[kmaj_off<N>(pl * GP + h, t)] = static_cast<uint8_t>(d[pl]);
        }
        if (t == 0) pacc[s] = o_fresh ? 0u : 1u;
        fence_async_smem();
        tc_fence_before();
        warp_arrive(&pfull[s], lane);
        o_fresh = false;
        ++o_groups;
        if (g == 0) finish_pending();
      }
      // ---- end of the chunk: sum l over tokens; O and the output follow
      // the next item's first group
      float* lred = red + 96 + (nout & 1) * 40;  // alternating l-sum areas
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        float x = l_part[h];
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(kFull, x, m);
        if (lane == 0) lred[warp * 8 + h] = x;
        if (t == 0) lred[32 + h] = m_ref[h];
      }
      consumers_sync();  // l sums visible
      ++nout;
      finish_pending();  // an item without groups leaves one behind
      pn_on = true;
      pn_drain = !o_fresh;
      pn_single = it.nchunks <= 1;
      pn_row0 = row0;
      pn_chunk = it.chunk;
      pn_e = e_run;
      pn_g = ngrp - 1;
      pn_slot = oslot;
      pn_red = lred;
#pragma unroll
      for (int h = 0; h < GP; ++h) pn_o[h] = o_acc[h];
    }
    finish_pending();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
}

template <int G, int NB>
int launch_tc(const DecodeParams& p, const CUtensorMap& tmk,
              const CUtensorMap& tmv, cudaStream_t stream) {
  auto kern = decode_tc_kernel<G, NB>;
  constexpr int smem = TcPlan<NB, 4 * (G < 4 ? 4 : G)>::kBytes;
  static LaunchFacts table[kMaxDevices];  // per device, this instantiation
  LaunchFacts* f = facts_for_current_device(table);
  if (!f) return -1;
  int resident = f->resident.load(std::memory_order_acquire);
  int sms = f->sms.load(std::memory_order_acquire);
  if (resident == 0 || sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return -1;
    // all of the unified L1 / shared storage as shared memory, so that the
    // occupancy computed below is what the launch gets
    if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return -1;
    int nsm = 0;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) !=
        cudaSuccess)
      return -1;
    sms = nsm;
    resident = resident_ctas(kern, kThreads, smem, kTmemCols);
    if (resident == 0) return -1;
    f->sms.store(sms, std::memory_order_release);
    f->resident.store(resident, std::memory_order_release);
  }
  const int64_t n_items =
      static_cast<int64_t>(p.max_chunks) * p.num_kv_heads * p.batch;
  int64_t ctas = static_cast<int64_t>(sms) * resident;
  if (ctas > n_items) ctas = n_items;
  if (ctas < 1) ctas = 1;
  kern<<<static_cast<unsigned>(ctas), kThreads, smem, stream>>>(p, tmk, tmv);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

int launch_decode_tc(const DecodeParams& p, const CUtensorMap& tmk,
                     const CUtensorMap& tmv, cudaStream_t stream) {
  switch (p.num_q_heads / p.num_kv_heads) {
    case 1: return launch_tc<1, 3>(p, tmk, tmv, stream);
    case 2: return launch_tc<2, 3>(p, tmk, tmv, stream);
    case 4: return launch_tc<4, 3>(p, tmk, tmv, stream);
    case 8: return launch_tc<8, 2>(p, tmk, tmv, stream);
    default: return -2;
  }
}

int read_tc_status(uint32_t* value, int clear) {
  if (cudaMemcpyFromSymbol(value, g_tc_status, sizeof(uint32_t)) != cudaSuccess)
    return -1;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_tc_status, &zero, sizeof(uint32_t)) != cudaSuccess)
      return -1;
  }
  return 0;
}

}  // namespace kv8
