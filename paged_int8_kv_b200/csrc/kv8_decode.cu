// kv8_decode.cu -- split-K paged INT8 decode attention and the split reduce.
//
// What is computed [KV Cache 优化全景解析——从基础原理到工程实践, §2.1 and
// §3.3; KV-Cache 全栈优化系统, 主要特性]: for one new query token per
// sequence, every query head h of KV group kvh = h / G attends over the
// sequence's cached tokens, each dequantised on the fly (k_hat = code * ks,
// v_hat = code * vs), out = softmax(q k_hat^T / sqrt(d)) v_hat, with fp32
// accumulation [大模型推理加速：KV Cache与vLLM技术解析, §4.1].
//
// Work decomposition (persistent CTAs of independent warps; one work item =
// one (sequence, KV head, context chunk), handled by one warp):
//   * A warp owns SPW shared-memory slots and streams its items' 16-token
//     pages through them: lane 0 resolves each page through the block table
//     [KV Cache 优化全景解析, §4.2] and issues two TMA tensor copies (the K
//     page and the V page, 128-byte swizzled so that the reads below are
//     bank-conflict free) plus two 64-byte bulk copies (the K and V scales)
//     that complete on the slot's mbarrier.  There is no producer warp and
//     no cross-warp handshake on the ring: the warp that consumes a slot
//     refills it.  Items come from a work counter, numbered chunk-major with
//     the KV head fastest.
//   * All G query heads of the KV group are computed together, so each K/V
//     byte is read from HBM once per step (the INT4 cache's groups of 8 run
//     as two sub-groups of 4 whose second read of a page comes from L2).
//   * Per page, the page math (kv8_page_math.cuh) scores the G heads against
//     the 16 tokens, folds the token's K scale into the score, keeps a base-2
//     online softmax (running max m and sum l per head), folds the token's V
//     scale into the probability and accumulates o += p * v_code; the
//     automatic form does both products on int8 tensor-core mma.
//   * At the end of its chunk the warp writes the result: the normalised
//     output for a sequence that fits one chunk, else the chunk's (m, l, o)
//     partial; the last chunk of each (sequence, KV group) to finish (a
//     ticket, never a wait) merges the partials by log-sum-exp.
//   * Fused append (kv8_paged_decode_attention_append): the warp that takes a
//     sequence's last chunk first quantises the step's new token into the
//     cache, then copies the page that holds it.
#include "../../include/kv8.h"
#include "kv8_common.cuh"
#include "kv8_internal.h"
#include "kv8_merge.cuh"
#include "kv8_page_math.cuh"

namespace kv8 {

__device__ uint32_t g_device_status = 0;

#ifdef KV8_TEST_HOOKS
// Test-hook build only: when set, warp 0 of CTA 0 arms the mbarrier of its
// first page (expect-tx) but issues none of that page's copies, so its wait
// for that page runs out; nothing is copied, nothing faults.
__device__ int g_test_skip_first_copy = 0;
#endif

namespace {

// --------------------------------------------------------------------------
// Shared-memory plan of a decode CTA of WPC independent warps (base aligned
// to 1024 bytes):
//   per warp w: SPW slots of [K page | V page]   (tiles; CodeBytes each:
//               2048 for INT8 codes, 1024 for packed INT4 codes)
//   per warp w: SPW slots of [ks 64 B | vs 64 B]              (scales)
//   per warp w: the page math's scratch (ScratchBytes, may be 0)
//   per warp w: SPW mbarriers, then its work queue (kQueue item indices)
// --------------------------------------------------------------------------
constexpr int kQueue = 16;  // > SPW + 1: queued items each hold an issued page
template <int WPC, int SPW, int ScratchBytes = 0, int CodeBytes = kPageBytes>
struct SmemPlan {
  static constexpr int kTileBytes = WPC * SPW * 2 * CodeBytes;
  static constexpr int kScaleBytes = WPC * SPW * 2 * kBS * 4;
  static constexpr int kScratchBytes = WPC * ScratchBytes;
  static_assert(SPW + 1 <= kQueue, "work queue too short for the page ring");
  static constexpr int kBarBytes = WPC * (SPW * 8 + kQueue * 4);
  static constexpr int kBytes =
      kTileBytes + kScaleBytes + kScratchBytes + kBarBytes + 16 + 1024;
};

// --------------------------------------------------------------------------
// The decode kernel.  Persistent: a grid of (SMs x resident CTAs) CTAs of
// WPC independent warps.  A work item is one (sequence, KV head, context
// chunk); items are numbered chunk-major with the KV head fastest (see
// item_set).  A warp's first item is fixed by its index; after that it takes
// the next untaken item from a counter (split launches) or steps by the
// grid's warp count.  A warp streams its items' pages through its own
// SPW-slot ring back to back: the issue cursor runs SPW pages ahead of the
// compute cursor, across item boundaries, so the ring never drains between
// chunks.  There are no CTA barriers in the loop: each warp writes its
// chunk's result straight from registers.
// --------------------------------------------------------------------------
struct Item {
  int b, kvh, chunk, n, tok0, tok1, npages;
};

// Item idx < max_chunks * B * H_kv (< 2^31), numbered chunk-major with the
// KV head fastest: idx = (chunk * B + b) * H_kv + kvh.  Neighbouring warps
// then stream the same blocks for different KV heads at about the same
// time, and a block's KV-head pages are contiguous in the cache (H_kv x 2 KB
// of codes, H_kv x 64 B of scales), so DRAM sees long runs instead of
// scattered 2 KB pages.
__device__ __forceinline__ void item_set(const DecodeParams& p, uint32_t idx,
                                         Item& it) {
  const uint32_t per_chunk = static_cast<uint32_t>(p.num_kv_heads) * p.batch;
  const uint32_t c = idx / per_chunk;
  const uint32_t rem = idx - c * per_chunk;
  it.chunk = static_cast<int>(c);
  it.b = static_cast<int>(rem / static_cast<uint32_t>(p.num_kv_heads));
  it.kvh = static_cast<int>(rem - static_cast<uint32_t>(it.b) * p.num_kv_heads);
}

// Fill in the item's extent; false if the chunk lies past its sequence (a
// context of length 0 keeps chunk 0, with no pages, so that its zero row is
// written).
__device__ __forceinline__ bool item_fill(const DecodeParams& p, Item& it) {
  it.n = p.context_lens[it.b];
  it.tok0 = it.chunk * p.chunk_tokens;
  if (p.partials_only && it.tok0 >= it.n) {  // an empty slot: (-inf, 0, 0)
    it.tok1 = it.tok0;
    it.npages = 0;
    return true;
  }
  if (it.tok0 >= it.n && !(it.n == 0 && it.chunk == 0)) return false;
  if (p.prefix_group) {  // whole chunks of a shared prefix: a prefix launch's
    const int g = p.prefix_group[it.b];
    if (g >= 0 && it.chunk < p.prefix_lens[g] / p.chunk_tokens) return false;
  }
  it.tok1 = min(it.n, it.tok0 + p.chunk_tokens);
  it.npages = (it.tok1 - it.tok0 + kBS - 1) / kBS;
  return true;
}

// Fused append, by one warp: quantise token T_b - 1 of sequence b for KV
// head kvh (its K and V rows, 128 bf16 each) into the INT8 cache at the
// slot the block table gives for that position -- the arithmetic of
// kv8_quantize_append (s = fl32(max|x| / 127), codes rint(fl32(x / s))
// clamped to +-127, IEEE divisions), so the codes and scales are the same
// bit for bit -- then make the writes visible to this thread's later TMA
// copies.  Each lane handles 4 dims.
__device__ __forceinline__ void append_token(const DecodeParams& p, int b,
                                             int kvh, int n, int lane) {
  const int pos = n - 1;
  const int64_t blk = p.block_tables[static_cast<int64_t>(b) * p.max_blocks_per_seq +
                                     pos / kBS];
  const int64_t slot = (blk * p.num_kv_heads + kvh) * kBS + pos % kBS;
  const int64_t row = static_cast<int64_t>(b) * p.num_kv_heads + kvh;
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
    const __nv_bfloat16* src = (kv ? p.v_new : p.k_new) + row * kD;
    const uint2 raw = reinterpret_cast<const uint2*>(src)[lane];
    float x[4];
    x[0] = __uint_as_float(raw.x << 16);
    x[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    x[2] = __uint_as_float(raw.y << 16);
    x[3] = __uint_as_float(raw.y & 0xFFFF0000u);
    float a = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, m));
    const float sc = (a == 0.0f) ? 0.0f : __fdiv_rn(a, 127.0f);
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int c = 0;
      if (sc != 0.0f) {
        const float r = fminf(fmaxf(rintf(__fdiv_rn(x[i], sc)), -127.0f), 127.0f);
        c = static_cast<int>(r);
      }
      packed |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * i);
    }
    reinterpret_cast<uint32_t*>((kv ? p.v_cache_w : p.k_cache_w) + slot * kD)[lane] =
        packed;
    if (lane == 0) (kv ? p.v_scales_w : p.k_scales_w)[slot] = sc;
  }
  fence_proxy_async_global();
  __syncwarp();
}

// The result of an item without pages: a zero output row for an empty
// context (a single-chunk item), else an empty partial (m = -inf, l = 0,
// o = 0) that a merge skips.  Warp-cooperative.
template <int G>
__device__ __forceinline__ void write_empty(const DecodeParams& p,
                                            const Item& it, int lane) {
  const int64_t row0 = static_cast<int64_t>(it.b) * p.num_q_heads + it.kvh * G;
  const int nchunks = (it.n + p.chunk_tokens - 1) / p.chunk_tokens;
  for (int h = 0; h < G; ++h) {
    if (nchunks <= 1 && !p.partials_only) {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        store_out(p.out, (row0 + h) * kD + 4 * lane + e, 0.0f, p.out_f32);
    } else {
      const int64_t ci = (row0 + h) * p.max_chunks + it.chunk;
      reinterpret_cast<float4*>(p.ws_o + ci * kD)[lane] =
          make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (lane == 0) {
        p.ws_ml[2 * ci] = -INFINITY;
        p.ws_ml[2 * ci + 1] = 0.0f;
      }
    }
  }
}

template <int G, int WPC, int SPW, class Math>
__global__ void __launch_bounds__(WPC * 32,
                                  Math::kWarpsPerSM / WPC > 0 ? Math::kWarpsPerSM / WPC : 1)
decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv) {
  using Plan = SmemPlan<WPC, SPW, Math::kScratchBytes, Math::kCodeBytes>;
  constexpr int kCB = Math::kCodeBytes;
  constexpr uint32_t kPageTx = 2 * kCB + 2 * kBS * sizeof(float);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint8_t* tiles = smem + warp * SPW * 2 * kCB;
  float* scl = reinterpret_cast<float*>(smem + Plan::kTileBytes) +
               warp * SPW * 2 * kBS;
  uint8_t* scratch =
      smem + Plan::kTileBytes + Plan::kScaleBytes + warp * Math::kScratchBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      smem + Plan::kTileBytes + Plan::kScaleBytes + Plan::kScratchBytes +
      warp * (SPW * 8 + kQueue * 4));
  const uint32_t tiles_s = smem_u32(tiles), scl_s = smem_u32(scl);
  if (lane == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
#pragma unroll
    for (int s = 0; s < SPW; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  // tensor memory for the page math, if it keeps state there: warp w uses
  // lanes 32w..32w+31 of the CTA's columns
  uint32_t* tslot = reinterpret_cast<uint32_t*>(
      smem + Plan::kTileBytes + Plan::kScaleBytes + Plan::kScratchBytes +
      Plan::kBarBytes);
  if constexpr (Math::kTmemCols > 0) {
    if (warp == 0) {
      asm volatile(
          "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
              smem_u32(tslot)),
          "r"(Math::kTmemCols)
          : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::
                       : "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  }

  // ---- work items.  A warp's first item is gw = CTA * WPC + warp; its
  // next ones are gw + W, gw + 2W, ... (W = warps in the grid) or, when the
  // launch has a work counter, W + (counter++): a warp that finishes early
  // takes more, so uneven items do not leave a slow tail.  The issue cursor
  // takes items and queues their indices in shared memory; the compute
  // cursor, up to SPW pages behind, pops them in the same order.  Items
  // without pages (an empty context, or a partials slot past a sequence's
  // end) are finished by the issue side when taken and never queued, so
  // every queued item holds a page in flight: at most SPW of them, plus the
  // end marker.
  int* wq = reinterpret_cast<int*>(bars + SPW);  // kQueue entries per warp
  uint32_t q_tail = 0, q_head = 0;
  // item indices fit 31 bits (the host checks max_chunks * H_kv * B).  In a
  // launch beside a shared-prefix launch, the chunks every sequence leaves
  // to that launch (the fewest whole prefix chunks of any sequence) are not
  // enumerated at all: items start at chunk c_first.
  const uint32_t per_chunk = static_cast<uint32_t>(p.num_kv_heads) * p.batch;
  uint32_t c_first = 0;
  if (p.prefix_group) {
    int mn = p.max_chunks;
    for (int b = lane; b < p.batch; b += 32) {
      const int g = p.prefix_group[b];
      mn = min(mn, g >= 0 ? p.prefix_lens[g] / p.chunk_tokens : 0);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) mn = min(mn, __shfl_xor_sync(kFull, mn, m));
    c_first = static_cast<uint32_t>(mn);
  }
  const uint32_t base = c_first * per_chunk;
  const uint32_t n_items = (static_cast<uint32_t>(p.max_chunks) - c_first) * per_chunk;
  const uint32_t W = gridDim.x * WPC;
  uint32_t next_idx = blockIdx.x * WPC + warp;
  bool first_take = true;
  // issue side: the next item that has work (or none); queues its index
  auto take = [&](Item& it) -> bool {
    for (;;) {
      uint32_t idx = next_idx;
      if (!first_take) {
        if (p.work_ctr) {
          uint32_t t = 0;
          if (lane == 0) t = atomicAdd(p.work_ctr, 1u);
          idx = W + __shfl_sync(kFull, t, 0);
        } else {
          idx = next_idx + W;
        }
      }
      first_take = false;
      next_idx = idx;
      const bool live = idx < n_items;  // (no wrap: W + counter < 2^32)
      if (live) item_set(p, base + idx, it);
      if (!live || item_fill(p, it)) {
        if (live && it.npages == 0) {
          write_empty<G>(p, it, lane);
          continue;
        }
        // fused append: the item holding the sequence's last page, before
        // any of its pages is copied (no other item reads that page)
        if (live && p.k_new && it.tok1 == it.n && it.n > 0)
          append_token(p, it.b, it.kvh, it.n, lane);
        if (live && lane < 2 * G) {
          // the item's q rows (G x 256 B) into L1 now, SPW pages before the
          // compute side loads them
          const __nv_bfloat16* qrow =
              p.q + (static_cast<int64_t>(it.b) * p.num_q_heads + it.kvh * G) * kD;
          asm volatile("prefetch.global.L1 [%0];" ::"l"(
              reinterpret_cast<const char*>(qrow) + 128 * lane));
        }
        if (lane == 0) wq[q_tail % kQueue] = live ? static_cast<int>(base + idx) : -1;
        ++q_tail;
        __syncwarp();
        return live;
      }
    }
  };
  // compute side: the next queued item (false: no more)
  auto pop = [&](Item& it) -> bool {
    __syncwarp();
    const int idx = wq[q_head % kQueue];
    ++q_head;
    if (idx < 0) return false;
    item_set(p, static_cast<uint32_t>(idx), it);
    item_fill(p, it);
    return true;
  };

  // ---- issue cursor: SPW pages ahead of the compute cursor.  Its state is
  // kept small (the page math needs the registers): the table offset of the
  // item's first page, its KV head and page count, and the page reached.
  const uint32_t bars_s = smem_u32(bars);
  bool iss_live;
  int iss_page = 0, iss_np = 0, iss_kvh = 0;
  int64_t iss_tab = 0;
  auto take_iss = [&]() {
    Item it;
    iss_live = take(it);
    iss_page = 0;
    if (iss_live) {
      iss_np = it.npages;
      iss_kvh = it.kvh;
      iss_tab = static_cast<int64_t>(it.b) * p.max_blocks_per_seq + it.tok0 / kBS;
    }
  };
  take_iss();
  int bt_reg = 0;
  uint32_t k_iss = 0;
  int slot_iss = 0;
  auto issue_one = [&]() {
    while (iss_live && iss_page >= iss_np) take_iss();
    if (!iss_live) return;
    if ((iss_page & 31) == 0) {
      const int j = iss_page + lane;
      bt_reg = j < iss_np ? p.block_tables[iss_tab + j] : 0;
    }
    const int blk = __shfl_sync(kFull, bt_reg, iss_page & 31);
    bool issue_copies = true;
#ifdef KV8_TEST_HOOKS
    issue_copies = !(g_test_skip_first_copy && blockIdx.x == 0 && warp == 0 &&
                     k_iss == 0);
#endif
    if (lane == 0) {
      const uint32_t bar = bars_s + slot_iss * 8;
      mbar_arrive_expect_tx_s(bar, kPageTx);
      if (issue_copies) {
        const int page = blk * (p.num_kv_heads >> p.kv_sub_shift) +
                         (iss_kvh >> p.kv_sub_shift);
        const uint32_t tk = tiles_s + slot_iss * (2 * kCB);
        const uint32_t sc = scl_s + slot_iss * (2 * kBS * 4);
        tma_load_3d_s(tk, &tmk, 0, 0, page, bar);
        tma_load_3d_s(tk + kCB, &tmv, 0, 0, page, bar);
        bulk_g2s_s(sc, p.k_scales + static_cast<int64_t>(page) * kBS,
                   kBS * sizeof(float), bar);
        bulk_g2s_s(sc + kBS * 4, p.v_scales + static_cast<int64_t>(page) * kBS,
                   kBS * sizeof(float), bar);
      }
    }
    ++k_iss;
    ++iss_page;
    slot_iss = slot_iss + 1 == SPW ? 0 : slot_iss + 1;
  };
#pragma unroll 1
  for (int s = 0; s < SPW; ++s) issue_one();

  Math math;
  math.attach(scratch);
  if constexpr (Math::kTmemCols > 0)
    math.attach_tmem(*tslot + (static_cast<uint32_t>(32 * warp) << 16));
  uint32_t k_cmp = 0;
  int slot = 0;
  uint32_t phase = 0;
  bool ok = true;
  Item cmp;
  bool cmp_live = pop(cmp);
  while (cmp_live) {
    const int64_t row0 = static_cast<int64_t>(cmp.b) * p.num_q_heads + cmp.kvh * G;
    math.init(p.q + row0 * kD, p.q_scale, lane);
    for (int j = 0; j < cmp.npages; ++j) {
      if (!mbar_wait_s(bars_s + slot * 8, phase, &g_device_status)) {
        ok = false;
        break;
      }
      const int nv = cmp.tok1 - (cmp.tok0 + j * kBS);
      if constexpr (Math::kSharedAddr) {
        const uint32_t tk = tiles_s + slot * (2 * kCB);
        const uint32_t ks = scl_s + slot * (2 * kBS * 4);
        if (nv >= kBS)
          math.template page_s<true>(tk, tk + kCB, ks, ks + kBS * 4, kBS);
        else
          math.template page_s<false>(tk, tk + kCB, ks, ks + kBS * 4, nv);
      } else {
        const uint8_t* tk = tiles + slot * 2 * kCB;
        const float* ks = scl + slot * 2 * kBS;
        if (nv >= kBS)
          math.template page<true>(tk, tk + kCB, ks, ks + kBS, kBS);
        else
          math.template page<false>(tk, tk + kCB, ks, ks + kBS, nv);
      }
      __syncwarp();
      issue_one();
      ++k_cmp;
      if (++slot == SPW) {
        slot = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;

    ChunkSink sk;
    sk.out = p.out;
    sk.ws_o = p.ws_o;
    sk.ws_ml = p.ws_ml;
    sk.row0 = row0;
    sk.ci0 = row0 * p.max_chunks + cmp.chunk;
    sk.max_chunks = p.max_chunks;
    const int nchunks = (cmp.n + p.chunk_tokens - 1) / p.chunk_tokens;
    sk.single = nchunks <= 1 && !p.partials_only;
    sk.out_f32 = p.out_f32;
    math.finish(sk);

    if (!sk.single && !p.partials_only) {
      // the last chunk of this (sequence, KV group) to finish merges them
      __threadfence();
      __syncwarp();
      unsigned int ticket = 0;
      if (lane == 0) ticket = atomicAdd(&p.ws_ctr[row0], 1u);
      ticket = __shfl_sync(kFull, ticket, 0);
      if (ticket == static_cast<unsigned int>(nchunks - 1)) {
        __threadfence();
        merge_group_warp<G>(p.ws_ml, p.ws_o, row0, p.max_chunks, nchunks,
                            p.out, p.out_f32);
      }
    }
    cmp_live = pop(cmp);
  }
  if (!ok) {
    // A copy never landed: drain the other copies in flight (bounded) and
    // stop.  The sticky status word reports it.
    for (uint32_t k = k_cmp + 1; k < k_iss; ++k)
      mbar_wait(&bars[k % SPW], (k / SPW) & 1, &g_device_status);
  }
  if constexpr (Math::kTmemCols > 0) {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(
                       *tslot),
                   "r"(Math::kTmemCols)
                   : "memory");
  }
}

// --------------------------------------------------------------------------
// Standalone split reduce: one warp per (b, hq), the same merge routine as
// the fused merge of the decode kernel.
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(32)
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
  merge_head_warp(ws_ml + static_cast<int64_t>(bh) * max_chunks * 2,
                  ws_o + static_cast<int64_t>(bh) * max_chunks * kD, nchunks,
                  out, bh, out_f32);
}

// --------------------------------------------------------------------------
// Merge across ranks: one warp per (b, hq) over ranks x max_chunks partials
// (empty ones carry m = -inf and weigh nothing).
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(32)
merge_ranks_kernel(const uint8_t* __restrict__ partials, size_t rank_stride,
                   size_t o_offset, int32_t ranks, int32_t max_chunks,
                   void* out, int32_t out_f32) {
  const int64_t bh = blockIdx.x;
  const int lane = threadIdx.x;
  const int total = ranks * max_chunks;
  auto ml_at = [&](int k) {
    const int r = k / max_chunks, c = k - r * max_chunks;
    return reinterpret_cast<const float*>(partials + r * rank_stride) +
           (bh * max_chunks + c) * 2;
  };
  auto o_at = [&](int k) {
    const int r = k / max_chunks, c = k - r * max_chunks;
    return reinterpret_cast<const float*>(partials + r * rank_stride + o_offset) +
           (bh * max_chunks + c) * kD;
  };
  float mx = -INFINITY;
  for (int k = lane; k < total; k += 32) mx = fmaxf(mx, ml_at(k)[0]);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
  float ls = 0.0f;
  for (int k = lane; k < total; k += 32) {
    const float* ml = ml_at(k);
    ls += ml[0] == -INFINITY ? 0.0f : ml[1] * ex2(ml[0] - mx);
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) ls += __shfl_xor_sync(kFull, ls, m);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k = 0; k < total; ++k) {
    const float mc = ml_at(k)[0];
    if (mc == -INFINITY) continue;
    const float w = ex2(mc - mx);
    const float4 v = reinterpret_cast<const float4*>(o_at(k))[lane];
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  const float inv = ls > 0.0f ? 1.0f / ls : 0.0f;
  const int64_t base = bh * kD + 4 * lane;
  store_out(out, base + 0, acc.x * inv, out_f32);
  store_out(out, base + 1, acc.y * inv, out_f32);
  store_out(out, base + 2, acc.z * inv, out_f32);
  store_out(out, base + 3, acc.w * inv, out_f32);
}

template <int G, int WPC, int SPW, class Math>
int launch_decode_kernel(const DecodeParams& p, const CUtensorMap& tmk,
                         const CUtensorMap& tmv, cudaStream_t stream) {
  auto kern = decode_kernel<G, WPC, SPW, Math>;
  constexpr int smem =
      SmemPlan<WPC, SPW, Math::kScratchBytes, Math::kCodeBytes>::kBytes;
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
    const int occ = resident_ctas(kern, WPC * 32, smem, Math::kTmemCols);
    if (occ == 0) return -1;
    sms = nsm;
    resident = occ;
    f->sms.store(sms, std::memory_order_release);
    f->resident.store(resident, std::memory_order_release);
  }
  const int64_t n_items =
      static_cast<int64_t>(p.max_chunks) * p.num_kv_heads * p.batch;
  int64_t ctas = static_cast<int64_t>(sms) * resident;
  const int64_t need = (n_items + WPC - 1) / WPC;
  if (ctas > need) ctas = need;
  if (ctas < 1) ctas = 1;
  kern<<<static_cast<unsigned>(ctas), WPC * 32, smem, stream>>>(p, tmk, tmv);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int G>
int launch_group(const DecodeParams& p, const CUtensorMap& tmk,
                 const CUtensorMap& tmv, int32_t variant, cudaStream_t stream) {
  if (variant == KV8_FORM_CUDA_CORE)
    return launch_decode_kernel<G, 4, 4, SimtMath<G>>(p, tmk, tmv, stream);
  // automatic: both products on int8 mma for groups of up to 4 heads
  // (their accumulators fit a warp), the fp16 p.v form for groups of 8
  if constexpr (G <= 4) {
    // partials in tensor memory leave room for a fourth page slot per warp
    if (variant == KV8_FORM_MMA_I8 || variant == KV8_FORM_AUTO)
      return launch_decode_kernel<G, 4, 4, I8Math<G, true>>(p, tmk, tmv, stream);
  }
  return launch_decode_kernel<G, 4, 3, MmaMath<G>>(p, tmk, tmv, stream);
}

// INT4 cache: 1 KB pages, so twice the slots of the INT8 form for the same
// bytes in flight per warp
template <int G>
int launch_group_int4(const DecodeParams& p, const CUtensorMap& tmk,
                      const CUtensorMap& tmv, cudaStream_t stream) {
  return launch_decode_kernel<G, 4, 8, I4Math<G>>(p, tmk, tmv, stream);
}

}  // namespace

#ifdef KV8_TEST_HOOKS
int test_skip_first_copy(int on) {
  return cudaMemcpyToSymbol(g_test_skip_first_copy, &on, sizeof(int)) ==
                 cudaSuccess
             ? 0
             : -1;
}
#endif

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
  uint32_t tc = 0, pf = 0, ex = 0;
  if (read_tc_status(&tc, clear) != 0) return -1;
  if (read_prefix_status(&pf, clear) != 0) return -1;
  if (read_ext_status(&ex, clear) != 0) return -1;
  *value |= tc | pf | ex;
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
  // merge tickets, then the work counter (padded to 16 bytes)
  return static_cast<size_t>(batch) * num_q_heads * sizeof(uint32_t) + 16;
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

int launch_decode_int4(const DecodeParams& p, const CUtensorMap& tmk,
                       const CUtensorMap& tmv, cudaStream_t stream) {
  const int g = p.num_q_heads / p.num_kv_heads;
  switch (g) {
    case 1: return launch_group_int4<1>(p, tmk, tmv, stream);
    case 2: return launch_group_int4<2>(p, tmk, tmv, stream);
    case 4: return launch_group_int4<4>(p, tmk, tmv, stream);
    case 8: {
      // groups of 8: two sub-groups of 4 query heads per KV head, each its
      // own item (a warp's integer accumulators hold 4 heads); the two
      // warps of a KV head read the same pages at about the same time
      // (sub-groups are numbered fastest), so the second read hits L2
      if (static_cast<int64_t>(p.max_chunks) * 2 * p.num_kv_heads * p.batch >
          INT32_MAX)
        return -2;
      DecodeParams q = p;
      q.num_kv_heads = 2 * p.num_kv_heads;
      q.kv_sub_shift = 1;
      return launch_group_int4<4>(q, tmk, tmv, stream);
    }
    default: return -2;
  }
}

int launch_merge_ranks(const uint8_t* partials, size_t rank_stride,
                       int32_t ranks, int32_t batch, int32_t num_q_heads,
                       int32_t max_chunks, void* out, int32_t out_f32,
                       cudaStream_t stream) {
  const int64_t nbh = static_cast<int64_t>(batch) * num_q_heads;
  if (nbh == 0) return 0;
  merge_ranks_kernel<<<static_cast<unsigned>(nbh), 32, 0, stream>>>(
      partials, rank_stride, workspace_ml_bytes(batch, num_q_heads, max_chunks),
      ranks, max_chunks, out, out_f32);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_split_reduce(const float* ws_ml, const float* ws_o,
                        const int32_t* context_lens, int32_t batch,
                        int32_t num_q_heads, int32_t chunk_tokens,
                        int32_t max_chunks, void* out, int32_t out_f32,
                        cudaStream_t stream) {
  const int64_t nbh = static_cast<int64_t>(batch) * num_q_heads;
  if (nbh == 0) return 0;
  split_reduce_kernel<<<static_cast<unsigned>(nbh), 32, 0, stream>>>(
      ws_ml, ws_o, context_lens, num_q_heads, chunk_tokens, max_chunks, out,
      out_f32);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace kv8
