// kv8_prefix.cu -- decode attention over the shared prefix of groups of
// sequences, on the 5th-generation tensor cores: the pages several sequences
// list at the start of their block tables are read, converted and scored
// once for all the group's query rows together.
//
// What is computed is unchanged from kv8_decode.cu [KV Cache 优化全景解析——
// 从基础原理到工程实践, §2.1, §3.3]; what changes is how shared pages are
// visited.  PagedAttention lets several sequences map the same physical
// blocks [same page, §4.2], and serving systems group the requests that
// share a prefix so the shared part is handled once [garden.houmin.site
// infra/kv-cache-optimize, §4.3.1 Prefix-aware Scheduling (BatchLLM)].
//
// For whole chunks of the shared prefix and one KV head, the new tokens of
// the group's members form a block of query rows -- member m, head h -- all
// attending to the same keys: a dense contraction of up to 128 rows, which
// is the extend kernel's tile.  A work item is (a run of whole prefix
// chunks of about 512 keys, KV head, group, round of 128 / G members); the
// CTA runs the extend kernel's roles from kv8_tc.cuh (TMA producer, tcgen05
// issuer, int8 -> fp16 converters, eight softmax warps, each row split over
// two of them) with no causal mask, and each row ends as the member's
// partial (m, l, o) in the split workspace, in the slot of the run's first
// chunk (the run's other slots hold empty partials).  It then advances the
// member's merge ticket by the run's chunk count: chunks computed here and
// the member's own chunks computed by the decode kernel merge into one
// output row by log-sum-exp, in either order.
#include "../../include/kv8.h"
#include "kv8_common.cuh"
#include "kv8_internal.h"
#include "kv8_tc.cuh"

namespace kv8 {

__device__ uint32_t g_prefix_status = 0;

namespace {

// Warp-wide scan of prefix_group: the sequence of rank `rank` (by sequence
// index) among the members of group g, each lane with its own rank; -1
// where the group has no member of that rank.
__device__ __forceinline__ int member_of(const DecodeParams& p, int g, int rank,
                                         int lane) {
  int found = -1, seen = 0;
  for (int base = 0; base < p.batch; base += 32) {
    const int b = base + lane;
    const int v = b < p.batch ? p.prefix_group[b] : -1;
    const uint32_t m = __ballot_sync(kFull, v == g);
    const int cnt = __popc(m);
    if (found < 0 && rank >= seen && rank < seen + cnt)
      found = base + static_cast<int>(__fns(m, 0, rank - seen + 1));
    seen += cnt;
    if (__all_sync(kFull, rank < seen)) break;
  }
  return found;
}

// Item idx = ((cg * H_kv + kvh) * groups + g) * rounds + rnd: chunks
// [c0, c1) of group g's whole prefix chunks, c0 = cg * chunks_per_item.
struct PrefixItem {
  int c0, c1, kvh, g, rnd;
};
__device__ __forceinline__ bool pitem_load(const DecodeParams& p,
                                           const PrefixShape& ps, int members,
                                           int64_t idx, PrefixItem& it,
                                           int& first, int lane) {
  it.rnd = static_cast<int>(idx % ps.rounds);
  idx /= ps.rounds;
  it.g = static_cast<int>(idx % ps.num_groups);
  idx /= ps.num_groups;
  it.kvh = static_cast<int>(idx % p.num_kv_heads);
  it.c0 = static_cast<int>(idx / p.num_kv_heads) * ps.chunks_per_item;
  const int whole = p.prefix_lens[it.g] / p.chunk_tokens;
  if (it.c0 >= whole) return false;
  it.c1 = min(whole, it.c0 + ps.chunks_per_item);
  // lane 0: the group's first member (its table lists the prefix blocks);
  // lane 1: the round's first member (none: the round is empty)
  const int b = member_of(p, it.g, lane == 1 ? members * it.rnd : 0, lane);
  first = __shfl_sync(kFull, b, 0);
  return __shfl_sync(kFull, b, 1) >= 0;
}

// The prefix items as the producer, issuer and converter roles see them.
struct PrefixItems {
  const DecodeParams& p;
  const PrefixShape& ps;
  int members;  // per round: 128 / G
  __device__ __forceinline__ int64_t size() const {
    const int64_t groups_of_chunks =
        (ps.prefix_chunks + ps.chunks_per_item - 1) / ps.chunks_per_item;
    return groups_of_chunks * p.num_kv_heads * ps.num_groups * ps.rounds;
  }
  __device__ __forceinline__ bool load(int64_t idx, TileItem& t, int lane) const {
    PrefixItem it;
    int first;
    if (!pitem_load(p, ps, members, idx, it, first, lane)) return false;
    const int keys = (it.c1 - it.c0) * p.chunk_tokens;
    t.tab = static_cast<int64_t>(first) * p.max_blocks_per_seq +
            it.c0 * (p.chunk_tokens / kBS);
    t.kvh = it.kvh;
    t.npages = keys / kBS;
    t.nkt = (keys + kKT - 1) / kKT;
    return true;
  }
};

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
prefix_kernel(const DecodeParams p, const PrefixShape ps,
              const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv) {
  constexpr int M = kRows / G;  // members per round
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ExtPlan::kBar);
  const uint32_t tmem = tc_setup(smem, &tmk, &tmv, warp);
  bool failed = false;

  const PrefixItems items{p, ps, M};
  if (warp == 0) {
    tc_produce(items, p.block_tables, p.num_kv_heads, p.k_scales, p.v_scales,
               &tmk, &tmv, smem, bars, failed, &g_prefix_status, lane);
  } else if (warp == 1) {
    tc_issue(items, smem, bars, tmem, failed, &g_prefix_status, lane);
  } else if (warp < 4) {
    tc_convert(items, smem, bars, failed, &g_prefix_status, threadIdx.x - 64,
               lane);
  } else {
    // ================================================= softmax (8 warps)
    // row r = 32 qd + lane = member r / G of the round, head r % G (a
    // member's G rows lie in one warp); half hf takes key columns and output
    // dims 64 hf .. 64 hf + 63
    const int sw = warp - 4, qd = sw & 3, hf = sw >> 2;
    const int r = 32 * qd + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * qd) << 16);
    const int mr = r / G, head = r % G;
    uint32_t u = 0, xk = 0;
    const int64_t n = items.size();
    for (int64_t idx = blockIdx.x; idx < n; idx += gridDim.x) {
      PrefixItem it;
      int first;
      if (!pitem_load(p, ps, M, idx, it, first, lane)) continue;
      const int b = member_of(p, it.g, M * it.rnd + mr, lane);
      const int keys = (it.c1 - it.c0) * p.chunk_tokens;  // this item's keys
      const int nkt = (keys + kKT - 1) / kKT;
      int n_b = 0;
      bool live = false;
      if (b >= 0) {
        n_b = p.context_lens[b];
        live = n_b >= it.c1 * p.chunk_tokens;
        if (!live && head == 0 && hf == 0)
          atomicOr(&g_prefix_status, KV8_DEV_BAD_PREFIX);
      }
      const int64_t row =
          static_cast<int64_t>(live ? b : 0) * p.num_q_heads + it.kvh * G + head;
      const float qf =
          tc_stage_q(smem, p.q + row * kD, live, r, hf, qd, p.q_scale, xk);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_Q_FULL]);
      {
        // the next item's q rows (this half: 128 bytes) into L1 while this
        // item's tiles run, so its staging does not wait on L2
        PrefixItem nx;
        int nfirst;
        const int64_t nidx = idx + gridDim.x;
        if (nidx < n && pitem_load(p, ps, M, nidx, nx, nfirst, lane)) {
          const int nb = member_of(p, nx.g, M * nx.rnd + mr, lane);
          if (nb >= 0) {
            const __nv_bfloat16* nq =
                p.q + (static_cast<int64_t>(nb) * p.num_q_heads + nx.kvh * G + head) * kD;
            asm volatile("prefetch.global.L1 [%0];" ::"l"(
                reinterpret_cast<const char*>(nq) + 128 * hf));
          }
        }
      }

      // ---- the item's keys (its chunks, one after the other), all visible
      // to every row
      const RowSoftmax rs =
          tc_row_tiles(smem, bars, trow, r, hf, qd, lane, live, keys, qf, nkt,
                       u, xk, failed, &g_prefix_status);
      u += nkt;
      const float l = rs.l + pair_xch(smem, xk, hf, r, qd, make_float2(rs.l, 0.0f)).x;
      ewait(&bars[B_O_DONE], (u - 1) & 1, failed, &g_prefix_status);
      __syncwarp();
      tc_fence_after();

      // ---- the row's result over the item's chunks (this half's dims): the
      // member's output row when they are its whole context, else one
      // partial (m, l, o) in the slot of the first chunk, o relative to m and
      // unnormalised, and empty partials (m = -inf, l = 0; a merge reads
      // nothing else of them) in the slots of the others
      const int nchunks = (n_b + p.chunk_tokens - 1) / p.chunk_tokens;
      const int nmine = it.c1 - it.c0;
      const bool single = nchunks <= nmine;
      const float f = single ? pow2i(rs.e) / (l > 0.0f ? l : 1.0f) : pow2i(rs.e);
      const int64_t ci = row * p.max_chunks + it.c0;
#pragma unroll 1
      for (int c = 0; c < kHalf / 32; ++c) {
        float o[32];
        const int d0 = kHalf * hf + 32 * c;
        __syncwarp();  // the stores below diverge by row; reconverge first
        tmem_ld32(trow + kColO + d0, o);
        if (!live) continue;
        if (!single) {
          float4* dst = reinterpret_cast<float4*>(p.ws_o + ci * kD + d0);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(o[4 * i] * f, o[4 * i + 1] * f,
                                 o[4 * i + 2] * f, o[4 * i + 3] * f);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            store_out(p.out, row * kD + d0 + i, o[i] * f, p.out_f32);
        }
      }
      if (live && !single && hf == 0) {
        p.ws_ml[2 * ci] = rs.m;
        p.ws_ml[2 * ci + 1] = l;
        for (int k = 1; k < nmine; ++k) {
          p.ws_ml[2 * (ci + k)] = -INFINITY;
          p.ws_ml[2 * (ci + k) + 1] = 0.0f;
        }
      }
      tc_fence_before();

      // ---- each member's ticket, taken by its head-0 row of half 0 once
      // both halves of the member's G rows are written; the last of the
      // member's chunks merges them
      __threadfence();
      pair_sync(qd);
      const bool lead = live && !single && head == 0 && hf == 0;
      unsigned int ticket = 0;
      if (lead) ticket = atomicAdd(&p.ws_ctr[row], static_cast<unsigned int>(nmine));
      uint32_t mm = __ballot_sync(
          kFull, lead && ticket + nmine == static_cast<unsigned int>(nchunks));
      while (mm) {
        const int src = __ffs(mm) - 1;
        mm &= mm - 1;
        const int bs = __shfl_sync(kFull, b, src);
        const int nch = __shfl_sync(kFull, nchunks, src);
        const int64_t r0 = static_cast<int64_t>(bs) * p.num_q_heads + it.kvh * G;
        __threadfence();
        merge_group_warp<G>(p.ws_ml, p.ws_o, r0, p.max_chunks, nch, p.out,
                            p.out_f32);
      }
    }
  }
  tc_teardown(tmem, warp);
}

template <int G>
int launch_prefix_group(const DecodeParams& p, PrefixShape ps,
                        const CUtensorMap& tmk, const CUtensorMap& tmv,
                        cudaStream_t stream) {
  auto kern = prefix_kernel<G>;
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
  constexpr int M = kRows / G;
  ps.rounds = (ps.max_group_size + M - 1) / M;
  // items of about 512 keys (4 tiles): with finer chunks an item covers
  // several, so the call can split the suffixes finely without one-tile
  // items here
  ps.chunks_per_item = p.chunk_tokens >= 512 ? 1 : 512 / p.chunk_tokens;
  const int64_t n_items =
      static_cast<int64_t>((ps.prefix_chunks + ps.chunks_per_item - 1) /
                           ps.chunks_per_item) *
      p.num_kv_heads * ps.num_groups * ps.rounds;
  if (n_items == 0) return 0;
  int64_t ctas = sms;
  if (ctas > n_items) ctas = n_items;
  kern<<<static_cast<unsigned>(ctas), kThreads, smem, stream>>>(p, ps, tmk, tmv);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

int launch_prefix(const DecodeParams& p, const PrefixShape& ps,
                  const CUtensorMap& tmk, const CUtensorMap& tmv,
                  cudaStream_t stream) {
  switch (p.num_q_heads / p.num_kv_heads) {
    case 1: return launch_prefix_group<1>(p, ps, tmk, tmv, stream);
    case 2: return launch_prefix_group<2>(p, ps, tmk, tmv, stream);
    case 4: return launch_prefix_group<4>(p, ps, tmk, tmv, stream);
    case 8: return launch_prefix_group<8>(p, ps, tmk, tmv, stream);
    default: return -2;
  }
}

int read_prefix_status(uint32_t* value, int clear) {
  if (cudaMemcpyFromSymbol(value, g_prefix_status, sizeof(uint32_t)) !=
      cudaSuccess)
    return -1;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_prefix_status, &zero, sizeof(uint32_t)) !=
        cudaSuccess)
      return -1;
  }
  return 0;
}

}  // namespace kv8
