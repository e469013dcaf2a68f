// kv8_prefix.cu -- decode attention over the shared prefix of groups of
// sequences: the pages several sequences list at the start of their block
// tables are read, converted and scored once for the whole group.
//
// What is computed is unchanged from kv8_decode.cu [KV Cache 优化全景解析——
// 从基础原理到工程实践, §2.1, §3.3]; what changes is how shared pages are
// visited.  PagedAttention lets several sequences map the same physical
// blocks [same page, §4.2], and serving systems group the requests that
// share a prefix so the shared part is handled once [garden.houmin.site
// infra/kv-cache-optimize, §4.3.1 Prefix-aware Scheduling (BatchLLM)].
//
// Work decomposition: a work item is one (prefix chunk, KV head, group,
// round of 8 members); a CTA of 8 warps takes items in turn (persistent
// grid), warp w serving member 8 * round + w of the group:
//   * warp 0 streams the chunk's pages (found through the block table of the
//     group's first member) into a ring of 4 slots with TMA, across item
//     boundaries, like the decode kernel's per-warp rings;
//   * each page's V codes are converted once to fp16 in shared memory, 2
//     tokens per warp, then a CTA barrier;
//   * each active warp runs the warp tensor-core page math (MmaMath) for its
//     member's G query heads on the shared K page and the converted V page;
//   * at the end of an item each warp hands its member's chunk result to the
//     same chunk partial / ticket / log-sum-exp merge as the decode kernel,
//     so chunks computed here and the member's own chunks computed by the
//     decode kernel merge into one output row, in either order.
#include "../../include/kv8.h"
#include "kv8_common.cuh"
#include "kv8_internal.h"
#include "kv8_merge.cuh"
#include "kv8_page_math.cuh"

namespace kv8 {

__device__ uint32_t g_prefix_status = 0;

namespace {

constexpr int kPW = 8;     // warps per CTA = members per round
constexpr int kPNB = 12;   // page slots in the CTA's ring (one CTA per SM:
                           // 11 pages in flight)
constexpr uint32_t kPTx = 2 * kPageBytes + 2 * kBS * sizeof(float);

// Shared memory (base aligned to 1024 bytes for the 128-byte swizzle):
//   [kPNB][K page 2048 | V page 2048]   TMA-staged int8 pages
//   [2][4096]                           V page as fp16 [16 tok][128 dims], by
//                                       page parity (page k's copy is free
//                                       once every warp is past page k+1's
//                                       barrier)
//   [kPNB][ks 64 | vs 64]               scales
//   [kPNB] mbarriers; two ints: a wait gave up, the first page not waited for
struct PrefixPlan {
  static constexpr int kTiles = 0;
  static constexpr int kVh = kTiles + kPNB * 2 * kPageBytes;
  static constexpr int kScl = kVh + 2 * 4096;
  static constexpr int kBar = kScl + kPNB * 2 * kBS * 4;
  static constexpr int kFail = kBar + kPNB * 8;
  static constexpr int kBytes = kFail + 16 + 1024;
};

struct PrefixItem {
  int chunk, kvh, g, rnd;
  int tok0, npages;
};

// Item idx, numbered chunk-major: idx = ((chunk * H_kv + kvh) * groups + g)
// * rounds + rnd.  False if the chunk is not a whole chunk of the group's
// prefix.
__device__ __forceinline__ bool pitem_load(const DecodeParams& p,
                                           const PrefixShape& ps, int64_t idx,
                                           PrefixItem& it) {
  it.rnd = static_cast<int>(idx % ps.rounds);
  idx /= ps.rounds;
  it.g = static_cast<int>(idx % ps.num_groups);
  idx /= ps.num_groups;
  it.kvh = static_cast<int>(idx % p.num_kv_heads);
  it.chunk = static_cast<int>(idx / p.num_kv_heads);
  const int whole = p.prefix_lens[it.g] / p.chunk_tokens;
  if (it.chunk >= whole) return false;
  it.tok0 = it.chunk * p.chunk_tokens;
  it.npages = p.chunk_tokens / kBS;
  return true;
}

// Warp-wide scan of prefix_group for group g: the first member (by sequence
// index) and the members of rank `mine` and `lead` (-1 where there is none).
__device__ __forceinline__ void find_members(const DecodeParams& p, int g,
                                             int mine, int lead, int lane,
                                             int& first, int& b_mine,
                                             int& b_lead) {
  first = b_mine = b_lead = -1;
  int seen = 0;
  for (int base = 0; base < p.batch; base += 32) {
    const int b = base + lane;
    const int v = b < p.batch ? p.prefix_group[b] : -1;
    const uint32_t m = __ballot_sync(kFull, v == g);
    const int cnt = __popc(m);
    if (m) {
      if (first < 0) first = base + __ffs(m) - 1;
      if (b_mine < 0 && mine < seen + cnt)
        b_mine = base + static_cast<int>(__fns(m, 0, mine - seen + 1));
      if (b_lead < 0 && lead < seen + cnt)
        b_lead = base + static_cast<int>(__fns(m, 0, lead - seen + 1));
    }
    seen += cnt;
    if (b_mine >= 0 && b_lead >= 0) break;
  }
}

// Bounded wait for page k; once any wait of the CTA has given up, later
// waits are skipped (the launch then only has to finish; the status word
// reports it) and the first page not waited for is recorded in fail[1].
__device__ __forceinline__ void pwait(uint64_t* bar, uint32_t parity,
                                      uint32_t k, volatile int* fail) {
  if (!fail[0] && mbar_wait(bar, parity, &g_prefix_status)) return;
  fail[0] = 1;
  atomicMin(const_cast<int*>(&fail[1]), static_cast<int>(k));
}

template <int G>
__global__ void __launch_bounds__(kPW * 32, 1)
prefix_kernel(const DecodeParams p, const PrefixShape ps,
              const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint8_t* tiles = smem + PrefixPlan::kTiles;
  uint8_t* vh = smem + PrefixPlan::kVh;
  float* scl = reinterpret_cast<float*>(smem + PrefixPlan::kScl);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PrefixPlan::kBar);
  volatile int* fail = reinterpret_cast<volatile int*>(smem + PrefixPlan::kFail);
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
    for (int s = 0; s < kPNB; ++s) mbar_init(&bars[s], 1);
    fail[0] = 0;
    fail[1] = 0x7fffffff;
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t n_items = static_cast<int64_t>(ps.prefix_chunks) *
                          p.num_kv_heads * ps.num_groups * ps.rounds;
  const int64_t stride = gridDim.x;

  // ---- issue cursor (warp 0): kPNB pages ahead, across items
  int64_t iss_idx = blockIdx.x;
  PrefixItem iss;
  int iss_page = 0, iss_first = -1, bt_reg = 0;
  bool iss_live = false;
  uint32_t k_iss = 0;
  auto iss_seek = [&]() {  // warp 0: the next item with pages, or none
    for (; iss_idx < n_items; iss_idx += stride) {
      if (!pitem_load(p, ps, iss_idx, iss)) continue;
      int b_mine, b_lead;
      find_members(p, iss.g, 0, 8 * iss.rnd, lane, iss_first, b_mine, b_lead);
      if (b_lead >= 0) {
        iss_live = true;
        iss_page = 0;
        return;
      }
    }
    iss_live = false;
  };
  auto issue_one = [&]() {  // warp 0
    if (!iss_live || __any_sync(kFull, fail[0] != 0)) return;
    if ((iss_page & 31) == 0) {
      const int j = iss_page + lane;
      bt_reg = j < iss.npages
                   ? p.block_tables[static_cast<int64_t>(iss_first) * p.max_blocks_per_seq +
                                    iss.tok0 / kBS + j]
                   : 0;
    }
    const int blk = __shfl_sync(kFull, bt_reg, iss_page & 31);
    if (lane == 0) {
      const int s = k_iss % kPNB;
      const int page = blk * p.num_kv_heads + iss.kvh;
      mbar_arrive_expect_tx(&bars[s], kPTx);
      uint8_t* tk = tiles + s * 2 * kPageBytes;
      tma_load_3d(tk, &tmk, 0, 0, page, &bars[s]);
      tma_load_3d(tk + kPageBytes, &tmv, 0, 0, page, &bars[s]);
      float* sc = scl + s * 2 * kBS;
      bulk_g2s(sc, p.k_scales + static_cast<int64_t>(page) * kBS,
               kBS * sizeof(float), &bars[s]);
      bulk_g2s(sc + kBS, p.v_scales + static_cast<int64_t>(page) * kBS,
               kBS * sizeof(float), &bars[s]);
    }
    ++k_iss;
    if (++iss_page == iss.npages) {
      iss_idx += stride;
      iss_seek();
    }
  };
  if (warp == 0) {
    iss_seek();
    for (int s = 0; s < kPNB; ++s) issue_one();
  }

  MmaMath<G, true> math;
  math.attach(nullptr);
  uint32_t k = 0;  // pages consumed by this CTA
  for (int64_t idx = blockIdx.x; idx < n_items; idx += stride) {
    PrefixItem it;
    if (!pitem_load(p, ps, idx, it)) continue;
    int first, b_w, b_lead;
    find_members(p, it.g, 8 * it.rnd + warp, 8 * it.rnd, lane, first, b_w,
                 b_lead);
    if (b_lead < 0) continue;  // the same decision in every warp
    int n_w = 0;
    if (b_w >= 0) {
      n_w = p.context_lens[b_w];
      if (n_w < it.tok0 + p.chunk_tokens) {  // shorter than the prefix
        if (lane == 0) atomicOr(&g_prefix_status, KV8_DEV_BAD_PREFIX);
        b_w = -1;
      }
    }
    const int64_t row0 =
        static_cast<int64_t>(b_w < 0 ? 0 : b_w) * p.num_q_heads + it.kvh * G;
    if (b_w >= 0) math.init(p.q + row0 * kD, p.q_scale, lane);
    for (int j = 0; j < it.npages; ++j, ++k) {
      const int s = k % kPNB;
      pwait(&bars[s], (k / kPNB) & 1, k, fail);
      // V page -> fp16 [16 tok][128 dims]: warp w converts tokens 2w, 2w+1;
      // lane = (token, 16-byte code chunk, half)
      {
        const int t = 2 * warp + (lane >> 4);
        const int cj = (lane & 15) >> 1, hf = lane & 1;
        const uint8_t* src = tiles + s * 2 * kPageBytes + kPageBytes + t * 128 +
                             ((cj ^ (t & 7)) << 4) + 8 * hf;
        const uint2 w8 = *reinterpret_cast<const uint2*>(src);
        const uint32_t x0 = w8.x ^ 0x80808080u, x1 = w8.y ^ 0x80808080u;
        uint4 o;
        o.x = hsub2_u32(prmt(x0, 0x64646464u, 0x4140u), kBias1152);
        o.y = hsub2_u32(prmt(x0, 0x64646464u, 0x4342u), kBias1152);
        o.z = hsub2_u32(prmt(x1, 0x64646464u, 0x4140u), kBias1152);
        o.w = hsub2_u32(prmt(x1, 0x64646464u, 0x4342u), kBias1152);
        const int ch = 2 * cj + hf;  // fp16 chunk: dims 8ch .. 8ch+7
        *reinterpret_cast<uint4*>(vh + (k & 1) * 4096 + t * 256 + ((ch ^ (t & 7)) << 4)) = o;
      }
      __syncthreads();
      // every warp is past page k-1: its slot is free for page k-1+kPNB
      if (warp == 0 && k >= 1) issue_one();
      if (b_w >= 0) {
        const uint8_t* tk = tiles + s * 2 * kPageBytes;
        const float* ks = scl + s * 2 * kBS;
        uint32_t h0, h2, g0, g2;
        math.template qk_softmax<true>(tk, ks, ks + kBS, kBS, h0, h2, g0, g2);
        math.pv_f16(smem_u32(vh + (k & 1) * 4096), h0, h2, g0, g2);
      }
    }
    if (b_w < 0) continue;
    // ---- this member's chunk: partial (or the output row), ticket, merge
    const int nchunks = (n_w + p.chunk_tokens - 1) / p.chunk_tokens;
    ChunkSink sk;
    sk.out = p.out;
    sk.ws_o = p.ws_o;
    sk.ws_ml = p.ws_ml;
    sk.row0 = row0;
    sk.ci0 = row0 * p.max_chunks + it.chunk;
    sk.max_chunks = p.max_chunks;
    sk.single = nchunks <= 1;
    sk.out_f32 = p.out_f32;
    math.finish(sk);
    if (!sk.single) {
      __threadfence();
      __syncwarp();
      unsigned int ticket = 0;
      if (lane == 0) ticket = atomicAdd(&p.ws_ctr[row0], 1u);
      ticket = __shfl_sync(kFull, ticket, 0);
      if (ticket == static_cast<unsigned int>(nchunks - 1)) {
        __threadfence();
        for (int h = 0; h < G; ++h)
          merge_head_warp(p.ws_ml + (row0 + h) * p.max_chunks * 2,
                          p.ws_o + (row0 + h) * p.max_chunks * kD, nchunks,
                          p.out, row0 + h, p.out_f32);
      }
    }
  }
  // a wait gave up: wait (bounded) for every copy that may still be in
  // flight (pages from the first one not waited for), then stop
  __syncthreads();
  if (fail[0] && warp == 0 && lane == 0) {
    for (uint32_t kk = static_cast<uint32_t>(fail[1]); kk < k_iss; ++kk)
      mbar_wait(&bars[kk % kPNB], (kk / kPNB) & 1, &g_prefix_status);
  }
}

template <int G>
int launch_prefix_group(const DecodeParams& p, const PrefixShape& ps,
                        const CUtensorMap& tmk, const CUtensorMap& tmv,
                        cudaStream_t stream) {
  auto kern = prefix_kernel<G>;
  constexpr int smem = PrefixPlan::kBytes;
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
  const int64_t n_items = static_cast<int64_t>(ps.prefix_chunks) *
                          p.num_kv_heads * ps.num_groups * ps.rounds;
  if (n_items == 0) return 0;
  int64_t ctas = sms;
  if (ctas > n_items) ctas = n_items;
  kern<<<static_cast<unsigned>(ctas), kPW * 32, smem, stream>>>(p, ps, tmk, tmv);
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
