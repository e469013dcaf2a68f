// kv8_internal.h -- launchers shared between the kv8 translation units.
// Not part of the public ABI (include/kv8.h is).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace kv8 {

// Launch facts of one kernel on one device (resident CTAs per SM and the SM
// count), found by its first launch on that device, with that device
// current, after the kernel's attributes were set there.  Zero = not yet
// known.  Racing first launches compute the same values.
constexpr int kMaxDevices = 64;
struct LaunchFacts {
  std::atomic<int> resident{0};
  std::atomic<int> sms{0};
};

// The facts slot of the current device (nullptr on a CUDA error or a
// device ordinal beyond kMaxDevices).
inline LaunchFacts* facts_for_current_device(LaunchFacts (&table)[kMaxDevices]) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nullptr;
  return &table[dev];
}

// CTAs of a kernel that fit one SM of the current device at once, from
// the per-SM limits (shared memory, threads, registers, and the SM's 512
// tensor-memory columns when the kernel allocates tmem_cols of them per
// CTA).  The runtime's occupancy query is not used: it reports one CTA per
// SM for any kernel that allocates tensor memory.  Returns 0 on a CUDA
// error, else >= 1.
template <class Kernel>
int resident_ctas(Kernel kern, int threads, int dyn_smem, int tmem_cols) {
  int dev = 0, smem_sm = 0, smem_rsv = 0, thr_sm = 0, regs_sm = 0;
  cudaFuncAttributes fa;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaFuncGetAttributes(&fa, kern) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor,
                             dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_rsv, cudaDevAttrReservedSharedMemoryPerBlock,
                             dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor,
                             dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor,
                             dev) != cudaSuccess)
    return 0;
  const int warps = (threads + 31) / 32;
  const int warp_regs = ((fa.numRegs * 32 + 255) / 256) * 256;
  int r = smem_sm / (dyn_smem + static_cast<int>(fa.sharedSizeBytes) + smem_rsv);
  if (thr_sm / threads < r) r = thr_sm / threads;
  if (warp_regs > 0 && regs_sm / (warp_regs * warps) < r)
    r = regs_sm / (warp_regs * warps);
  if (tmem_cols > 0 && 512 / tmem_cols < r) r = 512 / tmem_cols;
  return r < 1 ? 1 : r;
}

constexpr int kHeadDim = 128;
constexpr int kBlockSize = 16;
constexpr int kPageBytes = kHeadDim * kBlockSize;  // 2048 code bytes

// Everything a decode launch needs besides the two tensor maps.
struct DecodeParams {
  const __nv_bfloat16* q;       // [B][Hq][128]
  const float* k_scales;        // [NB][Hkv][16]
  const float* v_scales;
  const int32_t* block_tables;  // [B][MBS]
  const int32_t* context_lens;  // [B]
  float* ws_ml;                 // [B][Hq][max_chunks][2] (m, l), base-2
  float* ws_o;                  // [B][Hq][max_chunks][128]
  uint32_t* ws_ctr;             // [B][Hq] tickets (index b*Hq + first head
                                // of the KV group), zero at launch
  uint32_t* work_ctr;           // items taken past the first wave, zero at
                                // launch (nullptr: static item order)
  void* out;                    // [B][Hq][128] bf16 or f32
  int32_t batch;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t max_blocks_per_seq;
  int32_t chunk_tokens;  // > 0, multiple of 16
  int32_t max_chunks;    // ceil(max_context_len / chunk_tokens)
  int32_t out_f32;       // 1 = fp32 output, 0 = bf16
  float q_scale;         // softmax_scale * log2(e)
  // shared prefixes (nullptr when the batch has none): sequence b belongs to
  // group prefix_group[b] (or none, -1), whose first
  // prefix_lens[g] / chunk_tokens whole chunks a prefix launch computes; a
  // decode launch then skips those chunks of b
  const int32_t* prefix_group;  // [B]
  const int32_t* prefix_lens;   // [num_groups]
  // 1: write the (m, l, o) partial of every chunk slot c < max_chunks of
  // every (sequence, query head), empty chunks as (-inf, 0, 0), and merge
  // nothing (the partials of several launches are merged afterwards)
  int32_t partials_only;
  // fused append (nullptr: none): before a sequence's last page is copied,
  // the warp that takes the sequence's last chunk quantises the step's new
  // token, k_new / v_new bf16 [B][H_kv][128] at position context_lens[b] - 1,
  // into the caches through these writable views of them
  // KV heads split into 2^kv_sub_shift sub-groups of query heads, each its
  // own item (num_kv_heads then counts the sub-groups; the page of item KV
  // index v is that of KV head v >> kv_sub_shift).  0: no split.
  int32_t kv_sub_shift;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  int8_t* k_cache_w;
  int8_t* v_cache_w;
  float* k_scales_w;
  float* v_scales_w;
};


// Extra launch facts of the shared-prefix kernel.
struct PrefixShape {
  int32_t num_groups;
  int32_t max_group_size;  // host bound on the members of a group
  int32_t rounds;          // set by launch_prefix: ceil(max_group_size /
                           // members per round)
  int32_t prefix_chunks;   // max over groups of prefix_lens / chunk_tokens
  int32_t chunks_per_item; // set by launch_prefix: whole prefix chunks a
                           // prefix-kernel item covers
};

// Workspace carve-up shared by the decode and reduce launchers.
size_t workspace_ml_bytes(int32_t batch, int32_t num_q_heads,
                          int32_t max_chunks);
size_t workspace_o_bytes(int32_t batch, int32_t num_q_heads,
                         int32_t max_chunks);
size_t workspace_ctr_bytes(int32_t batch, int32_t num_q_heads);
size_t workspace_total_bytes(int32_t batch, int32_t num_q_heads,
                             int32_t max_chunks);

// Merge of the chunk partials of several launches (one per rank of a
// context-parallel decode): rank r's partials, laid out as a workspace's
// (m, l) and o regions, start `rank_stride` bytes after rank r-1's.
int launch_merge_ranks(const uint8_t* partials, size_t rank_stride,
                       int32_t ranks, int32_t batch, int32_t num_q_heads,
                       int32_t max_chunks, void* out, int32_t out_f32,
                       cudaStream_t stream);

// bits = 8: int8 codes; bits = 4: the INT4 variant (excess-8 nibbles).
int launch_quantize_append(const void* k_new, const void* v_new,
                           const int64_t* slot_mapping, int64_t n_tokens,
                           int32_t num_kv_heads, int8_t* k_cache,
                           int8_t* v_cache, float* k_scales, float* v_scales,
                           cudaStream_t stream, int32_t bits = 8);

// Returns 0 on success, -1 on a CUDA error, -2 if the group size has no
// compiled kernel.
int launch_decode(const DecodeParams& p, const CUtensorMap& tmk,
                  const CUtensorMap& tmv, int32_t variant,
                  cudaStream_t stream);

// The INT4 cache (packed excess-8 nibbles, 1 KB pages): groups of 1, 2, 4.
// Same return codes as launch_decode.
int launch_decode_int4(const DecodeParams& p, const CUtensorMap& tmk,
                       const CUtensorMap& tmv, cudaStream_t stream);

int launch_split_reduce(const float* ws_ml, const float* ws_o,
                        const int32_t* context_lens, int32_t batch,
                        int32_t num_q_heads, int32_t chunk_tokens,
                        int32_t max_chunks, void* out, int32_t out_f32,
                        cudaStream_t stream);

// The shared-prefix chunks of a batch (kv8_prefix.cu): one CTA of 8 warps
// per (chunk, KV head, group, round of 8 members).  Same return codes as
// launch_decode.
int launch_prefix(const DecodeParams& p, const PrefixShape& ps,
                  const CUtensorMap& tmk, const CUtensorMap& tmv,
                  cudaStream_t stream);

// Sticky status word of the shared-prefix kernel (no synchronize).
int read_prefix_status(uint32_t* value, int clear);

// Extend (prefill) attention on tcgen05 (kv8_extend.cu).  Same return codes
// as launch_decode.
int launch_extend(const void* q, const float* k_scales, const float* v_scales,
                  const int32_t* block_tables, const int32_t* context_lens,
                  const int32_t* q_start, int32_t batch, int32_t num_q_heads,
                  int32_t num_kv_heads, int32_t max_blocks_per_seq,
                  int32_t max_q_len, float softmax_scale, void* out,
                  int32_t out_f32, const CUtensorMap& tmk,
                  const CUtensorMap& tmv, cudaStream_t stream);

// Sticky status word of the extend kernel (no synchronize).
int read_ext_status(uint32_t* value, int clear);

// Decode on the tcgen05 tensor cores (kv8_decode_tc.cu); same contract as
// launch_decode.
int launch_decode_tc(const DecodeParams& p, const CUtensorMap& tmk,
                     const CUtensorMap& tmv, cudaStream_t stream);

// Sticky status word of the tcgen05 decode kernel (no synchronize).
int read_tc_status(uint32_t* value, int clear);

// Reads (and optionally clears) the sticky device status words of every
// decode kernel after a device-wide synchronize, OR-ed together.  Returns 0,
// or -1 on a CUDA error.
int read_device_status(uint32_t* value, int clear);

#ifdef KV8_TEST_HOOKS
// Test-hook build only (see kv8_test_hooks.h).
int test_skip_first_copy(int on);
#endif

}  // namespace kv8
