// kv8_check.cu -- debug checks of the device-resident indices the decode
// and append calls trust: context lengths, the block-table entries a decode
// reads, and slot-mapping entries.  Each check is its own small kernel that
// only reads the index arrays (within the bounds its arguments give) and
// counts what is out of range into a caller-owned device array; nothing else
// is read or written, so it can run on inputs that would make a decode read
// out of bounds.  Use: run it before a call while debugging, read the counts.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kv8.h"

namespace {

constexpr int kBlock = 16;  // tokens per block

// One CTA per sequence: counts[0] += context length outside
// [0, max_context_len]; counts[1] += block-table entries the decode would
// read (the first ceil(len / 16) of the row, len clamped to the row's
// capacity and to max_context_len) outside [0, num_blocks).
__global__ void __launch_bounds__(128)
check_decode_kernel(const int32_t* __restrict__ block_tables,
                    const int32_t* __restrict__ context_lens,
                    int32_t max_blocks_per_seq, int64_t num_blocks,
                    int32_t max_context_len, uint32_t* counts) {
  const int b = blockIdx.x;
  const int32_t len = context_lens[b];
  if (threadIdx.x == 0 && (len < 0 || len > max_context_len)) atomicAdd(&counts[0], 1u);
  int64_t n = len < 0 ? 0 : len;
  if (n > max_context_len) n = max_context_len;
  const int64_t cap = static_cast<int64_t>(max_blocks_per_seq) * kBlock;
  if (n > cap) n = cap;
  const int64_t pages = (n + kBlock - 1) / kBlock;
  const int32_t* row = block_tables + static_cast<int64_t>(b) * max_blocks_per_seq;
  uint32_t bad = 0;
  for (int64_t j = threadIdx.x; j < pages; j += blockDim.x) {
    const int32_t e = row[j];
    bad += (e < 0 || e >= num_blocks) ? 1u : 0u;
  }
  if (bad) atomicAdd(&counts[1], bad);
}

// counts[2] += slot-mapping entries at or past num_blocks * 16 (negative
// entries are padding and allowed).
__global__ void __launch_bounds__(256)
check_slots_kernel(const int64_t* __restrict__ slot_mapping, int64_t n_tokens,
                   int64_t num_slots, uint32_t* counts) {
  uint32_t bad = 0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
       i < n_tokens; i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    bad += slot_mapping[i] >= num_slots ? 1u : 0u;
  if (bad) atomicAdd(&counts[2], bad);
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

}  // namespace

extern "C" {

int32_t kv8_check_indices(const int32_t* block_tables,
                          const int32_t* context_lens, int32_t batch,
                          int32_t max_blocks_per_seq, int64_t num_blocks,
                          int32_t max_context_len, const int64_t* slot_mapping,
                          int64_t n_tokens, uint32_t* counts, void* stream) {
  if (batch < 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 ||
      max_context_len < 0 || n_tokens < 0 || !counts || !aligned4(counts))
    return KV8_ERR_INVALID_ARG;
  if (batch > 0 && (!block_tables || !context_lens || !aligned4(block_tables) ||
                    !aligned4(context_lens)))
    return KV8_ERR_INVALID_ARG;
  if (n_tokens > 0 && (!slot_mapping ||
                       (reinterpret_cast<uintptr_t>(slot_mapping) & 7) != 0))
    return KV8_ERR_INVALID_ARG;
  if (num_blocks > INT64_MAX / kBlock) return KV8_ERR_UNSUPPORTED;
  if (batch > INT32_MAX) return KV8_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(counts, 0, 3 * sizeof(uint32_t), st) != cudaSuccess)
    return KV8_ERR_CUDA;
  if (batch > 0)
    check_decode_kernel<<<static_cast<unsigned>(batch), 128, 0, st>>>(
        block_tables, context_lens, max_blocks_per_seq, num_blocks,
        max_context_len, counts);
  if (n_tokens > 0) {
    const int64_t blocks = (n_tokens + 255) / 256;
    check_slots_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, st>>>(
        slot_mapping, n_tokens, num_blocks * kBlock, counts);
  }
  return cudaGetLastError() == cudaSuccess ? KV8_OK : KV8_ERR_CUDA;
}

}  // extern "C"
