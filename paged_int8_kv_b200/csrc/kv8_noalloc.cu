// kv8_noalloc.cu -- kv8_paged_decode_attention_noalloc: the split-K decode
// for callers that cannot allocate device memory.
//
// Who needs it: code that runs inside a host framework which owns all device
// memory (an inference server that reserves nearly the whole GPU up front for
// its KV pool, a plugin or custom op whose host gives it no workspace hook),
// and latency-critical paths where a cudaMalloc -- which can synchronise the
// device -- is not acceptable.  Such a caller cannot provide the split-K
// workspace that kv8_paged_decode_attention asks for.
//
// What it does instead: the chunk partials go to one fixed scratch array in
// this file, a static __device__ array of KV8_NOALLOC_WORKSPACE_BYTES that
// every GPU which loads the library holds until the process exits.  No call
// here allocates or frees memory.
//
// The array's name is only a host-side stand-in in host code.  Its device
// address is looked up once per device (cudaGetSymbolAddress, with that
// device current) by the first call made on that device, and handed to the
// kernels as a plain pointer.
//
// Sharing rules: every call uses the same array, which keeps whatever the
// last call left in it.  The chunk partials need no initial value (the split
// kernel writes every partial before the merge reads it); the merge tickets
// at the end of the array must start at zero, and the call clears them on
// its stream before its kernel, as the allocating entry point does with a
// caller's workspace.  Two calls whose kernels overlap on the GPU (for
// instance on two streams without ordering between them) race on both the
// partials and the tickets.
//
// The cached device address stays valid for the life of the CUDA context;
// a device reset after the first call on a device is not supported.
#include <mutex>

#include "../../include/kv8.h"
#include "kv8_internal.h"

namespace {

static __device__ __align__(256) unsigned char
    g_noalloc_scratch[KV8_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on
// first use).  Returns nullptr on a CUDA error.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess ||
        ptr == nullptr)
      return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int32_t kv8_paged_decode_attention_noalloc(
    const void* q, const int8_t* k_cache, const int8_t* v_cache,
    const float* k_scales, const float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void* out, int32_t out_dtype,
    void* stream) {
  // Same shape rules as kv8_paged_decode_attention; the workspace size check
  // is against the fixed array instead of a caller buffer.
  const size_t need = kv8_decode_workspace_bytes(
      batch, num_q_heads, head_dim, max_context_len, chunk_tokens);
  if (need > static_cast<size_t>(KV8_NOALLOC_WORKSPACE_BYTES))
    return KV8_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    ws = scratch_on_current_device();
    if (!ws) return KV8_ERR_CUDA;
  }
  // the array's real size: the allocating entry point checks it against its
  // own requirement too, so an oversized split is refused twice over
  return kv8_paged_decode_attention(
      q, k_cache, v_cache, k_scales, v_scales, block_tables, context_lens,
      batch, num_q_heads, num_kv_heads, head_dim, block_size,
      max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
      chunk_tokens, ws, ws ? static_cast<size_t>(KV8_NOALLOC_WORKSPACE_BYTES) : 0,
      out, out_dtype, stream);
}
