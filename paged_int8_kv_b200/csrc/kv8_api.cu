// kv8_api.cu -- the extern "C" entry points of libkv8 (declared, with their
// contracts, in include/kv8.h): host-side argument checks, tensor-map
// encoding for the TMA page copies, and kernel launches.
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "../../include/kv8.h"
#include "kv8_internal.h"
#include "kv8_test_hooks.h"

namespace {

using kv8::kBlockSize;
using kv8::kHeadDim;

bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool aligned4(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 3u) == 0;
}

bool group_supported(int32_t g) { return g == 1 || g == 2 || g == 4 || g == 8; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr,
                                cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Tensor map over a code cache viewed as [num_blocks*H_kv pages][rows]
// [128 bytes]: one box is one page, written to shared memory with the
// 128-byte swizzle (16-byte chunk j of row r lands at chunk j ^ (r & 7)).
// INT8 codes: 16 rows, one token each.  Packed INT4 codes (64 bytes a
// token): 8 rows, tokens 2r and 2r+1 in row r.
bool encode_page_map(CUtensorMap* map, const void* cache, int64_t pages,
                     int bits = 8) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int rows = bits == 4 ? kBlockSize / 2 : kBlockSize;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim),
                        static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(pages)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim),
                           static_cast<cuuint64_t>(kHeadDim * rows)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kHeadDim),
                       static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                  const_cast<void*>(cache), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Effective split: chunk tokens and chunk count for a launch.
void split_shape(int32_t max_context_len, int32_t chunk_tokens,
                 int32_t* chunk_eff, int32_t* max_chunks) {
  if (chunk_tokens <= 0) {
    int32_t c = ((max_context_len + kBlockSize - 1) / kBlockSize) * kBlockSize;
    *chunk_eff = c < kBlockSize ? kBlockSize : c;
    *max_chunks = 1;
  } else {
    *chunk_eff = chunk_tokens;
    int32_t mc = (max_context_len + chunk_tokens - 1) / chunk_tokens;
    *max_chunks = mc < 1 ? 1 : mc;
  }
}

// Everything a decode launch needs, from the arguments of an entry point.
struct DecodeSetup {
  kv8::DecodeParams p;
  CUtensorMap tmk, tmv;
  bool nothing = false;  // batch == 0: checked, nothing to launch
};

// The argument checks and parameter set-up shared by the decode entry
// points.  Returns a KV8 status; launches nothing.
int32_t prepare_decode(
    const void* q, const int8_t* k_cache, const int8_t* v_cache,
    const float* k_scales, const float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void* workspace,
    size_t workspace_bytes, void* out, int32_t out_dtype, DecodeSetup* d,
    bool partials_only = false, int bits = 8) {
  // ---- shape checks
  if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 ||
      max_context_len < 0 || chunk_tokens < 0)
    return KV8_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return KV8_ERR_INVALID_ARG;
  if (out_dtype != KV8_OUT_BF16 && out_dtype != KV8_OUT_F32)
    return KV8_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || block_size != kBlockSize)
    return KV8_ERR_UNSUPPORTED;
  if (!group_supported(num_q_heads / num_kv_heads)) return KV8_ERR_UNSUPPORTED;
  if (chunk_tokens % block_size != 0) return KV8_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_context_len) >
      static_cast<int64_t>(max_blocks_per_seq) * block_size)
    return KV8_ERR_INVALID_ARG;
  if (batch > 65535 || num_kv_heads > 65535) return KV8_ERR_UNSUPPORTED;
  if (num_blocks > INT32_MAX / num_kv_heads) return KV8_ERR_UNSUPPORTED;
  if (batch == 0) {
    d->nothing = true;
    return KV8_OK;
  }
  // ---- pointer checks
  if (!q || !k_cache || !v_cache || !k_scales || !v_scales || !block_tables ||
      !context_lens || !out)
    return KV8_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(k_scales) || !aligned16(v_scales) || !aligned4(block_tables) ||
      !aligned4(context_lens) || !aligned16(out))
    return KV8_ERR_INVALID_ARG;

  int32_t chunk_eff, max_chunks;
  split_shape(max_context_len, chunk_tokens, &chunk_eff, &max_chunks);
  if (static_cast<int64_t>(max_chunks) * num_kv_heads * batch > INT32_MAX)
    return KV8_ERR_UNSUPPORTED;
  float* ws_ml = nullptr;
  float* ws_o = nullptr;
  uint32_t* ws_ctr = nullptr;
  if (max_chunks > 1 || partials_only) {
    const size_t ml_bytes = kv8::workspace_ml_bytes(batch, num_q_heads, max_chunks);
    const size_t o_bytes = kv8::workspace_o_bytes(batch, num_q_heads, max_chunks);
    const size_t need =
        partials_only ? ml_bytes + o_bytes
                      : kv8::workspace_total_bytes(batch, num_q_heads, max_chunks);
    if (!workspace || workspace_bytes < need || !aligned16(workspace))
      return KV8_ERR_WORKSPACE;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    ws_ml = reinterpret_cast<float*>(base);
    ws_o = reinterpret_cast<float*>(base + ml_bytes);
    if (!partials_only)
      ws_ctr = reinterpret_cast<uint32_t*>(base + ml_bytes + o_bytes);
  }

  const int64_t pages = num_blocks * num_kv_heads;
  if (!encode_page_map(&d->tmk, k_cache, pages, bits) ||
      !encode_page_map(&d->tmv, v_cache, pages, bits))
    return KV8_ERR_CUDA;

  if (!(softmax_scale > 0.0f))
    softmax_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(head_dim)));
  kv8::DecodeParams& p = d->p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_scales = k_scales;
  p.v_scales = v_scales;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.ws_ml = ws_ml;
  p.ws_o = ws_o;
  p.ws_ctr = ws_ctr;
  p.out = out;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.chunk_tokens = chunk_eff;
  p.max_chunks = max_chunks;
  p.out_f32 = out_dtype == KV8_OUT_F32 ? 1 : 0;
  p.q_scale = static_cast<float>(static_cast<double>(softmax_scale) *
                                 1.4426950408889634074);  // log2(e)
  p.prefix_group = nullptr;
  p.prefix_lens = nullptr;
  p.partials_only = partials_only ? 1 : 0;
  p.kv_sub_shift = 0;
  p.k_new = nullptr;
  p.v_new = nullptr;
  p.k_cache_w = nullptr;
  p.v_cache_w = nullptr;
  p.k_scales_w = nullptr;
  p.v_scales_w = nullptr;
  p.work_ctr = ws_ctr ? ws_ctr + static_cast<size_t>(batch) * num_q_heads : nullptr;
  return KV8_OK;
}

// Zero the merge tickets of a split launch on `st` (nothing when unsplit).
bool clear_tickets(const DecodeSetup& d, int32_t batch, int32_t num_q_heads,
                   cudaStream_t st) {
  return !d.p.ws_ctr ||
         cudaMemsetAsync(d.p.ws_ctr, 0,
                         kv8::workspace_ctr_bytes(batch, num_q_heads),
                         st) == cudaSuccess;
}

}  // namespace

extern "C" {

const char* kv8_status_string(int32_t status) {
  switch (status) {
    case KV8_OK: return "KV8_OK";
    case KV8_ERR_INVALID_ARG: return "KV8_ERR_INVALID_ARG";
    case KV8_ERR_UNSUPPORTED: return "KV8_ERR_UNSUPPORTED";
    case KV8_ERR_WORKSPACE: return "KV8_ERR_WORKSPACE";
    case KV8_ERR_CUDA: return "KV8_ERR_CUDA";
    default: return "KV8_ERR_UNKNOWN";
  }
}

int32_t kv8_quantize_append(const void* k_new, const void* v_new,
                            const int64_t* slot_mapping, int64_t n_tokens,
                            int32_t num_kv_heads, int32_t head_dim,
                            int32_t block_size, int64_t num_blocks,
                            int8_t* k_cache, int8_t* v_cache, float* k_scales,
                            float* v_scales, void* stream) {
  if (n_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0)
    return KV8_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || block_size != kBlockSize)
    return KV8_ERR_UNSUPPORTED;
  if (n_tokens == 0) return KV8_OK;
  if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache || !k_scales ||
      !v_scales)
    return KV8_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned4(k_scales) || !aligned4(v_scales) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return KV8_ERR_INVALID_ARG;
  if (n_tokens > (int64_t(1) << 40) / num_kv_heads) return KV8_ERR_UNSUPPORTED;
  int rc = kv8::launch_quantize_append(
      k_new, v_new, slot_mapping, n_tokens, num_kv_heads, k_cache, v_cache,
      k_scales, v_scales, static_cast<cudaStream_t>(stream));
  return rc == 0 ? KV8_OK : KV8_ERR_CUDA;
}

size_t kv8_decode_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                  int32_t head_dim, int32_t max_context_len,
                                  int32_t chunk_tokens) {
  if (batch <= 0 || num_q_heads <= 0 || head_dim != kHeadDim ||
      max_context_len <= 0 || chunk_tokens <= 0)
    return 0;
  int32_t chunk_eff, max_chunks;
  split_shape(max_context_len, chunk_tokens, &chunk_eff, &max_chunks);
  if (max_chunks <= 1) return 0;
  return kv8::workspace_total_bytes(batch, num_q_heads, max_chunks);
}

int32_t kv8_decode_chunk_tokens(int32_t batch, int32_t num_kv_heads,
                                int32_t max_context_len) {
  if (batch <= 0 || num_kv_heads <= 0 || max_context_len <= 0) return 0;
  constexpr int32_t kMinChunk = 4 * kBlockSize, kMaxChunk = 32 * kBlockSize;
  constexpr int64_t kWarpsPerSM = 12;
  if (max_context_len <= kMinChunk) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
          cudaSuccess ||
      sms <= 0) {
    cudaGetLastError();  // no device here: clear the sticky error
    sms = 148;
  }
  // one item per resident warp: past that, a warp's per-item work (loading
  // q, writing and merging partials) costs more than the finer split saves
  const int64_t want_items = kWarpsPerSM * sms;
  const int64_t units = static_cast<int64_t>(batch) * num_kv_heads;
  const int64_t splits = (want_items + units - 1) / units;
  int64_t chunk = (max_context_len + splits - 1) / splits;
  chunk = (chunk + kBlockSize - 1) / kBlockSize * kBlockSize;
  if (chunk < kMinChunk) chunk = kMinChunk;
  if (chunk > kMaxChunk) {
    // equal chunks of at most kMaxChunk tokens
    const int64_t n = (max_context_len + kMaxChunk - 1) / kMaxChunk;
    chunk = (max_context_len + n - 1) / n;
    chunk = (chunk + kBlockSize - 1) / kBlockSize * kBlockSize;
  }
  return static_cast<int32_t>(chunk);
}

int32_t kv8_paged_decode_attention(
    const void* q, const int8_t* k_cache, const int8_t* v_cache,
    const float* k_scales, const float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void* workspace,
    size_t workspace_bytes, void* out, int32_t out_dtype, void* stream) {
  return kv8_paged_decode_attention_form(
      q, k_cache, v_cache, k_scales, v_scales, block_tables, context_lens,
      batch, num_q_heads, num_kv_heads, head_dim, block_size,
      max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
      chunk_tokens, workspace, workspace_bytes, out, out_dtype, KV8_FORM_AUTO,
      stream);
}

int32_t kv8_paged_decode_attention_form(
    const void* q, const int8_t* k_cache, const int8_t* v_cache,
    const float* k_scales, const float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void* workspace,
    size_t workspace_bytes, void* out, int32_t out_dtype, int32_t form,
    void* stream) {
  if (form < KV8_FORM_AUTO || form > KV8_FORM_MMA_I8) return KV8_ERR_INVALID_ARG;
  DecodeSetup d;
  const int32_t rc0 = prepare_decode(
      q, k_cache, v_cache, k_scales, v_scales, block_tables, context_lens,
      batch, num_q_heads, num_kv_heads, head_dim, block_size,
      max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
      chunk_tokens, workspace, workspace_bytes, out, out_dtype, &d);
  if (rc0 != KV8_OK || d.nothing) return rc0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!clear_tickets(d, batch, num_q_heads, st)) return KV8_ERR_CUDA;
  int rc = form == KV8_FORM_TCGEN05
               ? kv8::launch_decode_tc(d.p, d.tmk, d.tmv, st)
               : kv8::launch_decode(d.p, d.tmk, d.tmv, form, st);
  if (rc == -2) return KV8_ERR_UNSUPPORTED;
  if (rc != 0) return KV8_ERR_CUDA;
  return KV8_OK;
}

int32_t kv8_paged_decode_attention_append(
    const void* q, const void* k_new, const void* v_new, int8_t* k_cache,
    int8_t* v_cache, float* k_scales, float* v_scales,
    const int32_t* block_tables, const int32_t* context_lens, int32_t batch,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, float softmax_scale, int32_t chunk_tokens,
    void* workspace, size_t workspace_bytes, void* out, int32_t out_dtype,
    void* stream) {
  DecodeSetup d;
  const int32_t rc0 = prepare_decode(
      q, k_cache, v_cache, k_scales, v_scales, block_tables, context_lens,
      batch, num_q_heads, num_kv_heads, head_dim, block_size,
      max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
      chunk_tokens, workspace, workspace_bytes, out, out_dtype, &d);
  if (rc0 != KV8_OK || d.nothing) return rc0;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new))
    return KV8_ERR_INVALID_ARG;
  d.p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  d.p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  d.p.k_cache_w = k_cache;
  d.p.v_cache_w = v_cache;
  d.p.k_scales_w = k_scales;
  d.p.v_scales_w = v_scales;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!clear_tickets(d, batch, num_q_heads, st)) return KV8_ERR_CUDA;
  const int rc = kv8::launch_decode(d.p, d.tmk, d.tmv, KV8_FORM_AUTO, st);
  if (rc == -2) return KV8_ERR_UNSUPPORTED;
  if (rc != 0) return KV8_ERR_CUDA;
  return KV8_OK;
}

int32_t kv8_paged_decode_attention_prefix(
    const void* q, const int8_t* k_cache, const int8_t* v_cache,
    const float* k_scales, const float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    const int32_t* prefix_group, const int32_t* prefix_lens,
    int32_t num_groups, int32_t max_group_size, int32_t max_prefix_len,
    float softmax_scale, int32_t chunk_tokens, void* workspace,
    size_t workspace_bytes, void* out, int32_t out_dtype, void* stream) {
  if (num_groups < 0 || max_group_size < 0 || max_prefix_len < 0 ||
      chunk_tokens <= 0 || max_prefix_len > max_context_len)
    return KV8_ERR_INVALID_ARG;
  if (num_groups > 0 && (!prefix_group || !prefix_lens ||
                         !aligned4(prefix_group) || !aligned4(prefix_lens)))
    return KV8_ERR_INVALID_ARG;
  DecodeSetup d;
  const int32_t rc0 = prepare_decode(
      q, k_cache, v_cache, k_scales, v_scales, block_tables, context_lens,
      batch, num_q_heads, num_kv_heads, head_dim, block_size,
      max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
      chunk_tokens, workspace, workspace_bytes, out, out_dtype, &d);
  if (rc0 != KV8_OK || d.nothing) return rc0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!clear_tickets(d, batch, num_q_heads, st)) return KV8_ERR_CUDA;
  kv8::PrefixShape ps;
  ps.num_groups = num_groups;
  ps.max_group_size = max_group_size;
  ps.rounds = 0;
  ps.prefix_chunks = max_prefix_len / d.p.chunk_tokens;
  if (num_groups > 0 && max_group_size > 0 && ps.prefix_chunks > 0) {
    d.p.prefix_group = prefix_group;
    d.p.prefix_lens = prefix_lens;
    const int rc = kv8::launch_prefix(d.p, ps, d.tmk, d.tmv, st);
    if (rc == -2) return KV8_ERR_UNSUPPORTED;
    if (rc != 0) return KV8_ERR_CUDA;
  }
  const int rc = kv8::launch_decode(d.p, d.tmk, d.tmv, KV8_FORM_AUTO, st);
  if (rc == -2) return KV8_ERR_UNSUPPORTED;
  if (rc != 0) return KV8_ERR_CUDA;
  return KV8_OK;
}

int32_t kv8_paged_extend_attention(
    const void* q, const int8_t* k_cache, const int8_t* v_cache,
    const float* k_scales, const float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, const int32_t* q_start, int32_t batch,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_q_len, float softmax_scale, void* out, int32_t out_dtype,
    void* stream) {
  if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 ||
      max_q_len < 0)
    return KV8_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return KV8_ERR_INVALID_ARG;
  if (out_dtype != KV8_OUT_BF16 && out_dtype != KV8_OUT_F32)
    return KV8_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || block_size != kBlockSize)
    return KV8_ERR_UNSUPPORTED;
  if (!group_supported(num_q_heads / num_kv_heads)) return KV8_ERR_UNSUPPORTED;
  if (batch > 65535 || num_kv_heads > 65535) return KV8_ERR_UNSUPPORTED;
  if (num_blocks > INT32_MAX / num_kv_heads) return KV8_ERR_UNSUPPORTED;
  if (batch == 0 || max_q_len == 0) return KV8_OK;
  if (!q || !k_cache || !v_cache || !k_scales || !v_scales || !block_tables ||
      !context_lens || !q_start || !out)
    return KV8_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(k_scales) || !aligned16(v_scales) || !aligned4(block_tables) ||
      !aligned4(context_lens) || !aligned4(q_start) || !aligned16(out))
    return KV8_ERR_INVALID_ARG;
  CUtensorMap tmk, tmv;
  const int64_t pages = num_blocks * num_kv_heads;
  if (!encode_page_map(&tmk, k_cache, pages) ||
      !encode_page_map(&tmv, v_cache, pages))
    return KV8_ERR_CUDA;
  if (!(softmax_scale > 0.0f))
    softmax_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(head_dim)));
  const int rc = kv8::launch_extend(
      q, k_scales, v_scales, block_tables, context_lens, q_start, batch,
      num_q_heads, num_kv_heads, max_blocks_per_seq, max_q_len, softmax_scale,
      out, out_dtype == KV8_OUT_F32 ? 1 : 0, tmk, tmv,
      static_cast<cudaStream_t>(stream));
  if (rc == -2) return KV8_ERR_UNSUPPORTED;
  return rc == 0 ? KV8_OK : KV8_ERR_CUDA;
}

size_t kv8_decode_partials_bytes(int32_t batch, int32_t num_q_heads,
                                 int32_t head_dim, int32_t max_context_len,
                                 int32_t chunk_tokens) {
  if (batch <= 0 || num_q_heads <= 0 || head_dim != kHeadDim ||
      max_context_len < 0 || chunk_tokens <= 0 || chunk_tokens % kBlockSize)
    return 0;
  int32_t chunk_eff, max_chunks;
  split_shape(max_context_len, chunk_tokens, &chunk_eff, &max_chunks);
  return kv8::workspace_ml_bytes(batch, num_q_heads, max_chunks) +
         kv8::workspace_o_bytes(batch, num_q_heads, max_chunks);
}

int32_t kv8_paged_decode_attention_partials(
    const void* q, const int8_t* k_cache, const int8_t* v_cache,
    const float* k_scales, const float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void* partials,
    size_t partials_bytes, void* stream) {
  if (chunk_tokens <= 0) return KV8_ERR_INVALID_ARG;
  DecodeSetup d;
  const int32_t rc0 = prepare_decode(
      q, k_cache, v_cache, k_scales, v_scales, block_tables, context_lens,
      batch, num_q_heads, num_kv_heads, head_dim, block_size,
      max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
      chunk_tokens, partials, partials_bytes, partials /* unused out */,
      KV8_OUT_F32, &d, true);
  if (rc0 != KV8_OK || d.nothing) return rc0;
  const int rc = kv8::launch_decode(d.p, d.tmk, d.tmv, KV8_FORM_AUTO,
                                    static_cast<cudaStream_t>(stream));
  if (rc == -2) return KV8_ERR_UNSUPPORTED;
  return rc == 0 ? KV8_OK : KV8_ERR_CUDA;
}

int32_t kv8_merge_partials(const void* partials, size_t rank_stride,
                           int32_t ranks, int32_t batch, int32_t num_q_heads,
                           int32_t head_dim, int32_t max_context_len,
                           int32_t chunk_tokens, void* out, int32_t out_dtype,
                           void* stream) {
  if (ranks <= 0 || batch < 0 || num_q_heads <= 0 || max_context_len < 0 ||
      chunk_tokens <= 0)
    return KV8_ERR_INVALID_ARG;
  if (out_dtype != KV8_OUT_BF16 && out_dtype != KV8_OUT_F32)
    return KV8_ERR_INVALID_ARG;
  if (head_dim != kHeadDim) return KV8_ERR_UNSUPPORTED;
  if (chunk_tokens % kBlockSize != 0) return KV8_ERR_INVALID_ARG;
  if (batch == 0) return KV8_OK;
  const size_t one = kv8_decode_partials_bytes(batch, num_q_heads, head_dim,
                                               max_context_len, chunk_tokens);
  if (!partials || !out || !aligned16(partials) || !aligned16(out) ||
      (rank_stride & 15u))
    return KV8_ERR_INVALID_ARG;
  if (ranks > 1 && rank_stride < one) return KV8_ERR_INVALID_ARG;
  int32_t chunk_eff, max_chunks;
  split_shape(max_context_len, chunk_tokens, &chunk_eff, &max_chunks);
  const int rc = kv8::launch_merge_ranks(
      static_cast<const uint8_t*>(partials), rank_stride, ranks, batch,
      num_q_heads, max_chunks, out, out_dtype == KV8_OUT_F32 ? 1 : 0,
      static_cast<cudaStream_t>(stream));
  return rc == 0 ? KV8_OK : KV8_ERR_CUDA;
}

int32_t kv8_split_reduce(const void* workspace, size_t workspace_bytes,
                         const int32_t* context_lens, int32_t batch,
                         int32_t num_q_heads, int32_t head_dim,
                         int32_t max_context_len, int32_t chunk_tokens,
                         void* out, int32_t out_dtype, void* stream) {
  if (batch < 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
      chunk_tokens <= 0)
    return KV8_ERR_INVALID_ARG;
  if (out_dtype != KV8_OUT_BF16 && out_dtype != KV8_OUT_F32)
    return KV8_ERR_INVALID_ARG;
  if (head_dim != kHeadDim) return KV8_ERR_UNSUPPORTED;
  if (chunk_tokens % kBlockSize != 0) return KV8_ERR_INVALID_ARG;
  if (batch == 0) return KV8_OK;
  if (!context_lens || !out || !aligned16(out) || !aligned4(context_lens))
    return KV8_ERR_INVALID_ARG;
  int32_t chunk_eff, max_chunks;
  split_shape(max_context_len, chunk_tokens, &chunk_eff, &max_chunks);
  if (max_chunks <= 1) return KV8_OK;  // nothing was split
  const size_t need = kv8::workspace_total_bytes(batch, num_q_heads, max_chunks);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return KV8_ERR_WORKSPACE;
  const float* ws_ml = static_cast<const float*>(workspace);
  const float* ws_o = reinterpret_cast<const float*>(
      static_cast<const uint8_t*>(workspace) +
      kv8::workspace_ml_bytes(batch, num_q_heads, max_chunks));
  int rc = kv8::launch_split_reduce(
      ws_ml, ws_o, context_lens, batch, num_q_heads, chunk_eff, max_chunks, out,
      out_dtype == KV8_OUT_F32 ? 1 : 0, static_cast<cudaStream_t>(stream));
  return rc == 0 ? KV8_OK : KV8_ERR_CUDA;
}

#ifdef KV8_TEST_HOOKS
int32_t kv8_test_skip_first_copy(int32_t on) {
  return kv8::test_skip_first_copy(on != 0) == 0 ? KV8_OK : KV8_ERR_CUDA;
}
#endif

int32_t kv8_read_device_status(uint32_t* status, int32_t clear) {
  if (!status) return KV8_ERR_INVALID_ARG;
  return kv8::read_device_status(status, clear) == 0 ? KV8_OK : KV8_ERR_CUDA;
}

int32_t kv8_int4_quantize_append(const void* k_new, const void* v_new,
                                 const int64_t* slot_mapping, int64_t n_tokens,
                                 int32_t num_kv_heads, int32_t head_dim,
                                 int32_t block_size, int64_t num_blocks,
                                 uint8_t* k_cache, uint8_t* v_cache,
                                 float* k_scales, float* v_scales,
                                 void* stream) {
  if (n_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0)
    return KV8_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || block_size != kBlockSize)
    return KV8_ERR_UNSUPPORTED;
  if (n_tokens == 0) return KV8_OK;
  if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache || !k_scales ||
      !v_scales)
    return KV8_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned4(k_scales) || !aligned4(v_scales) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return KV8_ERR_INVALID_ARG;
  if (n_tokens > (int64_t(1) << 40) / num_kv_heads) return KV8_ERR_UNSUPPORTED;
  int rc = kv8::launch_quantize_append(
      k_new, v_new, slot_mapping, n_tokens, num_kv_heads,
      reinterpret_cast<int8_t*>(k_cache), reinterpret_cast<int8_t*>(v_cache),
      k_scales, v_scales, static_cast<cudaStream_t>(stream), 4);
  return rc == 0 ? KV8_OK : KV8_ERR_CUDA;
}

int32_t kv8_int4_paged_decode_attention(
    const void* q, const uint8_t* k_cache, const uint8_t* v_cache,
    const float* k_scales, const float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float softmax_scale, int32_t chunk_tokens, void* workspace,
    size_t workspace_bytes, void* out, int32_t out_dtype, void* stream) {
  DecodeSetup d;
  const int32_t rc0 = prepare_decode(
      q, reinterpret_cast<const int8_t*>(k_cache),
      reinterpret_cast<const int8_t*>(v_cache), k_scales, v_scales,
      block_tables, context_lens, batch, num_q_heads, num_kv_heads, head_dim,
      block_size, max_blocks_per_seq, num_blocks, max_context_len,
      softmax_scale, chunk_tokens, workspace, workspace_bytes, out, out_dtype,
      &d, false, 4);
  if (rc0 != KV8_OK || d.nothing) return rc0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!clear_tickets(d, batch, num_q_heads, st)) return KV8_ERR_CUDA;
  const int rc = kv8::launch_decode_int4(d.p, d.tmk, d.tmv, st);
  if (rc == -2) return KV8_ERR_UNSUPPORTED;
  if (rc != 0) return KV8_ERR_CUDA;
  return KV8_OK;
}

}  // extern "C"
