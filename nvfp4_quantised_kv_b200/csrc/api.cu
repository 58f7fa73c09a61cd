// api.cu -- the C ABI of libnvfp4kv (declared in include/nvfp4kv.h): argument checks,
// workspace sizing and dispatch to the kernels.  No device memory is allocated here.
#include <cstdio>

#include <algorithm>
#include <vector>

#include "internal.h"

using namespace nvfp4kv;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape and pointer checks shared by every entry point that takes a cache.
int check_cache(const nvfp4kv_cache* c) {
  if (!c) return NVFP4KV_ERR_INVALID_ARG;
  if (c->batch <= 0 || c->heads <= 0 || c->head_dim <= 0 || c->chunk_tokens <= 0 ||
      c->capacity_chunks <= 0)
    return NVFP4KV_ERR_INVALID_ARG;
  if (c->batch > 65535 || c->heads > 65535) return NVFP4KV_ERR_INVALID_ARG;
  if (static_cast<int64_t>(c->chunk_tokens) * c->capacity_chunks > (int64_t(1) << 30))
    return NVFP4KV_ERR_INVALID_ARG;
  if (c->head_dim != kHeadDim || (c->chunk_tokens & 1)) return NVFP4KV_ERR_UNSUPPORTED;
  const void* ptrs[] = {c->k_codes, c->v_codes, c->k_scales, c->v_scales,
                        c->k_gscale, c->v_gscale, c->status};
  for (const void* p : ptrs)
    if (!p) return NVFP4KV_ERR_INVALID_ARG;
  const void* arrays[] = {c->k_codes, c->v_codes, c->k_scales, c->v_scales, c->k_gscale, c->v_gscale};
  for (const void* p : arrays)
    if (!aligned16(p)) return NVFP4KV_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(c->status) & 3u) return NVFP4KV_ERR_INVALID_ARG;
  if (c->flags & ~static_cast<uint32_t>(NVFP4KV_K_SMOOTH | NVFP4KV_V_ADAPTIVE_SCALE)) return NVFP4KV_ERR_INVALID_ARG;
  if ((c->flags & NVFP4KV_K_SMOOTH) && (!c->k_mean || !aligned16(c->k_mean))) return NVFP4KV_ERR_INVALID_ARG;
  // the channel-mean kernel's exact integer sums have headroom for 2^23 keys per chunk
  if ((c->flags & NVFP4KV_K_SMOOTH) && c->chunk_tokens > (1 << 23)) return NVFP4KV_ERR_UNSUPPORTED;
  return NVFP4KV_OK;
}

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4KV_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return NVFP4KV_ERR_CUDA;
  if (major != 10 || minor != 0) return NVFP4KV_ERR_UNSUPPORTED;
  return NVFP4KV_OK;
}

}  // namespace

namespace {

// Checks shared by the attention entry points, then the launch; vis is ascending and distinct.
int attention_checked(const nvfp4kv_cache* cache, const void* q_bf16, int32_t q_tokens,
                      int64_t q_token_stride, const std::vector<int>& vis, float softmax_scale,
                      void* out, int32_t out_dtype, void* workspace, size_t workspace_bytes,
                      void* cuda_stream) {
  if (!q_bf16 || !out || !aligned16(q_bf16) || !aligned16(out)) return NVFP4KV_ERR_INVALID_ARG;
  if (q_tokens <= 0 || q_tokens > (1 << 24)) return NVFP4KV_ERR_INVALID_ARG;
  if (q_token_stride < static_cast<int64_t>(cache->heads) * cache->head_dim || q_token_stride % 8 != 0)
    return NVFP4KV_ERR_INVALID_ARG;
  if (out_dtype != NVFP4KV_OUT_F32 && out_dtype != NVFP4KV_OUT_BF16) return NVFP4KV_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return NVFP4KV_ERR_INVALID_ARG;  // NaN
  if (vis.empty()) return NVFP4KV_ERR_INVALID_ARG;
  // smoothed keys: a 128-key tile may span at most two chunks (the kernel holds two mean terms)
  if ((cache->flags & NVFP4KV_K_SMOOTH) && cache->chunk_tokens < 128) return NVFP4KV_ERR_UNSUPPORTED;
  if (attention_runs(vis) > kAttnMaxRuns) return NVFP4KV_ERR_UNSUPPORTED;
  int64_t keys = 0;
  for (size_t i = 0; i < vis.size(); ++i) keys += cache->chunk_tokens;
  if (!attention_shape_supported(*cache, q_tokens, (keys + 127) / 128 + kAttnMaxRuns))
    return NVFP4KV_ERR_UNSUPPORTED;
  const int rc = check_device();
  if (rc != NVFP4KV_OK) return rc;
  // the workspace is sized for the current device (one partial-result pair per SM)
  const size_t need = attention_workspace_bytes(*cache, q_tokens);
  if (need > 0 && (!workspace || !aligned16(workspace) || workspace_bytes < need))
    return NVFP4KV_ERR_WORKSPACE;
  return launch_attention(*cache, static_cast<const uint16_t*>(q_bf16), q_tokens, q_token_stride, vis,
                          softmax_scale, out, out_dtype, workspace, workspace_bytes,
                          static_cast<cudaStream_t>(cuda_stream));
}

}  // namespace

extern "C" {

int nvfp4kv_cache_sizes(int32_t batch, int32_t heads, int32_t head_dim, int32_t chunk_tokens,
                        int32_t capacity_chunks, size_t* codes_bytes, size_t* scales_bytes,
                        size_t* gscale_bytes) {
  if (batch <= 0 || heads <= 0 || head_dim <= 0 || head_dim % kBlock != 0 || chunk_tokens <= 0 ||
      capacity_chunks <= 0)
    return NVFP4KV_ERR_INVALID_ARG;
  const size_t rows = static_cast<size_t>(batch) * heads * chunk_tokens * capacity_chunks;
  if (codes_bytes) *codes_bytes = rows * (head_dim / 2);
  if (scales_bytes) *scales_bytes = rows * (head_dim / kBlock);
  if (gscale_bytes) *gscale_bytes = static_cast<size_t>(batch) * heads * capacity_chunks * sizeof(float);
  return NVFP4KV_OK;
}

size_t nvfp4kv_workspace_bytes(const nvfp4kv_cache* cache, int32_t q_tokens) {
  if (check_cache(cache) != NVFP4KV_OK || q_tokens < 0) return 0;
  size_t q = quantize_workspace_bytes(cache->batch, cache->heads, cache->chunk_tokens);
  size_t a = attention_workspace_bytes(*cache, q_tokens);
  size_t w = q > a ? q : a;
  return w < 256 ? 256 : w;
}

int nvfp4_kv_quantize(const nvfp4kv_cache* cache, int32_t chunk_slot, const void* k_bf16,
                      const void* v_bf16, int64_t token_stride, void* workspace,
                      size_t workspace_bytes, void* cuda_stream) {
  int rc = check_cache(cache);
  if (rc != NVFP4KV_OK) return rc;
  if (chunk_slot < 0 || chunk_slot >= cache->capacity_chunks) return NVFP4KV_ERR_INVALID_ARG;
  if (!k_bf16 || !v_bf16 || !aligned16(k_bf16) || !aligned16(v_bf16)) return NVFP4KV_ERR_INVALID_ARG;
  if (token_stride < static_cast<int64_t>(cache->heads) * cache->head_dim || token_stride % 8 != 0)
    return NVFP4KV_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < quantize_workspace_bytes(cache->batch, cache->heads, cache->chunk_tokens))
    return NVFP4KV_ERR_WORKSPACE;
  rc = check_device();
  if (rc != NVFP4KV_OK) return rc;
  const cudaError_t e = launch_quantize(*cache, chunk_slot, static_cast<const uint16_t*>(k_bf16),
                                        static_cast<const uint16_t*>(v_bf16), token_stride,
                                        workspace, static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

size_t nvfp4kv_quantize_layers_workspace_bytes(const nvfp4kv_cache* caches, int32_t n_layers) {
  if (!caches || n_layers < 1 || n_layers > 64 || check_cache(&caches[0]) != NVFP4KV_OK) return 0;
  return quantize_layers_workspace_bytes(n_layers, caches[0].batch, caches[0].heads);
}

int nvfp4_kv_quantize_layers(const nvfp4kv_cache* caches, int32_t n_layers, int32_t chunk_slot,
                             const void* const* k_bf16, const void* const* v_bf16, int64_t token_stride,
                             void* workspace, size_t workspace_bytes, void* cuda_stream) {
  if (!caches || !k_bf16 || !v_bf16 || n_layers < 1) return NVFP4KV_ERR_INVALID_ARG;
  int rc = check_cache(&caches[0]);
  if (rc != NVFP4KV_OK) return rc;
  const nvfp4kv_cache& c0 = caches[0];
  if (!quantize_layers_supported(n_layers, c0.batch, c0.heads, c0.chunk_tokens)) return NVFP4KV_ERR_UNSUPPORTED;
  for (int32_t l = 0; l < n_layers; ++l) {
    const nvfp4kv_cache& c = caches[l];
    rc = check_cache(&c);
    if (rc != NVFP4KV_OK) return rc;
    if (c.batch != c0.batch || c.heads != c0.heads || c.chunk_tokens != c0.chunk_tokens ||
        c.capacity_chunks != c0.capacity_chunks)
      return NVFP4KV_ERR_INVALID_ARG;
    if (c.flags != 0) return NVFP4KV_ERR_UNSUPPORTED;  // recipe options: one layer at a time
    if (!k_bf16[l] || !v_bf16[l] || !aligned16(k_bf16[l]) || !aligned16(v_bf16[l])) return NVFP4KV_ERR_INVALID_ARG;
  }
  if (chunk_slot < 0 || chunk_slot >= c0.capacity_chunks) return NVFP4KV_ERR_INVALID_ARG;
  if (token_stride < static_cast<int64_t>(c0.heads) * c0.head_dim || token_stride % 8 != 0)
    return NVFP4KV_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < quantize_layers_workspace_bytes(n_layers, c0.batch, c0.heads))
    return NVFP4KV_ERR_WORKSPACE;
  rc = check_device();
  if (rc != NVFP4KV_OK) return rc;
  const cudaError_t e = launch_quantize_layers(caches, n_layers, chunk_slot,
                                               reinterpret_cast<const uint16_t* const*>(k_bf16),
                                               reinterpret_cast<const uint16_t* const*>(v_bf16), token_stride,
                                               workspace, static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

int nvfp4_kv_quantize_static_scratch(const nvfp4kv_cache* cache, int32_t chunk_slot,
                                     const void* k_bf16, const void* v_bf16, int64_t token_stride,
                                     void* cuda_stream) {
  int rc = check_cache(cache);
  if (rc != NVFP4KV_OK) return rc;
  if (chunk_slot < 0 || chunk_slot >= cache->capacity_chunks) return NVFP4KV_ERR_INVALID_ARG;
  if (!k_bf16 || !v_bf16 || !aligned16(k_bf16) || !aligned16(v_bf16)) return NVFP4KV_ERR_INVALID_ARG;
  if (token_stride < static_cast<int64_t>(cache->heads) * cache->head_dim || token_stride % 8 != 0)
    return NVFP4KV_ERR_INVALID_ARG;
  // The partials must fit the fixed array; larger caches have to use nvfp4_kv_quantize.
  if (quantize_workspace_bytes(cache->batch, cache->heads, cache->chunk_tokens) > kStaticScratchBytes)
    return NVFP4KV_ERR_WORKSPACE;
  rc = check_device();
  if (rc != NVFP4KV_OK) return rc;
  void* scratch = nullptr;
  if (static_scratch_address(&scratch) != cudaSuccess) return NVFP4KV_ERR_CUDA;
  const cudaError_t e = launch_quantize(*cache, chunk_slot, static_cast<const uint16_t*>(k_bf16),
                                        static_cast<const uint16_t*>(v_bf16), token_stride, scratch,
                                        static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

int nvfp4_kv_attention(const nvfp4kv_cache* cache, const void* q_bf16, int32_t q_tokens,
                       int64_t q_token_stride, int32_t q_chunk, int32_t n_sink_chunks,
                       int32_t window_chunks, float softmax_scale, void* out, int32_t out_dtype,
                       void* workspace, size_t workspace_bytes, void* cuda_stream) {
  int rc = check_cache(cache);
  if (rc != NVFP4KV_OK) return rc;
  if (q_chunk < 0 || q_chunk >= cache->capacity_chunks || n_sink_chunks < 0 || window_chunks < 1)
    return NVFP4KV_ERR_INVALID_ARG;
  // V(t) = {c < n_sink} U {t - window < c <= t}, each slot once, ascending.
  std::vector<int> vis;
  for (int ch = 0; ch < cache->capacity_chunks; ++ch)
    if (ch < n_sink_chunks || (ch > q_chunk - window_chunks && ch <= q_chunk)) vis.push_back(ch);
  return attention_checked(cache, q_bf16, q_tokens, q_token_stride, vis, softmax_scale, out, out_dtype,
                           workspace, workspace_bytes, cuda_stream);
}

int nvfp4_kv_attention_slots(const nvfp4kv_cache* cache, const void* q_bf16, int32_t q_tokens,
                             int64_t q_token_stride, const int32_t* slots, int32_t n_slots,
                             float softmax_scale, void* out, int32_t out_dtype, void* workspace,
                             size_t workspace_bytes, void* cuda_stream) {
  int rc = check_cache(cache);
  if (rc != NVFP4KV_OK) return rc;
  if (!slots || n_slots < 1) return NVFP4KV_ERR_INVALID_ARG;
  std::vector<int> vis;
  vis.reserve(static_cast<size_t>(n_slots));
  for (int32_t i = 0; i < n_slots; ++i) {
    if (slots[i] < 0 || slots[i] >= cache->capacity_chunks) return NVFP4KV_ERR_INVALID_ARG;
    vis.push_back(slots[i]);
  }
  std::sort(vis.begin(), vis.end());  // the union of the listed chunks, each once
  vis.erase(std::unique(vis.begin(), vis.end()), vis.end());
  return attention_checked(cache, q_bf16, q_tokens, q_token_stride, vis, softmax_scale, out, out_dtype,
                           workspace, workspace_bytes, cuda_stream);
}

int nvfp4_kv_attention_multishot(const nvfp4kv_cache* cache, const void* q_bf16, int32_t q_tokens,
                                 int64_t q_token_stride, int32_t q_chunk, int32_t n_sink_chunks,
                                 int32_t window_chunks, int32_t shot_start, int32_t shot_len,
                                 float softmax_scale, void* out, int32_t out_dtype, void* workspace,
                                 size_t workspace_bytes, void* cuda_stream) {
  int rc = check_cache(cache);
  if (rc != NVFP4KV_OK) return rc;
  if (q_chunk < 0 || q_chunk >= cache->capacity_chunks || n_sink_chunks < 0 || window_chunks < 1)
    return NVFP4KV_ERR_INVALID_ARG;
  // the shot's sink is history of the current shot: it ends at or before the query chunk
  if (shot_start < 0 || shot_len < 0 || static_cast<int64_t>(shot_start) + shot_len > q_chunk + 1)
    return NVFP4KV_ERR_INVALID_ARG;
  // K_eff = global sink U shot sink U window, each slot once, ascending.
  std::vector<int> vis;
  for (int ch = 0; ch < cache->capacity_chunks; ++ch) {
    const bool global_sink = ch < n_sink_chunks;
    const bool shot_sink = ch >= shot_start && ch < shot_start + shot_len;
    const bool window = ch > q_chunk - window_chunks && ch <= q_chunk;
    if (global_sink || shot_sink || window) vis.push_back(ch);
  }
  return attention_checked(cache, q_bf16, q_tokens, q_token_stride, vis, softmax_scale, out, out_dtype,
                           workspace, workspace_bytes, cuda_stream);
}

int nvfp4_kv_dequantize(const nvfp4kv_cache* cache, int32_t which, int32_t first_slot,
                        int32_t n_slots, float* out, void* cuda_stream) {
  int rc = check_cache(cache);
  if (rc != NVFP4KV_OK) return rc;
  if (which != 0 && which != 1) return NVFP4KV_ERR_INVALID_ARG;
  if (first_slot < 0 || n_slots <= 0 || first_slot + n_slots > cache->capacity_chunks)
    return NVFP4KV_ERR_INVALID_ARG;
  if (!out || !aligned16(out)) return NVFP4KV_ERR_INVALID_ARG;
  rc = check_device();
  if (rc != NVFP4KV_OK) return rc;
  const cudaError_t e =
      launch_dequantize(*cache, which, first_slot, n_slots, out, static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

int nvfp4kv_debug_encode(const float* x, int64_t n, uint8_t* e2m1_codes, uint8_t* e4m3_codes,
                         void* cuda_stream) {
  if (!x || !e2m1_codes || !e4m3_codes || n <= 0) return NVFP4KV_ERR_INVALID_ARG;
  const int rc = check_device();
  if (rc != NVFP4KV_OK) return rc;
  const cudaError_t e = launch_encode_probe(x, n, e2m1_codes, e4m3_codes,
                                            static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

int nvfp4kv_debug_wait_timeout(const nvfp4kv_cache* cache, void* cuda_stream) {
  const int rc = check_cache(cache);
  if (rc != NVFP4KV_OK) return rc;
  const int dc = check_device();
  if (dc != NVFP4KV_OK) return dc;
  return launch_wait_timeout_probe(cache->status, static_cast<cudaStream_t>(cuda_stream)) == cudaSuccess
             ? NVFP4KV_OK
             : NVFP4KV_ERR_CUDA;
}

int nvfp4kv_attention_plan(const nvfp4kv_cache* cache, int32_t q_tokens, int32_t kv_tiles, int32_t n_sms,
                           int32_t cta, int32_t seg, int32_t* out) {
  int rc = check_cache(cache);
  if (rc != NVFP4KV_OK) return rc;
  if (q_tokens <= 0 || q_tokens > (1 << 24) || kv_tiles <= 0 || !out) return NVFP4KV_ERR_INVALID_ARG;
  if (!attention_shape_supported(*cache, q_tokens, kv_tiles)) return NVFP4KV_ERR_UNSUPPORTED;
  if (n_sms <= 0) {
    n_sms = current_sm_count();
    if (n_sms <= 0) return NVFP4KV_ERR_CUDA;
  }
  int o[8];
  rc = attention_plan(*cache, q_tokens, kv_tiles, n_sms, cta, seg, o);
  for (int i = 0; i < 8; ++i) out[i] = o[i];
  return rc;
}

int nvfp4kv_quantize_launches(const nvfp4kv_cache* cache) {
  int rc = check_cache(cache);
  if (rc != NVFP4KV_OK) return -rc;
  rc = check_device();
  if (rc != NVFP4KV_OK) return -rc;
  return quantize_launches(*cache);
}

int nvfp4kv_read_status(const nvfp4kv_cache* cache, void* cuda_stream, uint32_t* out) {
  if (!cache || !cache->status || !out) return NVFP4KV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, cache->status, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return NVFP4KV_ERR_CUDA;
  if (cudaMemsetAsync(cache->status, 0, sizeof v, s) != cudaSuccess) return NVFP4KV_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4KV_ERR_CUDA;
  *out = v;
  return NVFP4KV_OK;
}

const char* nvfp4kv_strerror(int status) {
  switch (status) {
    case NVFP4KV_OK: return "ok";
    case NVFP4KV_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4KV_ERR_UNSUPPORTED: return "unsupported shape or device";
    case NVFP4KV_ERR_CUDA: return "CUDA call failed";
    case NVFP4KV_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out";
    case NVFP4KV_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

}  // extern "C"
