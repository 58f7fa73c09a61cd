// internal.h -- declarations shared by the library's translation units (not installed).
#pragma once

#include <cstddef>
#include <cstdint>
#include <map>
#include <mutex>
#include <vector>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "../../include/nvfp4kv.h"

namespace nvfp4kv {

constexpr int kHeadDim = 128;
constexpr int kBlock = 16;                    // elements per E4M3 block scale
constexpr int kCodeBytes = kHeadDim / 2;      // 64 bytes of E2M1 codes per token and head
constexpr int kScaleBytes = kHeadDim / kBlock;  // 8 E4M3 scale bytes per token and head
constexpr uint32_t kStatusTimeout = 1u << NVFP4KV_ERR_DEVICE_TIMEOUT;

// Bounded-wait limit for every in-kernel wait (nanoseconds of %globaltimer).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// Runs a set-up step once per device: CUDA keeps function attributes (dynamic shared-memory
// limit, cluster options) per device, so a process that uses several GPUs sets them on each.
// The result of the first run on a device is remembered and returned on later calls.
class PerDeviceOnce {
 public:
  template <class F>
  cudaError_t run(F&& fn) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu_);
    auto it = done_.find(dev);
    if (it != done_.end()) return it->second;
    e = fn();
    done_[dev] = e;
    return e;
  }

 private:
  std::mutex mu_;
  std::map<int, cudaError_t> done_;
};

// SM count of the current device, or -1 without a usable device.
int current_sm_count();

// ---- quantiser (quantize.cu)
// Number of amax partial slots per (b, h, tensor) and the workspace bytes they need.
int quantize_parts(int batch, int heads, int chunk_tokens);
size_t quantize_workspace_bytes(int batch, int heads, int chunk_tokens);
// Size of the fixed device array the no-workspace quantiser variant uses for its partials.
constexpr size_t kStaticScratchBytes = 64 * 1024;
// Device address of that array on the current device (looked up on first use per device).
cudaError_t static_scratch_address(void** out);
cudaError_t launch_quantize(const nvfp4kv_cache& c, int slot, const uint16_t* k, const uint16_t* v,
                            int64_t token_stride, void* workspace, cudaStream_t stream);
// The single-launch quantiser over several layers' caches of one shape (ticketed kernel): its
// counter workspace, its size limits, and the launch (a memset of the counters, then the kernel).
size_t quantize_layers_workspace_bytes(int layers, int batch, int heads);
bool quantize_layers_supported(int layers, int batch, int heads, int chunk_tokens);
cudaError_t launch_quantize_layers(const nvfp4kv_cache* caches, int layers, int slot, const uint16_t* const* k,
                                   const uint16_t* const* v, int64_t token_stride, void* workspace,
                                   cudaStream_t stream);
// Kernels launch_quantize launches for this cache shape on the current device (1 or 2).
int quantize_launches(const nvfp4kv_cache& c);

// ---- tensor maps (attention.cu): the driver's encoder, looked up once; null if unavailable.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// ---- attention (attention.cu)
constexpr int kAttnMaxRuns = 4;  // runs of consecutive visible chunk slots one attention call takes
// Workspace of the attention call on the current device (partial results of split work items).
size_t attention_workspace_bytes(const nvfp4kv_cache& c, int q_tokens);
// Number of runs of consecutive slots in an ascending, duplicate-free slot list.
int attention_runs(const std::vector<int>& vis);
// Whether the work split of a launch fits the 64-bit unit arithmetic of the planner.
bool attention_shape_supported(const nvfp4kv_cache& c, int q_tokens, int64_t kv_tiles);
// The attention launch's work split (see nvfp4kv_attention_plan in the public header).
int attention_plan(const nvfp4kv_cache& c, int q_tokens, int kv_tiles, int n_sms, int cta, int seg,
                   int out[8]);
// vis: the visible chunk slots, ascending and distinct, at most kAttnMaxRuns runs.
int launch_attention(const nvfp4kv_cache& c, const uint16_t* q, int q_tokens, int64_t q_stride,
                     const std::vector<int>& vis, float softmax_scale, void* out, int out_dtype,
                     void* workspace, size_t workspace_bytes, cudaStream_t stream);

// A kernel whose bounded wait runs out (nothing arrives at its barrier): the device-timeout path,
// for tests (attention.cu).
cudaError_t launch_wait_timeout_probe(uint32_t* status, cudaStream_t stream);

// ---- diagnostics (dequantize.cu)
cudaError_t launch_dequantize(const nvfp4kv_cache& c, int which, int first_slot, int n_slots,
                              float* out, cudaStream_t stream);
cudaError_t launch_encode_probe(const float* x, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                                cudaStream_t stream);

}  // namespace nvfp4kv
