// quantize.cu -- NVFP4 quantisation of a new frame chunk's K and V into a cache slot.
//
// Method: "LongLive-2.0" reading note (yingwang.github.io), "The inference infrastructure"
// (K and V re-quantised to NVFP4 at frame-chunk granularity) and "The NVFP4 quantization
// format" (FP32 scale, E4M3 scale per 16 elements, E2M1 elements); constants 16 / 448 / 6
// from the paper page, section 2.2 "NVFP4 Training".  The per-(chunk, head) FP32 scale
// needs the chunk maximum before any element can be encoded, so the work is two
// memory-bound passes over the bf16 input:
//   pass 1 (amax_kernel)     every CTA reduces a token range of one (b, h, tensor) to
//                            max|x| and writes it to a workspace slot (no atomics, no
//                            zero-fill, deterministic);
//   pass 2 (quantize_kernel) every CTA folds the partial maxima of its (b, h, tensor) into
//                            g, then encodes its token range: two lanes per 16-element
//                            block, 16-byte loads, a shuffle for the block maximum, hardware
//                            RNE/satfinite conversions to E4M3 and E2M1, 4-byte code stores
//                            that are contiguous across the warp.
// The second pass re-reads its input right after the first, from L2 for chunks that fit.
// Every fp32 step uses an explicitly rounded intrinsic (no contraction, no flush to zero),
// so the codes are bit-identical to the fp32 definition of the method.
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4kv {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTargetCtas = 148 * 4;  // four CTAs per SM in flight on a B200

struct QuantArgs {
  const uint16_t* x[2];  // K, V (bf16 bits)
  uint8_t* codes[2];
  uint8_t* scales[2];
  float* gscale[2];
  uint32_t* partial;  // [2][B*H][parts], bf16 bit pattern of a partial max|x|
  int64_t token_stride;
  int64_t T;  // tokens per (b, h) in the cache
  int B, H, L, C, slot, parts, tokens_per_part;
};

__device__ __forceinline__ uint4 ld_row16(const uint16_t* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t absmax_bits(uint4 w) {
  uint32_t m = __vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, w.z & 0x7FFF7FFFu);
  m = __vmaxu2(m, w.w & 0x7FFF7FFFu);
  return m;
}

__global__ void __launch_bounds__(kThreads) amax_kernel(const __grid_constant__ QuantArgs a) {
  const int part = blockIdx.x, bh = blockIdx.y, tensor = blockIdx.z;
  const int b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_begin = part * a.tokens_per_part;
  const int t_end = min(a.L, t_begin + a.tokens_per_part);
  const uint16_t* x = a.x[tensor] + static_cast<int64_t>(b) * a.L * a.token_stride +
                      static_cast<int64_t>(h) * kHeadDim + (lane & 15) * 8;
  uint32_t acc = 0;
  constexpr int kUnroll = 4;
  for (int t0 = t_begin + 2 * warp; t0 < t_end; t0 += 2 * kWarps * kUnroll) {
    uint4 w[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = t0 + 2 * kWarps * u + (lane >> 4);
      w[u] = (t < t_end) ? ld_row16(x + t * a.token_stride) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) acc = __vmaxu2(acc, absmax_bits(w[u]));
  }
  uint32_t m = max(acc & 0xFFFFu, acc >> 16);
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t red[kWarps];
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) r = max(r, red[i]);
    a.partial[(static_cast<int64_t>(tensor) * a.B * a.H + bh) * a.parts + part] = r;
  }
}

__global__ void __launch_bounds__(kThreads) quantize_kernel(const __grid_constant__ QuantArgs a) {
  const int part = blockIdx.x, bh = blockIdx.y, tensor = blockIdx.z;
  const int b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // FP32 scale of this (chunk, head, tensor): g = max|x| / (448 * 6).
  __shared__ float s_g;
  if (warp == 0) {
    const uint32_t* p = a.partial + (static_cast<int64_t>(tensor) * a.B * a.H + bh) * a.parts;
    uint32_t m = 0;
    for (int i = lane; i < a.parts; i += 32) m = max(m, p[i]);
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (lane == 0) {
      const float A = __uint_as_float(m << 16);
      const float g = (A == 0.0f) ? 0.0f : __fdiv_rn(A, 2688.0f);
      s_g = g;
      if (part == 0) a.gscale[tensor][static_cast<int64_t>(bh) * a.C + a.slot] = g;
    }
  }
  __syncthreads();
  const float g = s_g;
  const float denom = __fmul_rn(6.0f, g);

  const int t_begin = part * a.tokens_per_part;
  const int t_end = min(a.L, t_begin + a.tokens_per_part);
  const uint16_t* x = a.x[tensor] + static_cast<int64_t>(b) * a.L * a.token_stride +
                      static_cast<int64_t>(h) * kHeadDim + (lane & 15) * 8;
  const int64_t row0 = static_cast<int64_t>(bh) * a.T + static_cast<int64_t>(a.slot) * a.L;
  uint8_t* codes = a.codes[tensor] + row0 * kCodeBytes + (lane & 15) * 4;
  uint8_t* scales = a.scales[tensor] + row0 * kScaleBytes + ((lane & 15) >> 1);

  // Warp-uniform trip count: lanes 0-15 take the even token of a pair, 16-31 the odd one.
  for (int t0 = t_begin + 2 * warp; t0 < t_end; t0 += 2 * kWarps) {
    const int t = t0 + (lane >> 4);
    const bool valid = t < t_end;
    const uint4 w = valid ? ld_row16(x + t * a.token_stride) : make_uint4(0, 0, 0, 0);
    uint32_t mb = absmax_bits(w);
    mb = max(mb & 0xFFFFu, mb >> 16);
    mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 1));  // the two lanes of one 16-element block
    const float ab = __uint_as_float(mb << 16);

    uint32_t s_code = 0;
    if (ab != 0.0f && g != 0.0f) s_code = ptx::f32_to_e4m3(__fdiv_rn(ab, denom));
    const float s = ptx::e4m3_to_f32(s_code);
    uint32_t q = 0;
    if (s != 0.0f) {
      const float r = __frcp_rn(__fmul_rn(s, g));
      if (r != __int_as_float(0x7F800000)) {  // 1/(s*g) overflowed: the block stays zero
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
        float y[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          y[2 * i] = __fmul_rn(__uint_as_float(wv[i] << 16), r);
          y[2 * i + 1] = __fmul_rn(__uint_as_float(wv[i] & 0xFFFF0000u), r);
        }
        q = ptx::f32x8_to_e2m1x8(y);
      }
    }
    if (valid) {
      *reinterpret_cast<uint32_t*>(codes + static_cast<int64_t>(t) * kCodeBytes) = q;
      if ((lane & 1) == 0) scales[static_cast<int64_t>(t) * kScaleBytes] = static_cast<uint8_t>(s_code);
    }
  }
}

}  // namespace

int quantize_parts(int batch, int heads, int chunk_tokens) {
  const int units = 2 * batch * heads;
  int parts = (kTargetCtas + units - 1) / units;
  const int max_parts = (chunk_tokens + 15) / 16;  // at least 16 tokens per CTA
  if (parts > max_parts) parts = max_parts;
  if (parts < 1) parts = 1;
  int tpp = (chunk_tokens + parts - 1) / parts;
  tpp = (tpp + 1) & ~1;
  return (chunk_tokens + tpp - 1) / tpp;
}

size_t quantize_workspace_bytes(int batch, int heads, int chunk_tokens) {
  return static_cast<size_t>(2) * batch * heads * quantize_parts(batch, heads, chunk_tokens) *
         sizeof(uint32_t);
}

cudaError_t launch_quantize(const nvfp4kv_cache& c, int slot, const uint16_t* k, const uint16_t* v,
                            int64_t token_stride, void* workspace, cudaStream_t stream) {
  QuantArgs a;
  a.x[0] = k;
  a.x[1] = v;
  a.codes[0] = c.k_codes;
  a.codes[1] = c.v_codes;
  a.scales[0] = c.k_scales;
  a.scales[1] = c.v_scales;
  a.gscale[0] = c.k_gscale;
  a.gscale[1] = c.v_gscale;
  a.partial = static_cast<uint32_t*>(workspace);
  a.token_stride = token_stride;
  a.T = static_cast<int64_t>(c.capacity_chunks) * c.chunk_tokens;
  a.B = c.batch;
  a.H = c.heads;
  a.L = c.chunk_tokens;
  a.C = c.capacity_chunks;
  a.slot = slot;
  a.parts = quantize_parts(c.batch, c.heads, c.chunk_tokens);
  int tpp = (c.chunk_tokens + a.parts - 1) / a.parts;
  a.tokens_per_part = (tpp + 1) & ~1;
  const dim3 grid(a.parts, c.batch * c.heads, 2);
  amax_kernel<<<grid, kThreads, 0, stream>>>(a);
  quantize_kernel<<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// Quantiser variant for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code that runs
// inside a pre-planned memory arena whose size was fixed before this library was linked,
// plugins whose host framework owns every device allocation, and real-time loops where an
// allocation could block or fragment the heap.  For them the amax partials live in this
// file-scope array instead of a caller workspace.  Every GPU that loads the library keeps
// the array (kStaticScratchBytes) until the process exits.  Each call overwrites all the
// partials it reads, so nothing has to start at zero; all calls share the one array, so
// calls that may overlap on the GPU (different streams without ordering) race on it.
static __device__ __align__(256) uint32_t g_quant_scratch[kStaticScratchBytes / sizeof(uint32_t)];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
}  // namespace

cudaError_t static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    // Host code only holds a stand-in for the array's name; its device address has to be
    // looked up once per device, with that device current.
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_quant_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace nvfp4kv

