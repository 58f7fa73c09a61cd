// dequantize.cu -- the NVFP4 dequantisation step on its own (diagnostics and tests) and a
// probe of the device's fp32 -> E2M1 / E4M3 conversions.
//
// Dequantisation follows the "LongLive-2.0" reading note, "The NVFP4 quantization format":
// x_hat = (E2M1 element) * (E4M3 block scale) * (FP32 scale).  The first product is formed
// exactly in 16-bit floating point with the same helpers the attention kernel uses for its
// in-shared-memory dequantisation (exact code * scale products), then multiplied by the FP32
// scale with a single fp32 rounding.  (Both 16-bit forms hold the product exactly; the attention
// kernel stages K and V as fp16.)
#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4kv {
namespace {

__global__ void dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                               const float* __restrict__ gscale, const float* __restrict__ kmean, int BH,
                               int Lc, int C, int first_slot, int n_slots, int as_bf16,
                               float* __restrict__ out) {
  const int64_t span = static_cast<int64_t>(n_slots) * Lc;
  const int64_t total = static_cast<int64_t>(BH) * span * 16;
  const int64_t T = static_cast<int64_t>(C) * Lc;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c16 = static_cast<int>(idx & 15);
    const int64_t rest = idx >> 4;
    const int64_t tt = rest % span;
    const int64_t bh = rest / span;
    const int64_t t = static_cast<int64_t>(first_slot) * Lc + tt;
    const int64_t row = bh * T + t;
    const uint32_t w = *reinterpret_cast<const uint32_t*>(codes + row * kCodeBytes + c16 * 4);
    const uint32_t sb = scales[row * kScaleBytes + (c16 >> 1)];
    const float g = gscale[bh * C + t / Lc];
    uint32_t hv[4];
    ptx::e2m1x8_to_f16x8(w, hv);
    const uint32_t s2 = ptx::e4m3_to_f16x2_bcast(sb);
    float o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t p = ptx::hmul2_u32(hv[i], s2);
      float lo, hi;
      if (as_bf16) {
        const uint32_t bb = ptx::f16x2_to_bf16x2(p);
        lo = __uint_as_float(bb << 16);
        hi = __uint_as_float(bb & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&p));
        lo = f.x;
        hi = f.y;
      }
      o[2 * i] = __fmul_rn(lo, g);
      o[2 * i + 1] = __fmul_rn(hi, g);
    }
    if (kmean) {  // a smoothed key: x_hat' + mu of its chunk
      const float* mu = kmean + (bh * C + t / Lc) * kHeadDim + c16 * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = __fadd_rn(o[i], mu[i]);
    }
    float4* dst = reinterpret_cast<float4*>(out + (bh * span + tt) * kHeadDim + c16 * 8);
    dst[0] = make_float4(o[0], o[1], o[2], o[3]);
    dst[1] = make_float4(o[4], o[5], o[6], o[7]);
  }
}

__global__ void encode_probe_kernel(const float* __restrict__ x, int64_t n,
                                    uint8_t* __restrict__ e2m1, uint8_t* __restrict__ e4m3) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = x[i];
    const float y[8] = {v, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    e2m1[i] = static_cast<uint8_t>(ptx::f32x8_to_e2m1x8(y) & 0xF);
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    e4m3[i] = static_cast<uint8_t>(r & 0xFF);
  }
}

}  // namespace

cudaError_t launch_dequantize(const nvfp4kv_cache& c, int which, int first_slot, int n_slots,
                              float* out, cudaStream_t stream) {
  const bool is_k = which == 0;
  const int BH = c.batch * c.heads;
  const int64_t total = static_cast<int64_t>(BH) * n_slots * c.chunk_tokens * 16;
  const int sms = current_sm_count();
  int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 16 * static_cast<int64_t>(sms > 0 ? sms : 1)));
  if (blocks < 1) blocks = 1;
  dequant_kernel<<<blocks, 256, 0, stream>>>(is_k ? c.k_codes : c.v_codes,
                                             is_k ? c.k_scales : c.v_scales,
                                             is_k ? c.k_gscale : c.v_gscale,
                                             is_k && (c.flags & NVFP4KV_K_SMOOTH) ? c.k_mean : nullptr, BH,
                                             c.chunk_tokens,
                                             c.capacity_chunks, first_slot, n_slots, is_k ? 1 : 0,
                                             out);
  return cudaGetLastError();
}

cudaError_t launch_encode_probe(const float* x, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                                cudaStream_t stream) {
  const int sms = current_sm_count();
  int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, 32 * static_cast<int64_t>(sms > 0 ? sms : 1)));
  if (blocks < 1) blocks = 1;
  encode_probe_kernel<<<blocks, 256, 0, stream>>>(x, n, e2m1, e4m3);
  return cudaGetLastError();
}

}  // namespace nvfp4kv
