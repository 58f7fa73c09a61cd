// quantize.cu -- NVFP4 quantisation of a new frame chunk's K and V into a cache slot.
//
// Method: "LongLive-2.0" reading note (yingwang.github.io), "The inference infrastructure"
// (K and V re-quantised to NVFP4 at frame-chunk granularity) and "The NVFP4 quantization
// format" (FP32 scale, E4M3 scale per 16 elements, E2M1 elements); constants 16 / 448 / 6
// from the paper page, section 2.2 "NVFP4 Training".  The per-(chunk, head) FP32 scale needs
// the chunk maximum before any element can be encoded.  Four paths, the same arithmetic (bit-
// identical codes): for one layer's chunk,
//   single pass (quantize_cluster_kernel), when one cluster per (b, h, tensor) fits the GPU in
//       one wave: the cluster's CTAs TMA their token rows into shared memory, reduce max|x|,
//       exchange the maxima through distributed shared memory, and encode from shared memory
//       (the input crosses HBM once);
//   two passes otherwise:
//       amax_kernel      every CTA reduces 128 tokens of one (b, h, tensor) to max|x| and writes
//                        it to a workspace slot (no atomics, no zero-fill, deterministic);
//       quantize_kernel  launched as a programmatic dependent of the amax grid: every CTA loads
//                        its 64 rows (from L2, where the first pass just read them), then waits
//                        for the amax grid, folds the partial maxima into g and encodes;
// for the new chunk of many layers at once, quantize_ticket_kernel (one launch, the input read from
// HBM once; see its own comment); and for caches with the recipe options (K-smoothing, adaptive
// {4, 6} block scales), key_mean_kernel + recipe_amax_kernel + recipe_encode_kernel.
// Encoding: two lanes per 16-element block, 16-byte loads, a shuffle for the block maximum,
// hardware RNE/satfinite conversions to E4M3 and E2M1, 4-byte code stores contiguous across the
// warp.  Every fp32 step is an explicitly rounded intrinsic (no contraction, no flush to zero),
// and the two shortcuts (a hoisted reciprocal with an exact FMA correction for the block-scale
// quotient, a per-code reciprocal table) reproduce the correctly rounded operations, so the codes
// are bit-identical to the fp32 definition of the method.
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4kv {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// Two-pass path: a CTA owns kPartTokens tokens of one (b, h, tensor); 16 threads read a 256-byte
// token row, so the CTA covers 16 rows per pass and issues all kPasses loads of every thread
// before it uses any (one memory latency per CTA).
constexpr int kPasses = 8;
constexpr int kPartTokens = (kThreads / 16) * kPasses;  // 128
// The encode pass holds fewer rows per CTA (it also keeps the encoder state): 64 tokens, so both
// grids run six CTAs per SM and more, smaller CTAs shorten the tail.
constexpr int kEncPasses = 4;
constexpr int kEncTokens = (kThreads / 16) * kEncPasses;  // 64

struct QuantArgs {
  const uint16_t* x[2];  // K, V (bf16 bits)
  uint8_t* codes[2];
  uint8_t* scales[2];
  float* gscale[2];
  uint32_t* partial;  // [2][B*H][parts], bf16 bit pattern of a partial max|x| (fp32 bits on the recipe path)
  const float* k_mean;  // recipe path with K-smoothing: the cache's k_mean, else null
  int64_t token_stride;
  int64_t T;  // tokens per (b, h) in the cache
  int B, H, L, C, slot, parts;
  uint32_t flags;  // recipe options (NVFP4KV_K_SMOOTH, NVFP4KV_V_ADAPTIVE_SCALE)
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

// Per-CTA encoder state for one (chunk, head, tensor).  The block-scale quotient a_b / (6 g) is
// the correctly rounded fp32 quotient: with y = RN(1 / d) and q = RN(a_b * y), the residual
// r = a_b - q d is exact in one FMA and RN(q + r y) = RN(a_b / d) (Markstein's correction
// theorem), valid while nothing underflows, i.e. for normal d and y and a_b >= 2^-100; smaller
// block maxima take the IEEE division.  rtab[c] = RN(1 / RN(s_c * g)) for every E4M3 code c of the
// block scale, or 0 where the block's codes are all zero (s_c = 0, or the reciprocal overflows).
struct Encoder {
  float g, d, y;
  bool fast;
};

__device__ __forceinline__ Encoder make_encoder(float g, float* rtab, int tid, int nthreads) {
  Encoder e;
  e.g = g;
  e.d = __fmul_rn(6.0f, g);
  e.y = g != 0.0f ? __frcp_rn(e.d) : 0.0f;
  e.fast = g != 0.0f && e.d >= 0x1p-126f && e.y >= 0x1p-126f && e.y < 0x1p127f;
  for (int c = tid; c < 128; c += nthreads) {
    const float s = ptx::e4m3_to_f32(static_cast<uint32_t>(c));
    float r = 0.0f;
    if (s != 0.0f && c != 0x7F) {
      r = __frcp_rn(__fmul_rn(s, g));
      if (r == __int_as_float(0x7F800000)) r = 0.0f;
    }
    rtab[c] = r;
  }
  return e;
}

// E4M3 code of the block scale s = RN_e4m3(a_b / (6 g)) for the block maximum a_b (0 when a_b or
// g is 0).
__device__ __forceinline__ uint32_t block_scale_code(float ab, const Encoder& e) {
  uint32_t s_code = 0;
  if (ab != 0.0f && e.g != 0.0f) {
    float q;
    if (e.fast && ab >= 0x1p-100f) {
      q = __fmul_rn(ab, e.y);
      const float r = __fmaf_rn(-q, e.d, ab);
      q = __fmaf_rn(r, e.y, q);
    } else {
      q = __fdiv_rn(ab, e.d);
    }
    s_code = ptx::f32_to_e4m3(q);
  }
  return s_code;
}

// E2M1 codes of 8 bf16 elements (one 16-byte word) times r, element 2j in the low nibble of
// byte j; 0 when r is 0.
__device__ __forceinline__ uint32_t codes8(uint4 w, float r) {
  if (r == 0.0f) return 0u;
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
  float y[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    y[2 * i] = __fmul_rn(__uint_as_float(wv[i] << 16), r);
    y[2 * i + 1] = __fmul_rn(__uint_as_float(wv[i] & 0xFFFF0000u), r);
  }
  return ptx::f32x8_to_e2m1x8(y);
}

// Encodes this lane's 8 elements of a 16-element block (its partner lane xor 1 holds the other 8)
// and stores the 4 code bytes and, from the even lane, the scale byte.
__device__ __forceinline__ void encode_store(uint4 w, const Encoder& e, const float* rtab, bool valid,
                                             uint8_t* code_dst, uint8_t* scale_dst, int lane) {
  uint32_t mb = absmax_bits(w);
  mb = max(mb & 0xFFFFu, mb >> 16);
  mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 1));
  const uint32_t s_code = block_scale_code(__uint_as_float(mb << 16), e);
  const uint32_t qc = codes8(w, rtab[s_code & 0x7F]);
  if (valid) {
    *reinterpret_cast<uint32_t*>(code_dst) = qc;
    if ((lane & 1) == 0) *scale_dst = static_cast<uint8_t>(s_code);
  }
}

__global__ void __launch_bounds__(kThreads, 6) amax_kernel(const __grid_constant__ QuantArgs a) {
  const int part = blockIdx.x, bh = blockIdx.y, tensor = blockIdx.z;
  const int b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the dependent encode grid may start loading its rows now; it waits for this grid's results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int t_begin = part * kPartTokens;
  const int t_end = min(a.L, t_begin + kPartTokens);
  const int sub = threadIdx.x >> 4;
  const uint16_t* x = a.x[tensor] + static_cast<int64_t>(b) * a.L * a.token_stride +
                      static_cast<int64_t>(h) * kHeadDim + (threadIdx.x & 15) * 8;
  uint4 w[kPasses];
#pragma unroll
  for (int u = 0; u < kPasses; ++u) {
    const int t = t_begin + u * (kThreads / 16) + sub;
    w[u] = t < t_end ? ld_row16(x + static_cast<int64_t>(t) * a.token_stride) : make_uint4(0, 0, 0, 0);
  }
  uint32_t acc = 0;
#pragma unroll
  for (int u = 0; u < kPasses; ++u) acc = __vmaxu2(acc, absmax_bits(w[u]));
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

__global__ void __launch_bounds__(kThreads, 6) quantize_kernel(const __grid_constant__ QuantArgs a) {
  const int part = blockIdx.x, bh = blockIdx.y, tensor = blockIdx.z;
  const int b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_begin = part * kEncTokens;
  const int t_end = min(a.L, t_begin + kEncTokens);
  const int sub = threadIdx.x >> 4;
  const uint16_t* x = a.x[tensor] + static_cast<int64_t>(b) * a.L * a.token_stride +
                      static_cast<int64_t>(h) * kHeadDim + (threadIdx.x & 15) * 8;
  // The rows do not depend on the amax grid: they are loaded (mostly from L2, where that grid
  // just read them) before waiting for its partial maxima.
  uint4 w[kEncPasses];
#pragma unroll
  for (int u = 0; u < kEncPasses; ++u) {
    const int t = t_begin + u * (kThreads / 16) + sub;
    w[u] = t < t_end ? ld_row16(x + static_cast<int64_t>(t) * a.token_stride) : make_uint4(0, 0, 0, 0);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

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
  __shared__ float rtab[128];
  __syncthreads();
  const Encoder enc = make_encoder(s_g, rtab, threadIdx.x, kThreads);
  __syncthreads();

  const int64_t row0 = static_cast<int64_t>(bh) * a.T + static_cast<int64_t>(a.slot) * a.L;
  uint8_t* codes = a.codes[tensor] + row0 * kCodeBytes + (lane & 15) * 4;
  uint8_t* scales = a.scales[tensor] + row0 * kScaleBytes + ((lane & 15) >> 1);
#pragma unroll
  for (int u = 0; u < kEncPasses; ++u) {
    const int t = t_begin + u * (kThreads / 16) + sub;
    encode_store(w[u], enc, rtab, t < t_end, codes + static_cast<int64_t>(t) * kCodeBytes,
                 scales + static_cast<int64_t>(t) * kScaleBytes, lane);
  }
}

// ---------------------------------------------------------------------------------------
// Recipe path, taken by caches with recipe options: K-smoothing of K and adaptive {4, 6}
// block-scale targets of V (reading note, "The inference infrastructure": both applied within
// each chunk; "Engineering details of NVFP4 training": candidate scale magnitudes {4, 6}).
//   key_mean_kernel       a cluster of CTAs per (32 channels, b, h): TMA brings 64-token slices
//                         of the chunk's keys into a ring in shared memory; eight warps add them, a
//                         lane per channel, exactly (an fp64 sum per slice where that is exact,
//                         integer bins otherwise); CTA 0 adds the cluster's bins and writes the
//                         exact mean rounded once to fp32 to the slot's k_mean.
//   recipe_amax_kernel    amax_kernel over x - mu for a smoothed K (fp32 magnitudes); the
//                         partials hold fp32 bit patterns for both tensors.
//   recipe_encode_kernel  quantize_kernel from x - mu for a smoothed K; for V with adaptive
//                         scales each block is encoded for both scale targets and keeps the one
//                         with the smaller fp64 squared error, ties keeping 6.
constexpr int kMeanTok = 64;    // tokens per ring stage
constexpr int kMeanCh = 32;     // channels per CTA (64 bytes of each token row)
constexpr int kMeanStages = 16;  // 16 x 4 KB in flight per CTA

struct MeanArgs {
  float* k_mean;
  uint32_t* status;
  int H, L, C, slot;
};

__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity) {
  uint64_t t0 = 0;
  int it = 0;
  while (!ptx::mbar_try_wait(bar, parity)) {
    const uint64_t now = ptx::globaltimer_ns();
    if (it++ == 0) t0 = now;
    if (now - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// fp32 nearest (ties to even) to S * 2^-133 / L for the exact signed integer S given as 32-bit
// digits d[0..n) (two's complement, d[n-1] holding the sign): the mean of L bf16 values whose
// sum is S units of 2^-133.  The magnitude is shifted into units of 2^-149 (the fp32 subnormal
// step), divided by L with its remainder, and rounded to 24 significant bits.
template <int n>
__device__ float exact_mean_to_f32(uint32_t (&d)[n], uint32_t L) {
  const bool neg = (d[n - 1] >> 31) != 0u;
  if (neg) {  // magnitude: two's complement negation
    uint32_t carry = 1u;
#pragma unroll
    for (int k = 0; k < n; ++k) {
      const uint64_t t = static_cast<uint64_t>(~d[k]) + carry;
      d[k] = static_cast<uint32_t>(t);
      carry = static_cast<uint32_t>(t >> 32);
    }
  }
  // times 2^16: units of 2^-149 (the top digit has room: |S| < 2^285 for L <= 2^23)
#pragma unroll
  for (int k = n - 1; k > 0; --k) d[k] = (d[k] << 16) | (d[k - 1] >> 16);
  d[0] <<= 16;
  // divided by L, most significant digit first
  uint64_t r = 0;
#pragma unroll
  for (int k = n - 1; k >= 0; --k) {
    const uint64_t cur = (r << 32) | d[k];
    d[k] = static_cast<uint32_t>(cur / L);
    r = cur % L;
  }
  int top = -1;  // highest non-zero digit of the quotient
#pragma unroll
  for (int k = 0; k < n; ++k)
    if (d[k] != 0u) top = k;
  if (top < 0 && r == 0) return 0.0f;
  const int nbits = top < 0 ? 0 : top * 32 + (32 - __clz(d[top]));  // bit length of the quotient
  auto bit = [&](int j) -> uint32_t {  // bit j of the quotient (j >= 0)
    uint32_t v = 0u;
#pragma unroll
    for (int k = 0; k < n; ++k)
      if (k == (j >> 5)) v = (d[k] >> (j & 31)) & 1u;
    return v;
  };
  double v;
  if (nbits <= 24) {  // below 2^-125: every whole number of 2^-149 up to 2^24 is an fp32 value
    const uint64_t q = (top < 0) ? 0u : (top == 0 ? d[0] : (static_cast<uint64_t>(d[1]) << 32) | d[0]);
    const bool up = 2 * r > L || (2 * r == L && (q & 1u));
    v = ldexp(static_cast<double>(q + (up ? 1u : 0u)), -149);
  } else {
    const int sh = nbits - 24;
    uint64_t mant = 0;
    for (int j = nbits - 1; j >= sh; --j) mant = (mant << 1) | bit(j);
    const bool guard = bit(sh - 1) != 0u;
    bool lower = r != 0;
    for (int j = sh - 2; j >= 0 && !lower; --j) lower = bit(j) != 0u;
    const bool up = guard && (lower || (mant & 1u));
    v = ldexp(static_cast<double>(mant + (up ? 1u : 0u)), sh - 149);
  }
  return __double2float_rn(neg ? -v : v);  // exact: at most 24 significant bits
}

// K-smoothing's channel means of one chunk: the exact mean of each channel's L bf16 keys, rounded
// once to fp32.  Every bf16 value is a whole number of 2^-133 (< 2^261 of them), so the sum is
// kept exactly as integers in nine 64-bit bins per channel, bin k counting units of 2^(32 k - 133):
// integer additions, so any order gives the same sum and the tokens are summed in parallel.
// A cluster of S CTAs per (32 channels, b, h), S chosen so the grid fills the SMs: CTA z of the
// cluster takes the 64-token slices z, z + S, ...; in each CTA a producer lane TMA-loads them
// (64 tokens x 32 channels) into a 16-stage ring and eight warps take the stages in turn, a lane
// per channel, each thread adding into bins of its own.  The bins are then summed over the warps,
// and CTA 0 adds the other CTAs' sums through distributed shared memory (integer additions, so
// the split changes no bit).
// A lane first sums its 64 values of a stage in fp64.  When the stage's non-zero magnitudes span
// at most 40 binades (2^(pos_hi - pos_lo) <= 2^39) every partial sum is a whole number of
// 2^(pos_lo - 133) below 2^(8 + 39 + 6) = 2^53, so fp64 holds each one exactly, in any order; the
// exact stage sum then goes into three bins as 32-bit pieces.  Other stages (a wider span, or an
// Inf/NaN bit pattern, which the bins read as the number its bits spell) are added value by value
// into the bins instead.  Each bin stays below 2^63 in magnitude for L <= 2^23: at most L values
// below 2^39 each, plus one piece below 2^32 per stage.
constexpr int kMeanWarps = 8;   // consumer warps
constexpr int kMeanBins = 9;    // a value lands in bin (pos >> 5) <= 7, a stage sum in bins <= 8
constexpr int kMeanSpan = 39;   // widest exponent span a stage may have for its fp64 sum
constexpr size_t kMeanSmem = static_cast<size_t>(kMeanStages) * kMeanTok * kMeanCh * 2;  // the ring

// |v| = m * 2^(pos - 133) for the bf16 bit pattern v: m < 256, 0 <= pos <= 254
__device__ __forceinline__ void bf16_units(uint32_t v, uint32_t& m, uint32_t& pos) {
  const uint32_t e = (v >> 7) & 0xFFu, f = v & 0x7Fu;
  m = e == 0u ? f : 128u + f;
  pos = e == 0u ? 0u : e - 1u;
}

__global__ void __launch_bounds__(32 * (kMeanWarps + 1)) key_mean_kernel(const __grid_constant__ CUtensorMap tm,
                                                                         const __grid_constant__ MeanArgs a) {
  extern __shared__ __align__(128) uint16_t ring[];  // [kMeanStages][kMeanTok][kMeanCh]
  __shared__ __align__(8) uint64_t full[kMeanStages], empty[kMeanStages];
  __shared__ unsigned long long bins[kMeanWarps][kMeanBins][kMeanCh];  // each slot owned by one thread
  __shared__ int s_issued;
  __shared__ int s_bad;
  __shared__ int s_ok;  // this CTA summed all of its slices
  const int cg = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.z, n_split = gridDim.z;  // cluster (1, 1, n_split): rank = split
  const int all_tiles = (a.L + kMeanTok - 1) / kMeanTok;
  const int n_tiles = split < all_tiles ? (all_tiles - split + n_split - 1) / n_split : 0;  // this CTA's
  for (int i = threadIdx.x; i < kMeanWarps * kMeanBins * kMeanCh; i += blockDim.x) (&bins[0][0][0])[i] = 0ull;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMeanStages; ++i) {
      ptx::mbar_init(ptx::smem_u32(&full[i]), 1);
      ptx::mbar_init(ptx::smem_u32(&empty[i]), 1);
    }
    ptx::fence_mbar_init();
    s_issued = 0;
    s_bad = 0;
  }
  __syncthreads();
  bool ok = true;
  if (warp == kMeanWarps) {
    // producer: one TMA box (64 tokens x 32 channels) per stage; a stage is reused once the warp
    // that summed it has released it
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int st = i % kMeanStages;
        if (i >= kMeanStages && !wait_phase(ptx::smem_u32(&empty[st]), ((i / kMeanStages) - 1) & 1)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(ptx::smem_u32(&full[st]), kMeanTok * kMeanCh * 2);
        ptx::tma_load_4d(ptx::smem_u32(ring + st * kMeanTok * kMeanCh), &tm, cg * kMeanCh, h,
                         (split + i * n_split) * kMeanTok, b, ptx::smem_u32(&full[st]));
        ++issued;
      }
      s_issued = issued;
    }
  } else {
    // warp w sums the stages of tiles w, w + 8, ...; lane = channel
    unsigned long long* my = &bins[warp][0][lane];  // bin k of this thread: my[k * kMeanCh]
    for (int i = warp; i < n_tiles; i += kMeanWarps) {
      const int st = i % kMeanStages;
      ok = __all_sync(0xFFFFFFFFu, wait_phase(ptx::smem_u32(&full[st]), (i / kMeanStages) & 1));
      if (!ok) break;
      const int n = min(kMeanTok, a.L - (split + i * n_split) * kMeanTok);
      const uint16_t* col = ring + st * kMeanTok * kMeanCh + lane;
      // fp64 sum of the stage, with the largest magnitude and the smallest non-zero one (as bit
      // patterns: a zero's pattern less one wraps to the top and never wins the minimum)
      double s[4] = {0.0, 0.0, 0.0, 0.0};
      uint32_t hi = 0u, lo_m1 = 0xFFFFFFFFu;
      if (n == kMeanTok) {
        uint32_t v[kMeanTok];
#pragma unroll
        for (int t = 0; t < kMeanTok; ++t) v[t] = col[t * kMeanCh];
#pragma unroll
        for (int t = 0; t < kMeanTok; ++t) {
          const uint32_t mag = v[t] & 0x7FFFu;
          hi = max(hi, mag);
          lo_m1 = min(lo_m1, mag - 1u);
          s[t & 3] = __dadd_rn(s[t & 3], static_cast<double>(__uint_as_float(v[t] << 16)));
        }
      } else {
        for (int t = 0; t < n; ++t) {
          const uint32_t v = col[t * kMeanCh];
          const uint32_t mag = v & 0x7FFFu;
          hi = max(hi, mag);
          lo_m1 = min(lo_m1, mag - 1u);
          s[0] = __dadd_rn(s[0], static_cast<double>(__uint_as_float(v << 16)));
        }
      }
      bool exact = hi < 0x7F80u;  // finite
      if (exact && hi != 0u) {
        const uint32_t lo = lo_m1 + 1u;
        const int p_hi = hi >= 0x80u ? static_cast<int>(hi >> 7) - 1 : 0;
        const int p_lo = lo >= 0x80u ? static_cast<int>(lo >> 7) - 1 : 0;
        exact = p_hi - p_lo <= kMeanSpan;
      }
      if (exact) {
        const double sum = __dadd_rn(__dadd_rn(s[0], s[1]), __dadd_rn(s[2], s[3]));
        if (sum != 0.0) {
          // sum = M * 2^(E - 1075) = M * 2^sh units of 2^-133; a whole number of them, so a
          // negative sh only drops zero bits of M
          const unsigned long long sb = static_cast<unsigned long long>(__double_as_longlong(sum));
          unsigned long long M = (sb & 0xFFFFFFFFFFFFFull) | (1ull << 52);
          int sh = static_cast<int>((sb >> 52) & 0x7FFu) - 942;
          if (sh < 0) {
            M >>= -sh;
            sh = 0;
          }
          const int k = sh >> 5, r = sh & 31;  // |sum| < 2^267 units: sh <= 214, k + 2 <= 8
          const unsigned long long lo64 = M << r, hi64 = r ? M >> (64 - r) : 0ull;
          unsigned long long p0 = lo64 & 0xFFFFFFFFull, p1 = lo64 >> 32, p2 = hi64;
          if (sb >> 63) {
            p0 = 0ull - p0;
            p1 = 0ull - p1;
            p2 = 0ull - p2;
          }
          my[k * kMeanCh] += p0;
          my[(k + 1) * kMeanCh] += p1;
          my[(k + 2) * kMeanCh] += p2;
        }
      } else {
        // value by value: bin (pos >> 5) gets m * 2^(pos & 31), negated for a negative value
        for (int t = 0; t < n; ++t) {
          const uint32_t v = col[t * kMeanCh];
          if ((v & 0x7FFFu) == 0u) continue;  // +-0 adds nothing
          uint32_t m, pos;
          bf16_units(v, m, pos);
          unsigned long long add = static_cast<unsigned long long>(m) << (pos & 31u);
          if (v & 0x8000u) add = 0ull - add;  // two's complement: the bins wrap, the sums do not
          my[(pos >> 5) * kMeanCh] += add;
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&empty[st]));
    }
    if (!ok && lane == 0) atomicOr(&s_bad, 1);
  }
  if (!ok && lane == 0) atomicOr(a.status, kStatusTimeout);
  __syncthreads();
  if (threadIdx.x == 32 * kMeanWarps) {
    // after a time-out some copies may still be in flight: let them land (bounded) before the
    // CTA's shared memory goes away
    for (int i = max(0, s_issued - kMeanStages); i < s_issued; ++i)
      if (!wait_phase(ptx::smem_u32(&full[i % kMeanStages]), (i / kMeanStages) & 1)) break;
  }
  if (warp == 0) {
    // this CTA's sum per bin: the warps' bins added into warp 0's (wrapping sums)
#pragma unroll
    for (int k = 0; k < kMeanBins; ++k) {
      unsigned long long bk = bins[0][k][lane];
#pragma unroll
      for (int w = 1; w < kMeanWarps; ++w) bk += bins[w][k][lane];
      bins[0][k][lane] = bk;
    }
    if (lane == 0) s_ok = (s_bad == 0 && s_issued == n_tiles) ? 1 : 0;
  }
  __syncthreads();
  if (n_split > 1) {  // every CTA's sums visible to the cluster
    ptx::cluster_arrive_release();
    ptx::cluster_wait_acquire();
  }
  if (split == 0 && warp == 0) {
    unsigned long long bk[kMeanBins];
#pragma unroll
    for (int k = 0; k < kMeanBins; ++k) bk[k] = bins[0][k][lane];
    bool all_ok = s_ok != 0;
    for (int r = 1; r < n_split; ++r) {
      all_ok = all_ok && ptx::ld_shared_cluster_u32(ptx::smem_u32(&s_ok), r) != 0u;
#pragma unroll
      for (int k = 0; k < kMeanBins; ++k) bk[k] += ptx::ld_shared_cluster_u64(ptx::smem_u32(&bins[0][k][lane]), r);
    }
    if (all_ok) {
      // S = sum over bins of bk[k] * 2^(32 k) as 32-bit digits (two's complement), then the mean
      constexpr int kDigits = kMeanBins + 1;
      uint32_t d[kDigits];
      int64_t carry = 0;
#pragma unroll
      for (int k = 0; k < kDigits; ++k) {
        const int64_t acc = carry + (k < kMeanBins ? static_cast<int64_t>(bk[k]) : 0);
        d[k] = static_cast<uint32_t>(acc);                                // the low 32 bits
        carry = (acc - static_cast<int64_t>(d[k])) / (int64_t(1) << 32);  // exact: the rest is a multiple
      }
      a.k_mean[(static_cast<int64_t>(bh) * a.C + a.slot) * kHeadDim + cg * kMeanCh + lane] =
          exact_mean_to_f32<kDigits>(d, static_cast<uint32_t>(a.L));
    }
  }
  if (n_split > 1) {  // CTA 0 has read the others' shared memory
    ptx::cluster_arrive_release();
    ptx::cluster_wait_acquire();
  }
}

// this thread's 8 elements of one token row as fp32: x, or x - mu (one fp32 subtraction each)
__device__ __forceinline__ void row_values(uint4 w, const float (&mu)[8], bool smooth, float (&y)[8]) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    y[2 * i] = __uint_as_float(wv[i] << 16);
    y[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
  }
  if (smooth) {
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fsub_rn(y[i], mu[i]);
  }
}

__device__ __forceinline__ void load_mu(const QuantArgs& a, int bh, int tensor, bool& smooth, float (&mu)[8]) {
  smooth = tensor == 0 && (a.flags & NVFP4KV_K_SMOOTH);
#pragma unroll
  for (int i = 0; i < 8; ++i) mu[i] = 0.0f;
  if (smooth) {
    const float* m = a.k_mean + (static_cast<int64_t>(bh) * a.C + a.slot) * kHeadDim + (threadIdx.x & 15) * 8;
    const float4 m0 = *reinterpret_cast<const float4*>(m), m1 = *reinterpret_cast<const float4*>(m + 4);
    mu[0] = m0.x; mu[1] = m0.y; mu[2] = m0.z; mu[3] = m0.w;
    mu[4] = m1.x; mu[5] = m1.y; mu[6] = m1.z; mu[7] = m1.w;
  }
}

__global__ void __launch_bounds__(kThreads, 4) recipe_amax_kernel(const __grid_constant__ QuantArgs a) {
  const int part = blockIdx.x, bh = blockIdx.y, tensor = blockIdx.z;
  const int b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int t_begin = part * kPartTokens;
  const int t_end = min(a.L, t_begin + kPartTokens);
  const int sub = threadIdx.x >> 4;
  const uint16_t* x = a.x[tensor] + static_cast<int64_t>(b) * a.L * a.token_stride +
                      static_cast<int64_t>(h) * kHeadDim + (threadIdx.x & 15) * 8;
  uint4 w[kPasses];
#pragma unroll
  for (int u = 0; u < kPasses; ++u) {
    const int t = t_begin + u * (kThreads / 16) + sub;
    w[u] = t < t_end ? ld_row16(x + static_cast<int64_t>(t) * a.token_stride) : make_uint4(0, 0, 0, 0);
  }
  bool smooth;
  float mu[8];
  load_mu(a, bh, tensor, smooth, mu);
  float m = 0.0f;
#pragma unroll
  for (int u = 0; u < kPasses; ++u) {
    const int t = t_begin + u * (kThreads / 16) + sub;
    float y[8];
    row_values(w[u], mu, smooth, y);
    if (t < t_end)
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(y[i]));
  }
  uint32_t mb = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m));  // non-negative floats order as integers
  __shared__ uint32_t red[kWarps];
  if (lane == 0) red[warp] = mb;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) r = max(r, red[i]);
    a.partial[(static_cast<int64_t>(tensor) * a.B * a.H + bh) * a.parts + part] = r;
  }
}

// E2M1 magnitude code (0..7) -> value {0, 0.5, 1, 1.5, 2, 3, 4, 6}
__device__ __forceinline__ double e2m1_value(uint32_t nib) {
  const uint32_t m = nib & 7u;
  const double v = m < 4 ? 0.5 * m : static_cast<double>(1u << ((m - 2) >> 1)) * ((m & 1u) ? 1.5 : 1.0);
  return (nib & 8u) ? -v : v;
}

// E2M1 codes of y * r (8 elements, element 2j in the low nibble of byte j); 0 when r is 0
__device__ __forceinline__ uint32_t codes8f(const float (&y)[8], float r) {
  if (r == 0.0f) return 0u;
  float z[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) z[i] = __fmul_rn(y[i], r);
  return ptx::f32x8_to_e2m1x8(z);
}

// squared error terms (y_i - E2M1(q_i) * s * g)^2 of this lane's 8 elements, each operation
// rounded once in fp64
__device__ __forceinline__ void sq_terms(const float (&y)[8], uint32_t q, uint32_t s_code, float g, double (&sq)[8]) {
  const double sv = static_cast<double>(ptx::e4m3_to_f32(s_code)), gd = static_cast<double>(g);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const double xh = __dmul_rn(__dmul_rn(e2m1_value((q >> (4 * i)) & 0xFu), sv), gd);
    const double diff = __dadd_rn(static_cast<double>(y[i]), -xh);
    sq[i] = __dmul_rn(diff, diff);
  }
}

// the block's squared error, summed over its 16 elements in order: the even lane of the pair
// holds elements 0-7, the odd lane 8-15 and continues from the even lane's partial sum
__device__ __forceinline__ double block_sq_error(const double (&sq)[8], int lane) {
  double acc = 0.0;
  if ((lane & 1) == 0)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc = __dadd_rn(acc, sq[i]);
  const double from_even = __shfl_xor_sync(0xFFFFFFFFu, acc, 1);
  if (lane & 1) {
    acc = from_even;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc = __dadd_rn(acc, sq[i]);
  }
  return acc;  // complete on the odd lane
}

__global__ void __launch_bounds__(kThreads, 2) recipe_encode_kernel(const __grid_constant__ QuantArgs a) {
  const int part = blockIdx.x, bh = blockIdx.y, tensor = blockIdx.z;
  const int b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_begin = part * kEncTokens;
  const int t_end = min(a.L, t_begin + kEncTokens);
  const int sub = threadIdx.x >> 4;
  const uint16_t* x = a.x[tensor] + static_cast<int64_t>(b) * a.L * a.token_stride +
                      static_cast<int64_t>(h) * kHeadDim + (threadIdx.x & 15) * 8;
  uint4 w[kEncPasses];
#pragma unroll
  for (int u = 0; u < kEncPasses; ++u) {
    const int t = t_begin + u * (kThreads / 16) + sub;
    w[u] = t < t_end ? ld_row16(x + static_cast<int64_t>(t) * a.token_stride) : make_uint4(0, 0, 0, 0);
  }
  bool smooth;
  float mu[8];
  load_mu(a, bh, tensor, smooth, mu);
  const bool adaptive = tensor == 1 && (a.flags & NVFP4KV_V_ADAPTIVE_SCALE);
  asm volatile("griddepcontrol.wait;" ::: "memory");

  __shared__ float s_g;
  if (warp == 0) {
    const uint32_t* p = a.partial + (static_cast<int64_t>(tensor) * a.B * a.H + bh) * a.parts;
    uint32_t m = 0;
    for (int i = lane; i < a.parts; i += 32) m = max(m, p[i]);
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (lane == 0) {
      const float A = __uint_as_float(m);
      const float g = (A == 0.0f) ? 0.0f : __fdiv_rn(A, 2688.0f);
      s_g = g;
      if (part == 0) a.gscale[tensor][static_cast<int64_t>(bh) * a.C + a.slot] = g;
    }
  }
  __shared__ float rtab[128];
  __syncthreads();
  const Encoder enc = make_encoder(s_g, rtab, threadIdx.x, kThreads);
  Encoder enc4 = enc;  // scale target 4: a_b / (4 g), with 4 g exact
  enc4.d = __fmul_rn(4.0f, enc.g);
  enc4.y = enc.g != 0.0f ? __frcp_rn(enc4.d) : 0.0f;
  enc4.fast = enc.g != 0.0f && enc4.d >= 0x1p-126f && enc4.y >= 0x1p-126f && enc4.y < 0x1p127f;
  __syncthreads();

  const int64_t row0 = static_cast<int64_t>(bh) * a.T + static_cast<int64_t>(a.slot) * a.L;
  uint8_t* codes = a.codes[tensor] + row0 * kCodeBytes + (lane & 15) * 4;
  uint8_t* scales = a.scales[tensor] + row0 * kScaleBytes + ((lane & 15) >> 1);
#pragma unroll
  for (int u = 0; u < kEncPasses; ++u) {
    const int t = t_begin + u * (kThreads / 16) + sub;
    float y[8];
    row_values(w[u], mu, smooth, y);
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(y[i]));
    const float ab = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
    uint32_t s_code = block_scale_code(ab, enc);
    uint32_t qc = codes8f(y, rtab[s_code & 0x7F]);
    if (adaptive) {  // warp-uniform: the tensor is the CTA's
      const uint32_t s4 = block_scale_code(ab, enc4);
      const uint32_t q4 = codes8f(y, rtab[s4 & 0x7F]);
      double sq6[8], sq4[8];
      sq_terms(y, qc, s_code, enc.g, sq6);
      sq_terms(y, q4, s4, enc.g, sq4);
      const double e6 = block_sq_error(sq6, lane), e4 = block_sq_error(sq4, lane);
      const bool pick4 = __shfl_sync(0xFFFFFFFFu, e4 < e6 ? 1 : 0, lane | 1) != 0;  // the odd lane decides
      if (pick4) {
        s_code = s4;
        qc = q4;
      }
    }
    if (t < t_end) {
      *reinterpret_cast<uint32_t*>(codes + static_cast<int64_t>(t) * kCodeBytes) = qc;
      if ((lane & 1) == 0) scales[static_cast<int64_t>(t) * kScaleBytes] = static_cast<uint8_t>(s_code);
    }
  }
}

// ---------------------------------------------------------------------------------------
// Single-launch path for one or many layers (ticketed).  A slice is one (layer, tensor, b, h) of
// the new chunk; a part is kTicketTokens of its tokens.  Every CTA takes a ticket t in the order
// CTAs start (an atomic counter) and
//   1. reduces max|x| over part t and folds it into its slice's maximum (atomicMax on the bf16
//      magnitude bits), then counts the part as done;
//   2. encodes part e = t - lag once every part of e's slice is done, re-reading its rows (still in
//      L2: lag parts of 32 KB were read since).  The lag exceeds the number of CTAs that can be
//      resident at once, so that slice is normally complete before the CTA gets there.
// Step 2 only waits for tickets below t, which belong to CTAs that already started and whose
// step 1 waits for nothing, so the wait always ends; it is still bounded (the status bit is set
// if it ever runs out).  The input crosses HBM once for any number of layers.
constexpr int kMaxLayers = 64;
constexpr int kTicketTokens = 128;

struct TicketArgs {
  const uint16_t* x[kMaxLayers][2];
  uint8_t* codes[kMaxLayers][2];
  uint8_t* scales[kMaxLayers][2];
  float* gscale[kMaxLayers][2];
  uint32_t* ctr;  // [0] ticket counter; per slice s: [1 + 2s] max|x| bits, [2 + 2s] parts done
  uint32_t* status;
  int64_t token_stride;
  int64_t T;  // tokens per (b, h) in the cache
  int B, H, L, C, slot, parts, lag;
  int n_work;  // slices * parts
};

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__global__ void __launch_bounds__(kThreads, 4) quantize_ticket_kernel(const __grid_constant__ TicketArgs a) {
  __shared__ int s_ticket;
  __shared__ uint32_t red[kWarps];
  __shared__ float s_g;
  __shared__ int s_ok;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) s_ticket = static_cast<int>(atomicAdd(a.ctr, 1u));
  __syncthreads();
  const int t = s_ticket;
  const int BH = a.B * a.H;
  if (t < a.n_work) {
    // ---- 1. max|x| over part t
    const int sl = t / a.parts, part = t % a.parts;
    const int bh = sl % BH, tensor = (sl / BH) & 1, layer = sl / (2 * BH);
    const int b = bh / a.H, h = bh % a.H;
    const int t_begin = part * kTicketTokens, t_end = min(a.L, t_begin + kTicketTokens);
    const uint16_t* x = a.x[layer][tensor] + static_cast<int64_t>(b) * a.L * a.token_stride +
                        static_cast<int64_t>(h) * kHeadDim + (threadIdx.x & 15) * 8;
    const int sub = threadIdx.x >> 4;
    uint4 w[kPasses];
#pragma unroll
    for (int u = 0; u < kPasses; ++u) {
      const int tt = t_begin + u * (kThreads / 16) + sub;
      w[u] = tt < t_end ? ld_row16(x + static_cast<int64_t>(tt) * a.token_stride) : make_uint4(0, 0, 0, 0);
    }
    uint32_t acc = 0;
#pragma unroll
    for (int u = 0; u < kPasses; ++u) acc = __vmaxu2(acc, absmax_bits(w[u]));
    uint32_t m = max(acc & 0xFFFFu, acc >> 16);
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t r = 0;
#pragma unroll
      for (int i = 0; i < kWarps; ++i) r = max(r, red[i]);
      atomicMax(a.ctr + 1 + 2 * sl, r);
      red_release_add(a.ctr + 2 + 2 * sl, 1u);  // orders the maximum before the count
    }
  }
  const int e = t - a.lag;
  if (e < 0 || e >= a.n_work) return;
  // ---- 2. encode part e; its rows do not depend on the slice maximum, so they load first
  const int sl = e / a.parts, part = e % a.parts;
  const int bh = sl % BH, tensor = (sl / BH) & 1, layer = sl / (2 * BH);
  const int b = bh / a.H, h = bh % a.H;
  const int t_begin = part * kTicketTokens, t_end = min(a.L, t_begin + kTicketTokens);
  const int j = threadIdx.x & 3, tok = threadIdx.x >> 2;  // 4 threads per token, 32 elements each
  const uint16_t* x = a.x[layer][tensor] + static_cast<int64_t>(b) * a.L * a.token_stride +
                      static_cast<int64_t>(h) * kHeadDim + j * 32;
  constexpr int kRowsPerPass = kThreads / 4;
  constexpr int kEncPass = kTicketTokens / kRowsPerPass;  // 2
  uint4 w[kEncPass][4];
#pragma unroll
  for (int u = 0; u < kEncPass; ++u) {
    const int tt = t_begin + u * kRowsPerPass + tok;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w[u][k] = tt < t_end ? ld_row16(x + static_cast<int64_t>(tt) * a.token_stride + 8 * k) : make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x == 0) {
    int ok = 1;
    const uint32_t* done = a.ctr + 2 + 2 * sl;
    uint64_t t0 = 0;
    int it = 0;
    while (ld_acquire_u32(done) < static_cast<uint32_t>(a.parts)) {
      const uint64_t now = ptx::globaltimer_ns();
      if (it++ == 0) t0 = now;
      if (now - t0 > kWaitLimitNs) {
        ok = 0;
        atomicOr(a.status, kStatusTimeout);
        break;
      }
      __nanosleep(64);
    }
    const float A = __uint_as_float(ld_acquire_u32(a.ctr + 1 + 2 * sl) << 16);
    // FP32 scale of this (chunk, head, tensor): g = max|x| / (448 * 6)
    s_g = (A == 0.0f) ? 0.0f : __fdiv_rn(A, 2688.0f);
    s_ok = ok;
    if (ok && part == 0) a.gscale[layer][tensor][static_cast<int64_t>(bh) * a.C + a.slot] = s_g;
  }
  __syncthreads();
  if (!s_ok) return;
  const float g = s_g;
  Encoder enc;
  enc.g = g;
  enc.d = __fmul_rn(6.0f, g);
  enc.y = g != 0.0f ? __frcp_rn(enc.d) : 0.0f;
  enc.fast = g != 0.0f && enc.d >= 0x1p-126f && enc.y >= 0x1p-126f && enc.y < 0x1p127f;
  const int64_t row0 = static_cast<int64_t>(bh) * a.T + static_cast<int64_t>(a.slot) * a.L;
  uint8_t* codes = a.codes[layer][tensor] + row0 * kCodeBytes + j * 16;
  uint8_t* scales = a.scales[layer][tensor] + row0 * kScaleBytes + j * 2;
#pragma unroll
  for (int u = 0; u < kEncPass; ++u) {
    const int tt = t_begin + u * kRowsPerPass + tok;
    if (tt >= t_end) continue;
    uint32_t qc[4], sc[2];
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
      uint32_t mb = __vmaxu2(absmax_bits(w[u][2 * blk]), absmax_bits(w[u][2 * blk + 1]));
      mb = max(mb & 0xFFFFu, mb >> 16);
      sc[blk] = block_scale_code(__uint_as_float(mb << 16), enc);
      // r = RN(1 / RN(s * g)); all-zero codes when s is 0 or the reciprocal overflows (the same
      // operations as the per-code table of make_encoder)
      const float sv = ptx::e4m3_to_f32(sc[blk]);
      float r = 0.0f;
      if (sv != 0.0f) {
        r = __frcp_rn(__fmul_rn(sv, g));
        if (r == __int_as_float(0x7F800000)) r = 0.0f;
      }
      qc[2 * blk] = codes8(w[u][2 * blk], r);
      qc[2 * blk + 1] = codes8(w[u][2 * blk + 1], r);
    }
    *reinterpret_cast<uint4*>(codes + static_cast<int64_t>(tt) * kCodeBytes) = make_uint4(qc[0], qc[1], qc[2], qc[3]);
    *reinterpret_cast<uint16_t*>(scales + static_cast<int64_t>(tt) * kScaleBytes) =
        static_cast<uint16_t>(sc[0] | (sc[1] << 8));
  }
}

// ---------------------------------------------------------------------------------------
// Single-pass path: one thread-block cluster per (b, h, tensor).  The cluster's CTAs split the
// chunk's tokens; each CTA brings its rows into shared memory with TMA (the input is read from
// HBM once), reduces its max|x|, and the CTAs exchange their maxima through distributed shared
// memory before every CTA encodes its rows from shared memory.
constexpr int kBoxTokens = 16;          // tokens per TMA box (16 x 256 B)
constexpr int kMaxCtaTokens = 448;      // 112 KB of bf16 rows: two CTAs per SM
constexpr int kMaxCluster = 16;
constexpr int kCThreads = 512;
constexpr int kCWarps = kCThreads / 32;

struct ClusterArgs {
  uint8_t* codes[2];
  uint8_t* scales[2];
  float* gscale[2];
  uint32_t* status;
  int64_t T;  // tokens per (b, h) in the cache
  int H, L, C, slot, cta_tokens;
};

__global__ void __launch_bounds__(kCThreads)
    quantize_cluster_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                            const __grid_constant__ ClusterArgs a) {
  extern __shared__ __align__(128) uint8_t qsm[];
  __shared__ __align__(8) uint64_t full_bar;
  __shared__ uint32_t red[kCWarps];
  __shared__ uint32_t cta_max;
  __shared__ float s_g;
  __shared__ float rtab[128];
  const uint32_t rank = ptx::cluster_ctarank();
  const int bh = blockIdx.y, tensor = blockIdx.z;
  const int b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = static_cast<int>(rank) * a.cta_tokens;
  const int n = max(0, min(a.L - t0, a.cta_tokens));
  const int nbox = (n + kBoxTokens - 1) / kBoxTokens;
  const uint32_t bar = ptx::smem_u32(&full_bar);
  const uint32_t xs = ptx::smem_u32(qsm);

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && nbox > 0) {
    const CUtensorMap* tm = tensor == 0 ? &tm_k : &tm_v;
    ptx::mbar_arrive_expect_tx(bar, nbox * kBoxTokens * kHeadDim * 2);
    for (int i = 0; i < nbox; ++i)
      ptx::tma_load_4d(xs + i * kBoxTokens * kHeadDim * 2, tm, 0, h, t0 + i * kBoxTokens, b, bar);
  }
  bool ok = true;
  if (nbox > 0) {
    uint64_t w0 = 0;
    int it = 0;
    while (!ptx::mbar_try_wait(bar, 0)) {
      const uint64_t now = ptx::globaltimer_ns();
      if (it++ == 0) w0 = now;
      if (now - w0 > kWaitLimitNs) {
        ok = false;
        break;
      }
    }
  }
  ok = __syncthreads_and(ok) != 0;
  if (!ok && threadIdx.x == 0) atomicOr(a.status, kStatusTimeout);

  // max|x| over this CTA's rows (bf16 magnitudes compare as integers)
  const uint16_t* rows = reinterpret_cast<const uint16_t*>(qsm) + (lane & 15) * 8;
  uint32_t acc = 0;
  if (ok)
    for (int t = 2 * warp + (lane >> 4); t < n; t += 2 * kCWarps)
      acc = __vmaxu2(acc, absmax_bits(*reinterpret_cast<const uint4*>(rows + t * kHeadDim)));
  uint32_t m = max(acc & 0xFFFFu, acc >> 16);
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < kCWarps; ++i) r = max(r, red[i]);
    cta_max = r;
  }
  // Exchange the maxima: every CTA's cta_max is written before the barrier; warp 0 then reads
  // all of them.  The second barrier's wait (at the end) keeps every CTA's shared memory alive
  // until all peers have read it.
  ptx::cluster_arrive_release();
  ptx::cluster_wait_acquire();
  if (warp == 0) {
    const uint32_t ncta = gridDim.x;
    uint32_t r = lane < static_cast<int>(ncta) ? ptx::ld_shared_cluster_u32(ptx::smem_u32(&cta_max), lane) : 0u;
    r = __reduce_max_sync(0xFFFFFFFFu, r);
    if (lane == 0) {
      const float A = __uint_as_float(r << 16);
      s_g = (A == 0.0f) ? 0.0f : __fdiv_rn(A, 2688.0f);
    }
  }
  ptx::cluster_arrive_release();
  __syncthreads();
  const float g = s_g;
  if (ok && rank == 0 && threadIdx.x == 0) a.gscale[tensor][static_cast<int64_t>(bh) * a.C + a.slot] = g;
  const Encoder enc = make_encoder(g, rtab, threadIdx.x, kCThreads);
  __syncthreads();
  const int64_t row0 = static_cast<int64_t>(bh) * a.T + static_cast<int64_t>(a.slot) * a.L + t0;
  uint8_t* codes = a.codes[tensor] + row0 * kCodeBytes + (lane & 15) * 4;
  uint8_t* scales = a.scales[tensor] + row0 * kScaleBytes + ((lane & 15) >> 1);
  if (ok) {
    // warp-uniform trip count; two independent token pairs per pass (lanes 0-15 take the even
    // token of a pair, 16-31 the odd one)
    for (int tp = 4 * warp; tp < n; tp += 4 * kCWarps) {
      const int ta = tp + (lane >> 4), tb = ta + 2;
      const uint4 wa = ta < n ? *reinterpret_cast<const uint4*>(rows + ta * kHeadDim) : make_uint4(0, 0, 0, 0);
      const uint4 wb = tb < n ? *reinterpret_cast<const uint4*>(rows + tb * kHeadDim) : make_uint4(0, 0, 0, 0);
      encode_store(wa, enc, rtab, ta < n, codes + static_cast<int64_t>(ta) * kCodeBytes,
                   scales + static_cast<int64_t>(ta) * kScaleBytes, lane);
      encode_store(wb, enc, rtab, tb < n, codes + static_cast<int64_t>(tb) * kCodeBytes,
                   scales + static_cast<int64_t>(tb) * kScaleBytes, lane);
    }
  } else if (nbox > 0 && threadIdx.x == 0) {
    // the copies were issued: let them land before the CTA's shared memory goes away
    uint64_t w0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, 0))
      if (ptx::globaltimer_ns() - w0 > kWaitLimitNs) break;
  }
  ptx::cluster_wait_acquire();
}

}  // namespace

int quantize_parts(int, int, int chunk_tokens) {
  return chunk_tokens > 0 ? (chunk_tokens + kPartTokens - 1) / kPartTokens : 1;
}

size_t quantize_workspace_bytes(int batch, int heads, int chunk_tokens) {
  return static_cast<size_t>(2) * batch * heads * quantize_parts(batch, heads, chunk_tokens) *
         sizeof(uint32_t);
}

namespace {

// Cluster size for the single-pass path, or 0 when the chunk does not fit it: about two CTAs
// per SM over the whole grid, at least 16 tokens and at most kMaxCtaTokens rows per CTA.
int cluster_size(int units, int L, int n_sms) {
  int cl = std::max(1, std::min(kMaxCluster, (2 * n_sms) / std::max(1, units)));
  cl = std::min(cl, std::max(1, L / 16));
  while (cl < kMaxCluster && (L + cl - 1) / cl > kMaxCtaTokens) ++cl;
  return (L + cl - 1) / cl > kMaxCtaTokens ? 0 : cl;
}

struct ClusterPlan {
  int cl = 0;  // 0: the two-pass path
  int cta_tokens = 0;
  size_t smem = 0;
};

cudaLaunchConfig_t cluster_config(const nvfp4kv_cache& c, const ClusterPlan& pl, cudaStream_t stream,
                                  cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.cl, c.batch * c.heads, 2);
  cfg.blockDim = dim3(kCThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = pl.cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// The single-pass plan for this cache shape on the current device, or cl = 0.  The path is only
// worth taking when every (b, h, tensor) gets its cluster in the first wave (a second wave
// would wait for the first to finish its whole load-reduce-encode sequence), so the number of
// co-resident clusters of the shape is asked once per (device, shape).
PerDeviceOnce g_cluster_attr;

ClusterPlan cluster_plan(const nvfp4kv_cache& c) {
  ClusterPlan pl;
  const int sms = current_sm_count();
  if (sms <= 0) return pl;
  const int cl = cluster_size(2 * c.batch * c.heads, c.chunk_tokens, sms);
  if (cl == 0 || tensor_map_encoder() == nullptr) return pl;
  // function attributes live per device: set them on each device the library runs on
  const cudaError_t attr_err = g_cluster_attr.run([] {
    cudaError_t e = cudaFuncSetAttribute(quantize_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kMaxCtaTokens * kHeadDim * 2);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(quantize_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
  });
  if (attr_err != cudaSuccess) return pl;
  ClusterPlan cand;
  cand.cl = cl;
  cand.cta_tokens = ((c.chunk_tokens + cl - 1) / cl + kBoxTokens - 1) / kBoxTokens * kBoxTokens;
  cand.smem = static_cast<size_t>(cand.cta_tokens) * kHeadDim * 2;
  static std::mutex mu;
  static std::map<std::tuple<int, int, size_t>, int> active;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return pl;
  int max_active = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(dev, cand.cl, cand.smem);
    auto it = active.find(key);
    if (it == active.end()) {
      cudaLaunchAttribute attr[1];
      const cudaLaunchConfig_t cfg = cluster_config(c, cand, nullptr, attr);
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, quantize_cluster_kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        clusters = 0;
      }
      it = active.emplace(key, clusters).first;
    }
    max_active = it->second;
  }
  return max_active >= 2 * c.batch * c.heads ? cand : pl;
}

cudaError_t launch_cluster(const nvfp4kv_cache& c, int slot, const uint16_t* k, const uint16_t* v,
                           int64_t token_stride, const ClusterPlan& pl, cudaStream_t stream, bool* launched) {
  *launched = false;
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  ClusterArgs a;
  a.codes[0] = c.k_codes;
  a.codes[1] = c.v_codes;
  a.scales[0] = c.k_scales;
  a.scales[1] = c.v_scales;
  a.gscale[0] = c.k_gscale;
  a.gscale[1] = c.v_gscale;
  a.status = c.status;
  a.T = static_cast<int64_t>(c.capacity_chunks) * c.chunk_tokens;
  a.H = c.heads;
  a.L = c.chunk_tokens;
  a.C = c.capacity_chunks;
  a.slot = slot;
  a.cta_tokens = pl.cta_tokens;
  CUtensorMap tm[2];
  const uint16_t* src[2] = {k, v};
  for (int i = 0; i < 2; ++i) {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(c.heads),
                                static_cast<cuuint64_t>(c.chunk_tokens), static_cast<cuuint64_t>(c.batch)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHeadDim) * 2,
                                   static_cast<cuuint64_t>(token_stride) * 2,
                                   static_cast<cuuint64_t>(c.chunk_tokens) * token_stride * 2};
    const cuuint32_t box[4] = {kHeadDim, 1, kBoxTokens, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (encode(&tm[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(src[i]), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaSuccess;  // not expressible as a tensor map: the two-pass path takes it
  }
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = cluster_config(c, pl, stream, attr);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_cluster_kernel, tm[0], tm[1], a);
  *launched = e == cudaSuccess;
  return e;
}

}  // namespace

int quantize_launches(const nvfp4kv_cache& c) {
  if (c.flags != 0) return (c.flags & NVFP4KV_K_SMOOTH) ? 3 : 2;
  return cluster_plan(c).cl > 0 ? 1 : 2;
}

namespace {

QuantArgs two_pass_args(const nvfp4kv_cache& c, int slot, const uint16_t* k, const uint16_t* v,
                        int64_t token_stride, void* workspace) {
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
  a.k_mean = c.k_mean;
  a.token_stride = token_stride;
  a.T = static_cast<int64_t>(c.capacity_chunks) * c.chunk_tokens;
  a.B = c.batch;
  a.H = c.heads;
  a.L = c.chunk_tokens;
  a.C = c.capacity_chunks;
  a.slot = slot;
  a.parts = quantize_parts(c.batch, c.heads, c.chunk_tokens);
  a.flags = c.flags;
  return a;
}

// The encode grid of the two-pass paths, a programmatic dependent of the amax grid: it launches
// while the amax grid drains and waits (griddepcontrol.wait) only before it reads the maxima.
template <typename Kernel>
cudaError_t launch_encode_dependent(Kernel kernel, const QuantArgs& a, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.L + kEncTokens - 1) / kEncTokens, a.B * a.H, 2);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

PerDeviceOnce g_mean_attr;

// CTAs per (32 channels, b, h) of the channel-mean grid: enough to fill the SMs once, at most 8 (a
// portable cluster), and at least four 64-token slices each.
unsigned mean_splits(const nvfp4kv_cache& c) {
  const int sms = current_sm_count();
  const int64_t ctas = static_cast<int64_t>(kHeadDim / kMeanCh) * c.batch * c.heads;
  const int64_t slices = (c.chunk_tokens + kMeanTok - 1) / kMeanTok;
  int64_t s = sms > 0 ? sms / ctas : 1;
  s = std::min<int64_t>(s, 8);
  s = std::min<int64_t>(s, slices / 4);
  return static_cast<unsigned>(std::max<int64_t>(s, 1));
}

cudaError_t launch_quantize_recipe(const nvfp4kv_cache& c, int slot, const uint16_t* k, const uint16_t* v,
                                   int64_t token_stride, void* workspace, cudaStream_t stream) {
  const QuantArgs a = two_pass_args(c, slot, k, v, token_stride, workspace);
  if (c.flags & NVFP4KV_K_SMOOTH) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap tm;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(c.heads),
                                static_cast<cuuint64_t>(c.chunk_tokens), static_cast<cuuint64_t>(c.batch)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHeadDim) * 2, static_cast<cuuint64_t>(token_stride) * 2,
                                   static_cast<cuuint64_t>(c.chunk_tokens) * token_stride * 2};
    const cuuint32_t box[4] = {kMeanCh, 1, kMeanTok, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (encode(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(k), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    MeanArgs m;
    m.k_mean = c.k_mean;
    m.status = c.status;
    m.H = c.heads;
    m.L = c.chunk_tokens;
    m.C = c.capacity_chunks;
    m.slot = slot;
    const cudaError_t attr_err = g_mean_attr.run([] {
      return cudaFuncSetAttribute(key_mean_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kMeanSmem));
    });
    if (attr_err != cudaSuccess) return attr_err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kHeadDim / kMeanCh, c.batch * c.heads, mean_splits(c));
    cfg.blockDim = dim3(32 * (kMeanWarps + 1), 1, 1);
    cfg.dynamicSmemBytes = kMeanSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = cfg.gridDim.z;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, key_mean_kernel, tm, m);
    if (e != cudaSuccess) return e;
  }
  recipe_amax_kernel<<<dim3(a.parts, c.batch * c.heads, 2), kThreads, 0, stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_encode_dependent(recipe_encode_kernel, a, stream);
}

}  // namespace

cudaError_t launch_quantize(const nvfp4kv_cache& c, int slot, const uint16_t* k, const uint16_t* v,
                            int64_t token_stride, void* workspace, cudaStream_t stream) {
  if (c.flags != 0) return launch_quantize_recipe(c, slot, k, v, token_stride, workspace, stream);
  const ClusterPlan pl = cluster_plan(c);
  if (pl.cl > 0) {
    bool launched = false;
    const cudaError_t e = launch_cluster(c, slot, k, v, token_stride, pl, stream, &launched);
    if (launched || e != cudaSuccess) return e;
  }
  const QuantArgs a = two_pass_args(c, slot, k, v, token_stride, workspace);
  amax_kernel<<<dim3(a.parts, c.batch * c.heads, 2), kThreads, 0, stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_encode_dependent(quantize_kernel, a, stream);
}

PerDeviceOnce g_ticket_occ;
int g_ticket_blocks_per_sm = 0;

size_t quantize_layers_workspace_bytes(int layers, int batch, int heads) {
  const size_t words = 1 + 2 * static_cast<size_t>(layers) * 2 * batch * heads;
  return (words * sizeof(uint32_t) + 255) / 256 * 256;
}

bool quantize_layers_supported(int layers, int batch, int heads, int chunk_tokens) {
  const int64_t parts = (chunk_tokens + kTicketTokens - 1) / kTicketTokens;
  const int64_t work = static_cast<int64_t>(layers) * 2 * batch * heads * parts;
  return layers >= 1 && layers <= kMaxLayers && work + 2 * parts < (int64_t(1) << 31);
}

cudaError_t launch_quantize_layers(const nvfp4kv_cache* caches, int layers, int slot, const uint16_t* const* k,
                                   const uint16_t* const* v, int64_t token_stride, void* workspace,
                                   cudaStream_t stream) {
  const nvfp4kv_cache& c = caches[0];
  TicketArgs a;
  for (int l = 0; l < layers; ++l) {
    a.x[l][0] = k[l];
    a.x[l][1] = v[l];
    a.codes[l][0] = caches[l].k_codes;
    a.codes[l][1] = caches[l].v_codes;
    a.scales[l][0] = caches[l].k_scales;
    a.scales[l][1] = caches[l].v_scales;
    a.gscale[l][0] = caches[l].k_gscale;
    a.gscale[l][1] = caches[l].v_gscale;
  }
  a.ctr = static_cast<uint32_t*>(workspace);
  a.status = c.status;
  a.token_stride = token_stride;
  a.T = static_cast<int64_t>(c.capacity_chunks) * c.chunk_tokens;
  a.B = c.batch;
  a.H = c.heads;
  a.L = c.chunk_tokens;
  a.C = c.capacity_chunks;
  a.slot = slot;
  a.parts = (c.chunk_tokens + kTicketTokens - 1) / kTicketTokens;
  a.n_work = layers * 2 * c.batch * c.heads * a.parts;
  // counters start at zero on every call
  cudaError_t e = cudaMemsetAsync(workspace, 0, quantize_layers_workspace_bytes(layers, c.batch, c.heads), stream);
  if (e != cudaSuccess) return e;
  // lag: more tickets than CTAs can be resident (so the slice of e is normally finished when its
  // encode starts) plus two slices; the re-read rows stay far inside L2
  e = g_ticket_occ.run([] {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&g_ticket_blocks_per_sm, quantize_ticket_kernel, kThreads, 0);
  });
  const int sms = current_sm_count();
  if (e != cudaSuccess || g_ticket_blocks_per_sm <= 0 || sms <= 0) return e != cudaSuccess ? e : cudaErrorUnknown;
  a.lag = g_ticket_blocks_per_sm * sms + 2 * a.parts;
  quantize_ticket_kernel<<<a.n_work + a.lag, kThreads, 0, stream>>>(a);
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

