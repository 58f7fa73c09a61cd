// attention.cu -- chunk attention over the NVFP4 KV cache on sm_100a.
//
// Method: "LongLive-2.0" paper page (paperpeel.com), section 1 and section 3.2 "Parallel KV
// Quantization": the cache stays in NVFP4 and is dequantised in parallel inside the
// attention kernel; section 4.2 "Inference with Multi-Shot Attention Sink": the query chunk
// attends to a permanent sink plus a sliding window of chunks (duplicates removed); section
// 2.1: a chunk sees its own tokens.  Reading note (yingwang.github.io), "The NVFP4
// quantization format": x_hat = E2M1 * E4M3 * FP32 scale.
//
// Work: every (batch, head) has ceil(Lq / 128) query tiles, grouped into work items of two tiles
// (the last item of a head holds one tile when the count is odd); an item walks all visible KV
// tiles (128 keys each; tiles lie inside runs of consecutive visible chunks, so chunks outside
// the mask are never read).  The grid is persistent: one CTA per SM, and the (item, KV tile)
// units are dealt out as equal-cost contiguous ranges (stream-K), so a CTA may finish one item,
// run a whole item, and start another.  A range that covers only part of an item's KV tiles
// leaves a partial result (unnormalised O, running max, running sum) in the workspace, and
// combine_kernel merges the parts of every split item.
//
// 512 threads, four warpgroups; warp roles:
//   softmax warps 0-3, 4-7    query tile 0 / 1 of the item: one query row per thread, online
//                             softmax over TMEM rows, epilogue; each warpgroup loads its own Q
//                             tile (TMA, 128B swizzle) and converts it to fp16 in place
//   producer warp 8           1-D bulk copies of each KV tile's packed codes + E4M3 scales into
//                             a ring of shared-memory slots
//   MMA warp 12               TMEM allocation; tcgen05.mma S = Q K^T (both operands in smem),
//                             O += P V (P from TMEM, V from smem), one elected lane
//   dequant warps 9-11, 13-15 E2M1 * E4M3 products, exact in fp16, written straight into the
//                             128B-swizzled UMMA operand layout: K (the B operand of Q K^T,
//                             K-major) and V (the B operand of P V, MN-major)
// TMEM per query tile q: S of a whole KV tile in columns [128 q, 128 q + 128) (one N = 128 QK
// chain), O in [256 + 128 q, 384 + 128 q).  The softmax warps take S in two 64-key sub-tiles and
// store P of sub-tile h over the first 32 columns of its S half; the P V of sub-tile h runs
// while the softmax works on h + 1, and the next KV tile's QK is issued behind the second P V
// (MMAs of one thread execute in order, so it cannot overwrite P before P V has read it).  The
// FP32 scales stay out of the MMAs: g_K(chunk) multiplies S per column, and g_V(chunk) / max g_V
// multiplies P per column before P is rounded to fp16 (fp16 P and V keep the P V product 8x
// finer than bf16).  Rows are rescaled lazily: the running max only moves when it grows by more
// than 2^14 (so P~ stays inside fp16's range).  With smoothed keys (the cache's K-smoothing
// option) every logit of a chunk's keys also gets scale * q . mu(chunk), computed once per
// (query row, chunk) from the fp16 Q row.
//
// Every mbarrier wait is bounded (%globaltimer); on a time-out the kernel ORs
// NVFP4KV_ERR_DEVICE_TIMEOUT into the status word, lets in-flight copies and MMAs finish,
// frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4kv {
namespace {

constexpr int BM = 128;  // query rows per tile (TMEM lanes)
constexpr int BN = 128;  // keys per KV tile
constexpr int SUB = 64;  // keys per S sub-tile
constexpr int D = kHeadDim;
constexpr int QT = 2;    // query tiles per work item
constexpr int NST = 2;   // stages of dequantised K / V tiles
constexpr int NPK = 3;   // slots of packed data (K and V tiles alternate)
constexpr int NCT = 4;   // slots of per-tile column tables
constexpr int PK_CODES = BN * kCodeBytes;               // 8192
constexpr int PK_BYTES = PK_CODES + BN * kScaleBytes;   // 9216
constexpr int TILE16 = BN * D * 2;                      // one 128 x 128 16-bit operand tile
constexpr int HALF16 = TILE16 / 2;                      // 128 rows x 64 elements (128 B rows)
constexpr int MAX_RUNS = kAttnMaxRuns;
constexpr int kMaxCtas = 1024;
// Relative cost of one KV tile of a two-tile item and of a one-tile item (the planner's weights;
// measured on B200: a one-tile item's KV tile takes about 0.78 of a two-tile item's).
constexpr int kWPair = 9, kWSingle = 7;
// Floats of one partial-result slot: O[QT][BM][D], m[QT][BM], l[QT][BM], the reference g_V.
constexpr int kSlotFloats = QT * BM * D + 2 * QT * BM + 4;

struct Cfg {
  static constexpr int kSoftmaxWarps = 4 * QT;
  // Warps are spread over the SM's four sub-partitions by index mod 4, and every sub-partition
  // holds two softmax warps.  The two light roles (producer, MMA issue) share sub-partition 0 and
  // the six dequant warps take two each on sub-partitions 1-3, so no softmax warp shares its
  // issue slots with the MMA warp.
  static constexpr int kProducerWarp = kSoftmaxWarps;      // warp 8
  static constexpr int kMmaWarp = kSoftmaxWarps + 4;       // warp 12
  // dequant warp index (0..5) of warp w in 9..15 other than the MMA warp
  __device__ static int dequant_index(int w) { return w < kMmaWarp ? w - kSoftmaxWarps - 1 : w - kSoftmaxWarps - 2; }
  static constexpr int kDequantWarps = 6;  // 2 in the producer/MMA warpgroup + one full warpgroup
  static constexpr int kDequantThreads = 32 * kDequantWarps;
  static_assert(kDequantThreads % 64 == 0, "dequant_tile deals blocks to a multiple of 64 threads");
  static constexpr int kThreads = 32 * (kSoftmaxWarps + 2 + kDequantWarps);  // whole warpgroups
  static_assert(kThreads == 512, "register split assumes four warpgroups");
  // TMEM columns: S sub-tile buffers S[q][b] at (2q + b) * SUB, O[q] at kTmemO + q * D.
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemO = 2 * QT * SUB;
  static_assert(kTmemO + QT * D <= kTmemCols, "TMEM budget");
  // shared memory map (bytes from a 1024-aligned base)
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + QT * TILE16;
  static constexpr int oV = oK + NST * TILE16;
  static constexpr int oPK = oV + NST * TILE16;
  // Per-tile column tables (fp32, BN each): K[j] = g_K(chunk) * scale * log2(e), L[j] = log2(cv),
  // I[j] = 1 / cv with cv = g_V(chunk) / max g_V (1 for an all-zero V chunk, whose V^ rows are 0);
  // masked columns K = 0, L = -inf, I = 0.  Plus int4 {n_valid, uniform}.  NCT slots.
  static constexpr int kColTab = 3 * BN * 4;
  static constexpr int oCol = oPK + NPK * PK_BYTES;
  static constexpr int oInfo = oCol + NCT * kColTab;
  static constexpr int oBar = oInfo + NCT * 16;
  // barrier indices
  static constexpr int bQFull = 0;                 // [QT] Q tile landed (TMA)
  static constexpr int bQReady = bQFull + QT;      // [QT] Q tile converted to fp16
  static constexpr int bPkFull = bQReady + QT;     // [NPK]
  static constexpr int bPkEmpty = bPkFull + NPK;   // [NPK]
  static constexpr int bKFull = bPkEmpty + NPK;    // [NST]
  static constexpr int bVFull = bKFull + NST;      // [NST]
  static constexpr int bKEmpty = bVFull + NST;     // [NST] K stage read by every QK of its tile
  static constexpr int bVEmpty = bKEmpty + NST;    // [NST] V stage read by every PV of its tile
  static constexpr int bTabFull = bVEmpty + NST;   // [NCT] column tables of a tile written
  static constexpr int bSFull = bTabFull + NCT;    // [QT] S of a whole KV tile computed
  static constexpr int bPFull = bSFull + QT;       // [QT][2] P sub-tile stored
  static constexpr int bODone = bPFull + 2 * QT;   // [QT][2] PV of a sub-tile complete
  static constexpr int bDrain = bODone + 2 * QT;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int oMisc = oBar + kNumBars * 8;  // [0] TMEM base, [1] abort flag
  static constexpr int kSmemBytes = oMisc + 16 + 1024;  // + slack for 1024-B alignment
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// The stream-K work split: units are (work item, KV tile) pairs, numbered item-major; a unit of
// a two-tile item costs wP, of a one-tile item wS.  CTA c takes the units whose weighted start
// lies in [c W / G, (c + 1) W / G).
struct Plan {
  int64_t units;  // bh * ipb * NT
  int64_t Wh;     // weighted cost of one (batch, head)
  int64_t W;      // bh * Wh
  int bh;         // batch * heads
  int n_qt;       // query tiles per (batch, head)
  int ipb;        // work items per (batch, head): ceil(n_qt / 2)
  int npairs;     // two-tile items per (batch, head): n_qt / 2
  int NT;         // KV tiles per item
  int wP, wS;
  int G;          // CTAs
};

// First unit of CTA c (c = G gives the end of the last range).
__host__ __device__ inline int64_t plan_cut(const Plan& p, int c) {
  if (c <= 0) return 0;
  if (c >= p.G) return p.units;
  const int64_t X = (p.W / p.G) * c + ((p.W % p.G) * c) / p.G;  // floor(W c / G)
  const int64_t h = X / p.Wh, r = X - h * p.Wh;
  const int64_t pw = static_cast<int64_t>(p.NT) * p.wP * p.npairs;
  int64_t u;
  if (r <= pw) u = (r + p.wP - 1) / p.wP;
  else u = static_cast<int64_t>(p.NT) * p.npairs + (r - pw + p.wS - 1) / p.wS;
  return h * p.ipb * static_cast<int64_t>(p.NT) + u;
}

// One segment of a CTA's range: the part of one work item between units u and uend.  Unit
// numbers stay below 2^31 (the launch checks it), so segments use 32-bit arithmetic.
struct Seg {
  int item;
  int t0, t1;  // KV tiles [t0, t1) of the item
  int bhi, m0, nq;
};

__host__ __device__ inline Seg plan_seg(const Plan& p, int u, int uend) {
  Seg s;
  s.item = u / p.NT;
  const int ib = s.item * p.NT;
  s.t0 = u - ib;
  s.t1 = (uend < ib + p.NT ? uend : ib + p.NT) - ib;
  s.bhi = s.item / p.ipb;
  const int k = s.item - s.bhi * p.ipb;
  s.m0 = 2 * k * BM;
  s.nq = (2 * k + 1 < p.n_qt) ? 2 : 1;
  return s;
}

__host__ __device__ inline int seg_end(const Plan& p, const Seg& s) { return s.item * p.NT + s.t1; }

struct AttnParams {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint8_t* k_scales;
  const uint8_t* v_scales;
  const float* k_g;
  const float* v_g;
  const float* k_mean;  // smoothed keys: [B*H][C][D] channel means, else null
  void* out;
  float* part;  // partial-result slots: [G][2][kSlotFloats]
  uint32_t* status;
  int64_t T;  // cached tokens per (b, h)
  int B, H, Lq, Lc, C;
  int out_bf16;
  int n_runs;
  int run_key0[MAX_RUNS];
  int run_key1[MAX_RUNS];
  int run_tile0[MAX_RUNS + 1];
  int n_tiles;
  float scale_log2;  // softmax scale * log2(e)
  Plan pl;
};

// ------------------------------------------------------------------ waits
__device__ __forceinline__ bool timed_out(uint64_t& t0, int& it) {
  const uint64_t now = ptx::globaltimer_ns();
  if (it++ == 0) t0 = now;
  return now - t0 > kWaitLimitNs;
}

// Single-thread wait; gives up when another thread aborted or the limit is reached.
__device__ __forceinline__ bool wait1(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                      uint32_t* status) {
  uint64_t t0 = 0;
  int it = 0;
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (timed_out(t0, it)) {
      *abort = 1;
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// Warp-collective wait: every lane observes the phase; the give-up decision is uniform.
__device__ __forceinline__ bool waitw(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                      uint32_t* status) {
  const int lane = threadIdx.x & 31;
  uint64_t t0 = 0;
  int it = 0;
  while (true) {
    const bool ok = ptx::mbar_try_wait(bar, parity);
    if (__all_sync(0xFFFFFFFFu, ok)) return true;
    uint32_t give_up = 0;
    if (lane == 0) {
      if (*abort) {
        give_up = 1;
      } else if (timed_out(t0, it)) {
        *abort = 1;
        atomicOr(status, kStatusTimeout);
        give_up = 1;
      }
    }
    if (__shfl_sync(0xFFFFFFFFu, give_up, 0)) return false;
  }
}

// Exit-path wait for work that is known to finish (copies or MMAs already issued).
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity, uint32_t* status) {
  uint64_t t0 = 0;
  int it = 0;
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (timed_out(t0, it)) {
      atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

__device__ __forceinline__ void tile_keys(const AttnParams& p, int j, int& key0, int& n) {
  int r = 0;
  while (r + 1 < p.n_runs && j >= p.run_tile0[r + 1]) ++r;
  key0 = p.run_key0[r] + (j - p.run_tile0[r]) * BN;
  n = min(BN, p.run_key1[r] - key0);
}

__device__ __forceinline__ float max_visible_gv(const AttnParams& p, int64_t bh) {
  float m = 0.0f;
  for (int r = 0; r < p.n_runs; ++r)
    for (int c = p.run_key0[r] / p.Lc; c < p.run_key1[r] / p.Lc; ++c)
      m = fmaxf(m, p.v_g[bh * p.C + c]);
  return m > 0.0f ? m : 1.0f;
}

// q' . mu for one query row: q' is the row's prescaled fp16 copy in the 128B-swizzled Q tile
// (16-byte chunk j of half hf at position j ^ (row % 8)), mu a chunk's fp32 channel means.
__device__ __forceinline__ float q_dot_mean(const uint8_t* qrow, int row, const float* mu) {
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    // a quarter's 32 means first (8 independent loads in flight), then its 32 products
    float4 m[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = __ldg(reinterpret_cast<const float4*>(mu + qq * 32) + k);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int hf = qq >> 1, j = (qq & 1) * 4 + jj;  // 16-byte chunk j of half hf
      const uint4 v = *reinterpret_cast<const uint4*>(qrow + hf * HALF16 + ((j ^ (row & 7)) << 4));
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
      const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
      const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&v.z));
      const float2 f3 = __half22float2(*reinterpret_cast<const __half2*>(&v.w));
      const float4 m0 = m[2 * jj], m1 = m[2 * jj + 1];
      acc[jj] = fmaf(f0.x, m0.x, fmaf(f0.y, m0.y, fmaf(f1.x, m0.z, fmaf(f1.y, m0.w, acc[jj]))));
      acc[jj] = fmaf(f2.x, m1.x, fmaf(f2.y, m1.y, fmaf(f3.x, m1.z, fmaf(f3.y, m1.w, acc[jj]))));
    }
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
  return __vmaxu2(a & 0x7FFF7FFFu, b & 0x7FFF7FFFu);
}

// Dequantise one packed tile (codes + E4M3 scales of BN keys) into a 128B-swizzled [key][d]
// operand tile of fp16 values, code * scale (exact: <= 6 significant bits, 2^-10 .. 2688).
// Thread dt of NT owns the 16-element block blk = dt % 8 of keys dt / 8 + (NT / 8) * it: NT / 8 is
// a multiple of 8, so the block, the swizzle phase key % 8 and the store order are fixed per
// thread and every address is a per-thread base plus a constant.  All
// shared-memory loads are issued first.  A 16-byte warp store is served in phases of 8 lanes (one
// key, all eight blocks): lanes of the second 64-element half store their odd chunk first, so the
// 8 lanes of a phase hit 8 distinct banks.  Keys >= n (past the run's end) are written as zeros.
template <int NT, bool kFull>
__device__ __forceinline__ void dequant_tile(const uint8_t* pk, uint8_t* dst, int n, int dt) {
  static_assert(NT % 64 == 0, "keys per pass must be a multiple of 8");
  constexpr int KS = NT / 8;               // keys per pass: 24 for 192 threads
  constexpr int kIt = (BN + KS - 1) / KS;  // passes; the last one may cover only part of the keys
  const int blk = dt & 7, kq = dt >> 3;
  const bool swap = blk >= 4;
  const int c0 = (blk & 3) * 2;
  const uint8_t* csrc = pk + kq * kCodeBytes + blk * 8;
  const uint8_t* ssrc = pk + PK_CODES + kq * kScaleBytes + blk;
  uint8_t* const row = dst + (blk >> 2) * HALF16 + kq * 128;
  uint8_t* const dA = row + (((c0 + (swap ? 1 : 0)) ^ (kq & 7)) << 4);  // first store
  uint8_t* const dB = row + (((c0 + (swap ? 0 : 1)) ^ (kq & 7)) << 4);
  const bool tail = kq + KS * (kIt - 1) < BN;  // this thread has a key in the last pass
  uint2 w[kIt];
  uint32_t sb[kIt];
#pragma unroll
  for (int it = 0; it < kIt; ++it) {
    if (it < kIt - 1 || tail) {
      w[it] = *reinterpret_cast<const uint2*>(csrc + it * KS * kCodeBytes);
      sb[it] = ssrc[it * KS * kScaleBytes];
    }
  }
#pragma unroll
  for (int it = 0; it < kIt; ++it) {
    if (it == kIt - 1 && !tail) break;
    const uint32_t s2 = ptx::e4m3_to_f16x2_bcast(sb[it]);
    const uint32_t first = swap ? w[it].y : w[it].x, second = swap ? w[it].x : w[it].y;
    uint32_t h[4], g[4];
    ptx::e2m1x8_to_f16x8(first, h);
    ptx::e2m1x8_to_f16x8(second, g);
    uint4 oA = make_uint4(ptx::hmul2_u32(h[0], s2), ptx::hmul2_u32(h[1], s2), ptx::hmul2_u32(h[2], s2),
                          ptx::hmul2_u32(h[3], s2));
    uint4 oB = make_uint4(ptx::hmul2_u32(g[0], s2), ptx::hmul2_u32(g[1], s2), ptx::hmul2_u32(g[2], s2),
                          ptx::hmul2_u32(g[3], s2));
    if (!kFull && kq + KS * it >= n) {
      oA = make_uint4(0, 0, 0, 0);
      oB = oA;
    }
    *reinterpret_cast<uint4*>(dA + it * KS * 128) = oA;
    *reinterpret_cast<uint4*>(dB + it * KS * 128) = oB;
  }
}

// kSmooth: the cache's keys are smoothed (p.k_mean is set); the plain kernel carries no trace of
// the per-chunk mean terms.
template <bool kSmooth>
__global__ void __launch_bounds__(Cfg::kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ AttnParams p) {
  using C = Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  // This CTA's range of (item, KV tile) units; every role walks the same segments.
  const int ubeg = static_cast<int>(plan_cut(p.pl, cta)), uend = static_cast<int>(plan_cut(p.pl, cta + 1));
  // the merge kernel may be scheduled now; it waits for this whole grid before reading anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int n_dq_warps = C::kDequantWarps;

  const uint32_t sbase = ptx::smem_u32(smem);
  auto bar = [&](int i) { return sbase + C::oBar + 8 * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::oMisc);
  volatile uint32_t* abort_flag = misc + 1;

  if (threadIdx.x == 0) {
    for (int q = 0; q < QT; ++q) {
      ptx::mbar_init(bar(C::bQFull + q), 1);
      ptx::mbar_init(bar(C::bQReady + q), 4);
      ptx::mbar_init(bar(C::bSFull + q), 1);
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(bar(C::bPFull + 2 * q + b), 4);
        ptx::mbar_init(bar(C::bODone + 2 * q + b), 1);
      }
    }
    for (int i = 0; i < NPK; ++i) {
      ptx::mbar_init(bar(C::bPkFull + i), 1);
      ptx::mbar_init(bar(C::bPkEmpty + i), n_dq_warps);
    }
    for (int i = 0; i < NST; ++i) {
      ptx::mbar_init(bar(C::bKFull + i), n_dq_warps);
      ptx::mbar_init(bar(C::bVFull + i), n_dq_warps);
      ptx::mbar_init(bar(C::bKEmpty + i), 1);
      ptx::mbar_init(bar(C::bVEmpty + i), 1);
    }
    for (int i = 0; i < NCT; ++i) ptx::mbar_init(bar(C::bTabFull + i), n_dq_warps);
    ptx::mbar_init(bar(C::bDrain), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == C::kMmaWarp) {
    ptx::tmem_alloc(sbase + C::oMisc, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc[0];
  // Registers move from the producer/MMA/dequant warpgroups (88 each) to the two softmax
  // warpgroups (168 each): 2*128*168 + 2*128*88 = 65536, exactly what the 512-thread block was
  // launched with.  Each role branch starts with its warpgroup's budget change.

  if (warp < C::kSoftmaxWarps) {
    // ============================================================ softmax + epilogue
    ptx::setmaxnreg_inc<168>();
    const int qt = warp >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS0 = tmem + lane_off + (2 * qt) * SUB;
    const uint32_t tO = tmem + lane_off + C::kTmemO + qt * D;
    const bool issuer = wq == 0 && lane == 0;
    uint8_t* const qbase = smem + C::oQ + qt * TILE16;
    // The Q tile of the next segment this warpgroup takes part in, loaded by one thread.
    auto issue_q = [&](int from) {
      for (int u = from; u < uend;) {
        const Seg s = plan_seg(p.pl, u, uend);
        if (qt < s.nq) {
          if (issuer) {
            const int hh = s.bhi % p.H, bb = s.bhi / p.H;
            ptx::mbar_arrive_expect_tx(bar(C::bQFull + qt), TILE16);
            for (int half = 0; half < 2; ++half)
              ptx::tma_load_4d(sbase + C::oQ + qt * TILE16 + half * HALF16, &tmap_q, half * 64, hh,
                               s.m0 + qt * BM, bb, bar(C::bQFull + qt));
          }
          return true;
        }
        u = seg_end(p.pl, s);
      }
      return false;
    };
    if (issuer) ptx::prefetch_tmap(&tmap_q);
    bool q_pending = issue_q(ubeg);
    bool ok = true;
    int sq = 0;        // segments this warpgroup took part in
    int g = 0;         // S sub-tiles this warpgroup processed (parity of its S/P/O barriers)
    int jjb = 0;       // KV tiles of the CTA before the current segment
    for (int u = ubeg; u < uend && ok;) {
      const Seg s = plan_seg(p.pl, u, uend);
      const int unext = seg_end(p.pl, s);
      const int ntl = s.t1 - s.t0;
      if (qt >= s.nq) {
        jjb += ntl;
        u = unext;
        continue;
      }
      const int h = s.bhi % p.H, b = s.bhi / p.H;
      const int64_t bh = static_cast<int64_t>(b) * p.H + h;
      ok = waitw(bar(C::bQFull + qt), sq & 1, abort_flag, p.status);
      if (!ok) break;
      q_pending = false;
      // ---- Q row: bf16 -> fp16 in place after a power-of-two prescale 2^-e that brings the row's
      // largest |q| into [2^14, 2^15) (e = floor(log2 max|q|) - 14, clamped to [-126, 113] so 2^e
      // and 2^-e are normal floats); row i of S depends on row i of Q only, so each thread scales
      // its own row and scales its S row back by 2^e with the logit factor.  The conversion is
      // exact for every element within 2^-28 of the row's largest (fp16's normal range holds
      // bf16's 8 significant bits); smaller ones round to fp16's subnormal spacing, an absolute
      // error of at most 2^-39 of the row's largest |q|.  No thread waits for another here.
      float q_unscale = 1.0f, pre_scale = 1.0f;
      uint8_t* qrow = qbase + row * 128;
      {
        uint32_t mb = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(qrow + (i >> 3) * HALF16 + (((i + lane) & 7) << 4));
          mb = __vmaxu2(mb, __vmaxu2(absmax_bf16x2(v.x, v.y), absmax_bf16x2(v.z, v.w)));
        }
        mb = max(mb & 0xFFFFu, mb >> 16);
        const int ex = static_cast<int>((mb >> 7) & 0xFF) - 127;  // floor(log2 max|q|)
        const int e = min(max(ex - 14, -126), 113);
        q_unscale = __int_as_float((127 + e) << 23);  // 2^e
        pre_scale = __int_as_float((127 - e) << 23);  // 2^-e
      }
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        uint4* ptr = reinterpret_cast<uint4*>(qrow + (i >> 3) * HALF16 + (((i + lane) & 7) << 4));
        const uint4 v = *ptr;
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          o[k] = ptx::f32x2_to_f16x2(__uint_as_float(wv[k] << 16) * pre_scale,
                                     __uint_as_float(wv[k] & 0xFFFF0000u) * pre_scale);
        *ptr = make_uint4(o[0], o[1], o[2], o[3]);
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(C::bQReady + qt));

      const float gv_ref = max_visible_gv(p, bh);
      float m_run = -INFINITY, l_run = 0.0f;
      // smoothed keys: the logit term scale * log2(e) * q . mu of the (at most two) chunks of the
      // current KV tile, computed when a chunk is first met in this segment
      int c_lo = -1;          // chunk of b_lo; b_hi (when hi_ok) belongs to chunk c_lo + 1
      bool hi_ok = false;
      float b_lo = 0.0f, b_hi = 0.0f;
      const int nh = 2 * ntl;
      for (int hs = 0; hs < nh && ok; ++hs, ++g) {
        const int jj = jjb + (hs >> 1);
        const int bf = g & 1, half = hs & 1;
        const uint32_t tS = tS0 + bf * SUB;
        // S of the whole KV tile arrives with its first sub-tile
        if (half == 0)
          ok = waitw(bar(C::bSFull + qt), (g >> 1) & 1, abort_flag, p.status) &&
               waitw(bar(C::bTabFull + jj % NCT), (jj / NCT) & 1, abort_flag, p.status);
        if (!ok) break;
        ptx::tc_fence_after();
        const int ct = static_cast<int>(jj % NCT);
        const int4 info = *reinterpret_cast<const int4*>(smem + C::oInfo + 16 * ct);
        const float* colK = reinterpret_cast<const float*>(smem + C::oCol + ct * C::kColTab) + half * SUB;
        const float* colL = colK + BN;
        const float* colI = colK + 2 * BN;
        // A tile inside one chunk with every key valid takes the uniform path (one logit factor,
        // one cv); any other tile works per column with the same arithmetic.
        const bool uni = info.y != 0;
        // chunk info.z holds columns [0, info.w), chunk info.z + 1 the valid columns after them
        if (kSmooth && half == 0 && (info.z != c_lo || (info.w < BN && !hi_ok))) {
          // a new chunk: at most two per tile, and the tiles of a segment ascend
          const float* const mu_bh = p.k_mean + bh * p.C * D;
          const float f = p.scale_log2 * q_unscale;
          if (info.z != c_lo) {
            b_lo = (hi_ok && info.z == c_lo + 1) ? b_hi : f * q_dot_mean(qrow, row, mu_bh + info.z * D);
            c_lo = info.z;
            hi_ok = false;
          }
          if (info.w < BN && !hi_ok) {
            b_hi = f * q_dot_mean(qrow, row, mu_bh + (c_lo + 1) * D);
            hi_ok = true;
          }
        }
        const int jsplit = kSmooth ? info.w - half * SUB : 0;  // first column here in chunk info.z + 1

        uint32_t sr[2][32];
        ptx::tmem_ld32(tS, sr[0]);
        ptx::tmem_ld32(tS + 32, sr[1]);
        ptx::tc_wait_ld_regs(sr[0]);
        ptx::reg_fence32(sr[1]);

        // Row maximum of x = S * g_K(chunk) * scale * log2(e) + log2(cv) (masked keys -inf); the
        // reference m only has to bound the exponents of P~ = 2^(x - m), which include cv.
        float mx;
        float ck = 0.0f, lc = 0.0f;
        if (uni) {
          ck = colK[0] * q_unscale;
          lc = kSmooth ? colL[0] + b_lo : colL[0];
          float m8[8];  // eight independent max chains
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = -INFINITY;
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const int k = 4 * c + ((i >> 2) & 1) * 2;
              m8[k] = ptx::fmax3(m8[k], __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]));
              m8[k + 1] = ptx::fmax3(m8[k + 1], __uint_as_float(sr[c][i + 2]), __uint_as_float(sr[c][i + 3]));
            }
          mx = fmaf(fmaxf(ptx::fmax3(m8[0], m8[1], m8[2]), ptx::fmax3(m8[3], m8[4], ptx::fmax3(m8[5], m8[6], m8[7]))),
                    ck, lc);
        } else {
          // x in place of S: x = S * K[j] * 2^e + L[j]
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              asm volatile("" ::: "memory");  // keep the table loads next to their use (registers)
              const float4 kk = *reinterpret_cast<const float4*>(colK + 32 * c + i);
              const float4 ll = *reinterpret_cast<const float4*>(colL + 32 * c + i);
              float4 l4 = ll;
              if (kSmooth) {  // the mean term of each column's chunk
                const int jc = 32 * c + i;  // column within the sub-tile
                l4.x += jc < jsplit ? b_lo : b_hi;
                l4.y += jc + 1 < jsplit ? b_lo : b_hi;
                l4.z += jc + 2 < jsplit ? b_lo : b_hi;
                l4.w += jc + 3 < jsplit ? b_lo : b_hi;
              }
              const float x0 = fmaf(__uint_as_float(sr[c][i]), kk.x * q_unscale, l4.x);
              const float x1 = fmaf(__uint_as_float(sr[c][i + 1]), kk.y * q_unscale, l4.y);
              const float x2 = fmaf(__uint_as_float(sr[c][i + 2]), kk.z * q_unscale, l4.z);
              const float x3 = fmaf(__uint_as_float(sr[c][i + 3]), kk.w * q_unscale, l4.w);
              sr[c][i] = __float_as_uint(x0);
              sr[c][i + 1] = __float_as_uint(x1);
              sr[c][i + 2] = __float_as_uint(x2);
              sr[c][i + 3] = __float_as_uint(x3);
              m4[(i >> 2) & 3] = fmaxf(m4[(i >> 2) & 3], ptx::fmax3(x0, x1, fmaxf(x2, x3)));
            }
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
        // Lazy rescale: the reference m only moves (to a whole number, so the rescale is an exact
        // power of two) when the row maximum exceeds it by more than 2^14; P~ = 2^(x - m) then stays
        // below 2^14 (fp16 holds up to 65504), and an O rescale, which waits for the tile's P V,
        // is rare.  The O rescale uses
        // warp-collective TMEM accesses, so it runs for the whole warp when any row moved
        // (alpha = 1 for the rows that did not).
        const bool grow = mx > m_run + 14.0f;
        if (__any_sync(0xFFFFFFFFu, grow)) {
          const float m_new = grow ? ceilf(mx) : m_run;
          const float alpha = grow ? ptx::ex2(m_run - m_new) : 1.0f;  // 0 while m is -inf
          l_run *= alpha;
          m_run = m_new;
          if (hs > 0) {  // O holds sub-tiles < hs of this segment once PV(g - 1) is complete
            ok = waitw(bar(C::bODone + 2 * qt + ((g - 1) & 1)), ((g - 1) >> 1) & 1, abort_flag, p.status);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll 1
            for (int oc = 0; oc < 8; ++oc) {  // 16 columns at a time: the S row stays in registers
              uint32_t o[16];
              ptx::tmem_ld16_wait(tO + 16 * oc, o);
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              ptx::tmem_st16p(tO + 16 * oc, o);
            }
          }
        }

        // P~ = 2^(x - m) (x includes log2(cv)), rounded to fp16 pairs and stored over the
        // sub-tile's first 32 S columns.  The row sum adds the same rounded values times 1 / cv,
        // so the rounding largely cancels in O / l.
        if (uni) {
          // x - m = S * ck + (log2(cv) - m) in packed pairs; eight independent row-sum chains.
          const float mneg = lc - m_run;
          float l8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) l8[k] = 0.0f;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float x0, x1;
              ptx::ffma2(x0, x1, __uint_as_float(sr[c][2 * i]), __uint_as_float(sr[c][2 * i + 1]), ck, mneg);
              pk[i] = ptx::f32x2_to_f16x2(ptx::ex2(x0), ptx::ex2(x1));
              l8[i & 7] = ptx::add_f16x2_f32(l8[i & 7], pk[i]);
            }
            ptx::tmem_st16p(tS + 16 * c, pk);
          }
          l_run = fmaf((((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]))), colI[0], l_run);
        } else {
          float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              asm volatile("" ::: "memory");
              const float4 iv = *reinterpret_cast<const float4*>(colI + 32 * c + 2 * i);
              const float p0 = ptx::ex2(__uint_as_float(sr[c][2 * i]) - m_run);
              const float p1 = ptx::ex2(__uint_as_float(sr[c][2 * i + 1]) - m_run);
              const float p2 = ptx::ex2(__uint_as_float(sr[c][2 * i + 2]) - m_run);
              const float p3 = ptx::ex2(__uint_as_float(sr[c][2 * i + 3]) - m_run);
              pk[i] = ptx::f32x2_to_f16x2(p0, p1);
              pk[i + 1] = ptx::f32x2_to_f16x2(p2, p3);
              const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&pk[i]));
              const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&pk[i + 1]));
              l4[0] = fmaf(h0.x, iv.x, l4[0]);
              l4[1] = fmaf(h0.y, iv.y, l4[1]);
              l4[2] = fmaf(h1.x, iv.z, l4[2]);
              l4[3] = fmaf(h1.y, iv.w, l4[3]);
            }
            ptx::tmem_st16p(tS + 16 * c, pk);
          }
          l_run += (l4[0] + l4[1]) + (l4[2] + l4[3]);
        }
        ptx::tc_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(C::bPFull + 2 * qt + bf));
      }
      if (!ok) break;
      // ---- epilogue: PV of the last sub-tile (and so every MMA of the segment) is complete
      ok = waitw(bar(C::bODone + 2 * qt + ((g - 1) & 1)), ((g - 1) >> 1) & 1, abort_flag, p.status);
      if (!ok) break;
      ptx::tc_fence_after();
      ++sq;
      // Q of this segment is no longer read: load the next segment's Q behind the epilogue.
      q_pending = issue_q(unext);
      const int qrow_i = s.m0 + qt * BM + row;
      const bool store = qrow_i < p.Lq;
      const bool full = s.t0 == 0 && s.t1 == p.pl.NT;
      if (full) {
        const float inv = gv_ref / l_run;
        const int64_t obase = ((static_cast<int64_t>(b) * p.Lq + qrow_i) * p.H + h) * D;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          ptx::tmem_ld32(tO + 32 * c, r);
          ptx::tc_wait_ld();
          if (store) {
            if (p.out_bf16) {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + obase + 32 * c);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                uint32_t w[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(r[8 * i + 2 * k]) * inv,
                                                            __uint_as_float(r[8 * i + 2 * k + 1]) * inv);
                  w[k] = *reinterpret_cast<uint32_t*>(&v2);
                }
                dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + obase + 32 * c);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                                     __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv);
            }
          }
        }
      } else {
        // Partial result: unnormalised O, the reference max and the running sum of this range.
        const int slot = 2 * cta + (u == ubeg ? 0 : 1);
        float* sp = p.part + static_cast<int64_t>(slot) * kSlotFloats;
        float4* dst = reinterpret_cast<float4*>(sp + (qt * BM + row) * D);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          ptx::tmem_ld32(tO + 32 * c, r);
          ptx::tc_wait_ld();
          if (store) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[8 * c + i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                           __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
          }
        }
        if (store) {
          sp[QT * BM * D + qt * BM + row] = m_run;
          sp[QT * BM * D + QT * BM + qt * BM + row] = l_run;
        }
        if (qt == 0 && row == 0) sp[QT * BM * D + 2 * QT * BM] = gv_ref;
      }
      jjb += ntl;
      u = unext;
    }
    if (!ok && q_pending && issuer) wait_drain(bar(C::bQFull + qt), sq & 1, p.status);
  } else {
    ptx::setmaxnreg_dec<88>();
    if (warp == C::kProducerWarp) {
      // ========================================================== TMA producer (packed K/V)
      if (lane == 0) {
        int issued = 0, pk = 0;
        bool ok = true;
        for (int u = ubeg; u < uend && ok;) {
          const Seg s = plan_seg(p.pl, u, uend);
          const int64_t bh = s.bhi;
          const uint8_t* kc = p.k_codes + bh * p.T * kCodeBytes;
          const uint8_t* vc = p.v_codes + bh * p.T * kCodeBytes;
          const uint8_t* ks = p.k_scales + bh * p.T * kScaleBytes;
          const uint8_t* vs = p.v_scales + bh * p.T * kScaleBytes;
          for (int j = s.t0; j < s.t1 && ok; ++j) {
            int key0, n;
            tile_keys(p, j, key0, n);
            for (int t = 0; t < 2; ++t, ++pk) {
              const int slot = static_cast<int>(pk % NPK);
              ok = wait1(bar(C::bPkEmpty + slot), static_cast<uint32_t>((pk / NPK) & 1) ^ 1u, abort_flag, p.status);
              if (!ok) break;
              const uint32_t dst = sbase + C::oPK + slot * PK_BYTES;
              ptx::mbar_arrive_expect_tx(bar(C::bPkFull + slot), n * (kCodeBytes + kScaleBytes));
              ptx::bulk_g2s(dst, (t == 0 ? kc : vc) + static_cast<int64_t>(key0) * kCodeBytes,
                            n * kCodeBytes, bar(C::bPkFull + slot));
              ptx::bulk_g2s(dst + PK_CODES, (t == 0 ? ks : vs) + static_cast<int64_t>(key0) * kScaleBytes,
                            n * kScaleBytes, bar(C::bPkFull + slot));
              issued = pk + 1;
            }
          }
          u = seg_end(p.pl, s);
        }
        if (!ok) {  // let every copy already issued land before the CTA can exit
          for (int k = std::max(0, issued - NPK); k < issued; ++k)
            wait_drain(bar(C::bPkFull + static_cast<int>(k % NPK)), static_cast<uint32_t>((k / NPK) & 1), p.status);
        }
      }
      __syncwarp();
    } else if (warp == C::kMmaWarp) {
      // ========================================================== MMA issuer
      // The whole warp runs this loop with warp-uniform values; one elected lane issues each
      // tcgen05 instruction.  kind::f16 instruction descriptors: fp16 x fp16 -> fp32; M = 128.
      constexpr uint32_t kIdescQK = (1u << 4) |  // A = Q and B = K^ both K-major; N = 128 keys
                                    (static_cast<uint32_t>(BN >> 3) << 17) |
                                    (static_cast<uint32_t>(BM >> 4) << 24);
      constexpr uint32_t kIdescPV = (1u << 4) | (1u << 16) |  // B = V^ MN-major; N = 128 dims
                                    (static_cast<uint32_t>(D >> 3) << 17) |
                                    (static_cast<uint32_t>(BM >> 4) << 24);
      // Shared-memory descriptors are built once; a step only advances the 14-bit start address
      // field (address >> 4).  Sub-tile `half` of a V stage starts 64 rows (8 KB) in.
      const uint64_t dQ0 = ptx::smem_desc_sw128(sbase + C::oQ, 16, 1024);
      const uint64_t dK0 = ptx::smem_desc_sw128(sbase + C::oK, 16, 1024);
      const uint64_t dV0 = ptx::smem_desc_sw128(sbase + C::oV, HALF16, 1024);
      // S = Q K^T of a whole KV tile (N = 128) into both S sub-buffers of query tile q
      auto issue_qk = [&](int q, int st) {
        const uint64_t dQ = dQ0 + static_cast<uint64_t>((q * TILE16) >> 4);
        const uint64_t dK = dK0 + static_cast<uint64_t>((st * TILE16) >> 4);
        ptx::mma_qk8_w(tmem + (2 * q) * SUB, dQ, dK, kIdescQK, 0u);
        ptx::mma_commit_w(bar(C::bSFull + q));
      };
      auto issue_pv = [&](int q, int bf, int st, int half, uint32_t acc) {
        const uint64_t dV = dV0 + static_cast<uint64_t>((st * TILE16 + half * SUB * 128) >> 4);
        ptx::mma_pv4_w(tmem + C::kTmemO + q * D, tmem + (2 * q + bf) * SUB, dV, kIdescPV, acc);
        ptx::mma_commit_w(bar(C::bODone + 2 * q + bf));
      };
      int gq[QT] = {0, 0}, sq[QT] = {0, 0};
      int jjb = 0;
      bool ok = true;
      for (int u = ubeg; u < uend && ok;) {
        const Seg s = plan_seg(p.pl, u, uend);
        const int ntl = s.t1 - s.t0, nq = s.nq, nh = 2 * ntl;
        for (int q = 0; q < nq && ok; ++q) ok = waitw(bar(C::bQReady + q), sq[q] & 1, abort_flag, p.status);
        const int st0 = static_cast<int>(jjb % NST);
        if (ok) ok = waitw(bar(C::bKFull + st0), static_cast<uint32_t>((jjb / NST) & 1), abort_flag, p.status);
        if (!ok) break;
        ptx::tc_fence_after();
        for (int q = 0; q < nq; ++q) issue_qk(q, st0);  // the segment's first KV tile
        ptx::mma_commit_w(bar(C::bKEmpty + st0));
        // Per sub-tile hs: PV(q, hs) as soon as softmax q has written P(q, hs); after the second
        // sub-tile of a KV tile, QK(q) of the next KV tile into the S buffers those PVs have read
        // (issue order keeps it behind them).  The two query tiles alternate.
        for (int hs = 0; hs < nh && ok; ++hs) {
          const int jt = jjb + (hs >> 1);
          const int st = static_cast<int>(jt % NST), half = hs & 1;
          for (int q = 0; q < nq; ++q) {
            const int gg = gq[q] + hs, bf = gg & 1;
            ok = waitw(bar(C::bPFull + 2 * q + bf), (gg >> 1) & 1, abort_flag, p.status);
            if (ok && q == 0 && half == 0) ok = waitw(bar(C::bVFull + st), static_cast<uint32_t>((jt / NST) & 1), abort_flag, p.status);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_pv(q, bf, st, half, hs > 0 ? 1u : 0u);
            if (q == nq - 1 && half == 1) ptx::mma_commit_w(bar(C::bVEmpty + st));
            if (half == 1 && hs + 1 < nh) {
              const int st1 = static_cast<int>((jt + 1) % NST);
              if (q == 0) {
                ok = waitw(bar(C::bKFull + st1), static_cast<uint32_t>(((jt + 1) / NST) & 1), abort_flag, p.status);
                if (!ok) break;
                ptx::tc_fence_after();
              }
              issue_qk(q, st1);
              if (q == nq - 1) ptx::mma_commit_w(bar(C::bKEmpty + st1));
            }
          }
        }
        for (int q = 0; q < nq; ++q) {
          gq[q] += nh;
          ++sq[q];
        }
        jjb += ntl;
        u = seg_end(p.pl, s);
      }
      // every MMA issued so far completes before the drain barrier's phase 0
      ptx::mma_commit_w(bar(C::bDrain));
      if (lane == 0) wait_drain(bar(C::bDrain), 0, p.status);
      __syncwarp();
    } else {
      // ========================================================== dequant warps
      // No barrier among the dequant warps: each works through the same tiles on its own, so a
      // warp that gives up after a time-out never leaves the others waiting.
      const int dt = C::dequant_index(warp) * 32 + lane;
      float inv_gv = 1.0f;
      int jj = 0;
      bool ok = true;
      for (int u = ubeg; u < uend && ok;) {
        const Seg s = plan_seg(p.pl, u, uend);
        const int64_t bh = s.bhi;
        inv_gv = 1.0f / max_visible_gv(p, bh);
        for (int j = s.t0; j < s.t1 && ok; ++j, ++jj) {
          const int st = static_cast<int>(jj % NST);
          int key0, n;
          tile_keys(p, j, key0, n);
          // The FP32 scales of this thread's key for the per-column tables, loaded before the waits.
          float gk = 0.0f, gvv = 0.0f;
          if (dt < n) {
            const int64_t c = bh * p.C + (key0 + dt) / p.Lc;
            gk = p.k_g[c] * p.scale_log2;
            gvv = p.v_g[c] * inv_gv;
            if (!(gvv > 0.0f)) gvv = 1.0f;  // an all-zero V chunk: V^ rows are 0, P only counts in l
          }
          for (int t = 0; t < 2 && ok; ++t) {
            // the stage's previous tile (jj - NST) is done with it: K after its QKs, V after its PVs
            if (jj >= NST)
              ok = waitw(bar((t == 0 ? C::bKEmpty : C::bVEmpty) + st), static_cast<uint32_t>(((jj / NST) - 1) & 1),
                         abort_flag, p.status);
            if (!ok) break;
            const int pk = 2 * jj + t;
            const int slot = static_cast<int>(pk % NPK);
            ok = waitw(bar(C::bPkFull + slot), static_cast<uint32_t>((pk / NPK) & 1), abort_flag, p.status);
            if (!ok) break;
            const uint8_t* src = smem + C::oPK + slot * PK_BYTES;
            uint8_t* dst = smem + (t == 0 ? C::oK : C::oV) + st * TILE16;
            if (n == BN) dequant_tile<C::kDequantThreads, true>(src, dst, n, dt);
            else dequant_tile<C::kDequantThreads, false>(src, dst, n, dt);
            if (t == 0 && dt < BN) {  // per-column tables: one thread per key of the tile
              const int ct = static_cast<int>(jj % NCT);
              float* colK = reinterpret_cast<float*>(smem + C::oCol + ct * C::kColTab);
              const bool valid = dt < n;
              colK[dt] = gk;
              colK[BN + dt] = valid ? __log2f(gvv) : -INFINITY;
              colK[2 * BN + dt] = valid ? __frcp_rn(gvv) : 0.0f;
              if (dt == 0) {
                const int c0 = key0 / p.Lc;
                const int uniform = (n == BN) && (c0 == (key0 + BN - 1) / p.Lc);
                const int split = (c0 + 1) * p.Lc - key0;  // first column in chunk c0 + 1
                *reinterpret_cast<int4*>(smem + C::oInfo + 16 * ct) = make_int4(n, uniform, c0, split < n ? split : BN);
              }
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              ptx::mbar_arrive(bar(C::bPkEmpty + slot));
              ptx::mbar_arrive(bar(t == 0 ? C::bKFull + st : C::bVFull + st));
              if (t == 0) ptx::mbar_arrive(bar(C::bTabFull + static_cast<int>(jj % NCT)));
            }
          }
        }
        u = seg_end(p.pl, s);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Merges the partial results of every work item whose KV tiles were split between CTAs.  Blocks
// (b - 1, rg) look at the boundary between CTAs b - 1 and b; the first boundary inside an item merges
// that item, rows [16 rg, 16 rg + 16) of its query rows, one warp per row (each lane owns 4 of the
// 128 columns; lane i loads the running max and sum of part i):
//   m* = max_k m_k;  O = sum_k O_k 2^(m_k - m*);  l = sum_k l_k 2^(m_k - m*);  out = O g_ref / l
// (the m_k are whole numbers, so every factor is an exact power of two).  Launched as a
// programmatic dependent of the attention grid: it waits for that grid before reading partials.
constexpr int kCombineRows = 32;  // rows of one split item per CTA: 8 warps x 4 rows
constexpr int kCombineParts = 4;  // parts merged with all their loads in flight at once

// One split item's 16 rows: the parts' (m, l, O) rows are all loaded before any is used, so a row
// costs one round trip to L2 (items split into more than kCombineParts parts loop).
__global__ void __launch_bounds__(32 * kCombineRows / 4) combine_kernel(const __grid_constant__ AttnParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const Plan& pl = p.pl;
  const int bnd = blockIdx.x + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int slots[kMaxCtas];
  __shared__ int n_slots;
  __shared__ int s_item;
  if (warp == 0) {
    // the item split at cut bnd and the CTAs whose ranges meet it: lane i looks at CTA bnd - 1 + i
    const int64_t u = plan_cut(pl, bnd);
    const bool split = u < pl.units && u % pl.NT != 0;
    const int64_t item = u / pl.NT, istart = item * pl.NT, iend = istart + pl.NT;
    int n = 0;
    // only the item's first cut merges it (an earlier cut inside the same item leaves it alone)
    if (split && plan_cut(pl, bnd - 1) <= istart) {
      for (int base = bnd - 1; base < pl.G; base += 32) {
        const int c = base + lane;
        const int64_t cs = c < pl.G ? plan_cut(pl, c) : iend, ce = c < pl.G ? plan_cut(pl, c + 1) : iend;
        const bool meets = c < pl.G && cs < iend && ce > istart && cs < ce;
        const unsigned mask = __ballot_sync(0xFFFFFFFFu, meets);
        if (meets) slots[n + __popc(mask & ((1u << lane) - 1u))] = 2 * c + (cs < istart ? 1 : 0);
        n += __popc(mask);
        if (__any_sync(0xFFFFFFFFu, c < pl.G && cs >= iend)) break;
      }
    }
    if (lane == 0) {
      n_slots = n;
      s_item = static_cast<int>(item);
    }
  }
  __syncthreads();
  const int ns = n_slots;
  if (ns == 0) return;
  const int item = s_item;
  const int bhi = item / pl.ipb, k = item % pl.ipb;
  const int m0 = 2 * k * BM, nq = (2 * k + 1 < pl.n_qt) ? 2 : 1;
  const int b = bhi / p.H, h = bhi % p.H;
  const float gv = p.part[static_cast<int64_t>(slots[0]) * kSlotFloats + QT * BM * D + 2 * QT * BM];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = blockIdx.y * kCombineRows + warp * 4 + rr;  // query row of the item
    const int qrow = m0 + r;
    if (r >= nq * BM || qrow >= p.Lq) continue;
    float mstar = -INFINITY, lsum = 0.0f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = 0; i0 < ns; i0 += kCombineParts) {
      float mv[kCombineParts], lv[kCombineParts];
      float4 ov[kCombineParts];
#pragma unroll
      for (int t = 0; t < kCombineParts; ++t) {  // every load of this group first
        const int i = i0 + t < ns ? i0 + t : i0;
        const float* sp = p.part + static_cast<int64_t>(slots[i]) * kSlotFloats;
        mv[t] = i0 + t < ns ? sp[QT * BM * D + r] : -INFINITY;
        lv[t] = sp[QT * BM * D + QT * BM + r];
        ov[t] = reinterpret_cast<const float4*>(sp + r * D)[lane];
      }
      float mg = mstar;
#pragma unroll
      for (int t = 0; t < kCombineParts; ++t) mg = fmaxf(mg, mv[t]);
      const float rs = ptx::ex2(mstar - mg);  // 0 while mstar is -inf
      lsum *= rs;
      acc = make_float4(acc.x * rs, acc.y * rs, acc.z * rs, acc.w * rs);
      mstar = mg;
#pragma unroll
      for (int t = 0; t < kCombineParts; ++t) {
        const float wv = i0 + t < ns ? ptx::ex2(mv[t] - mstar) : 0.0f;
        lsum = fmaf(wv, lv[t], lsum);
        acc = make_float4(fmaf(wv, ov[t].x, acc.x), fmaf(wv, ov[t].y, acc.y), fmaf(wv, ov[t].z, acc.z),
                          fmaf(wv, ov[t].w, acc.w));
      }
    }
    const float inv = gv / lsum;
    const int64_t obase = ((static_cast<int64_t>(b) * p.Lq + qrow) * p.H + h) * D + 4 * lane;
    if (p.out_bf16) {
      __nv_bfloat162 v0 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
      __nv_bfloat162 v1 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&v0);
      w.y = *reinterpret_cast<uint32_t*>(&v1);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + obase) = w;
    } else {
      *reinterpret_cast<float4*>(static_cast<float*>(p.out) + obase) =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
  }
}

// Fault-injection probe: one warp waits, with the same bounded warp-collective wait the kernels
// use, on an mbarrier that nothing arrives at.  After kWaitLimitNs the wait gives up, ORs
// NVFP4KV_ERR_DEVICE_TIMEOUT into *status, and the kernel returns with the context intact.
__global__ void __launch_bounds__(32) wait_timeout_probe(uint32_t* status) {
  __shared__ __align__(8) uint64_t never_arrived;
  __shared__ uint32_t abort_word;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&never_arrived), 1);
    abort_word = 0;
    ptx::fence_mbar_init();
  }
  __syncwarp();
  waitw(ptx::smem_u32(&never_arrived), 0, &abort_word, status);
}

// ------------------------------------------------------------------ host side
PerDeviceOnce g_attn_attr;

// The work split for bh (batch, head) pairs of n_qt query tiles over NT KV tiles on n_sms SMs.
Plan make_plan(int64_t bh, int n_qt, int NT, int n_sms) {
  Plan pl{};
  pl.bh = static_cast<int>(bh);
  pl.n_qt = n_qt;
  pl.ipb = (n_qt + 1) / 2;
  pl.npairs = n_qt / 2;
  pl.NT = NT;
  pl.wP = kWPair;
  pl.wS = kWSingle;
  pl.units = bh * pl.ipb * static_cast<int64_t>(NT);
  pl.Wh = static_cast<int64_t>(NT) * (static_cast<int64_t>(pl.wP) * pl.npairs +
                                      static_cast<int64_t>(pl.wS) * (pl.ipb - pl.npairs));
  pl.W = bh * pl.Wh;
  // one CTA per SM, at least two KV tiles of work each
  int64_t g = std::min<int64_t>(std::min(n_sms, kMaxCtas), std::max<int64_t>(1, pl.units / 2));
  pl.G = static_cast<int>(std::max<int64_t>(1, g));
  return pl;
}

bool plan_has_splits(const Plan& pl) {
  for (int c = 1; c < pl.G; ++c) {
    const int64_t u = plan_cut(pl, c);
    if (u < pl.units && u % pl.NT != 0) return true;
  }
  return false;
}

size_t slot_bytes() { return static_cast<size_t>(kSlotFloats) * sizeof(float); }

}  // namespace

int current_sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return sms;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Two partial-result slots per CTA, one CTA per SM of the current device (148 when no device
// can be queried).
size_t attention_workspace_bytes(const nvfp4kv_cache&, int) {
  int sms = current_sm_count();
  if (sms <= 0) sms = 148;
  return 2 * static_cast<size_t>(std::min(sms, kMaxCtas)) * slot_bytes();
}

bool attention_shape_supported(const nvfp4kv_cache& c, int q_tokens, int64_t kv_tiles) {
  const int64_t bh = static_cast<int64_t>(c.batch) * c.heads;
  const int64_t ipb = ((q_tokens + BM - 1) / BM + 1) / 2;
  // weighted unit arithmetic stays far below 2^62
  return kv_tiles > 0 && kv_tiles < (int64_t(1) << 24) &&
         static_cast<double>(bh) * ipb * kv_tiles < 2147483647.0;
}

cudaError_t launch_wait_timeout_probe(uint32_t* status, cudaStream_t stream) {
  wait_timeout_probe<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

int attention_plan(const nvfp4kv_cache& c, int q_tokens, int kv_tiles, int n_sms, int cta, int seg,
                   int out[8]) {
  for (int i = 0; i < 8; ++i) out[i] = 0;
  const int n_qt = (q_tokens + BM - 1) / BM;
  const Plan pl = make_plan(static_cast<int64_t>(c.batch) * c.heads, n_qt, kv_tiles, n_sms);
  out[0] = pl.G;
  out[1] = plan_has_splits(pl) ? 2 : 1;
  if (cta < 0) return NVFP4KV_OK;
  if (cta >= pl.G) return NVFP4KV_ERR_INVALID_ARG;
  const int64_t ubeg = plan_cut(pl, cta), uend = plan_cut(pl, cta + 1);
  int n = 0;
  for (int u = static_cast<int>(ubeg); u < static_cast<int>(uend); ++n) {
    const Seg s = plan_seg(pl, u, static_cast<int>(uend));
    if (n == seg) {
      out[2] = s.bhi;
      out[3] = s.m0;
      out[4] = s.nq;
      out[5] = s.t0;
      out[6] = s.t1;
      out[7] = (s.t0 == 0 && s.t1 == pl.NT) ? -1 : 2 * cta + (u == ubeg ? 0 : 1);
    }
    u = seg_end(pl, s);
  }
  out[1] = n;  // segments of this CTA
  if (seg >= n) return seg < 0 ? NVFP4KV_OK : NVFP4KV_ERR_INVALID_ARG;
  return NVFP4KV_OK;
}

int attention_runs(const std::vector<int>& vis) {
  int runs = 0;
  for (size_t i = 0; i < vis.size(); ++i)
    if (i == 0 || vis[i] != vis[i - 1] + 1) ++runs;
  return runs;
}

int launch_attention(const nvfp4kv_cache& c, const uint16_t* q, int q_tokens, int64_t q_stride,
                     const std::vector<int>& vis, float softmax_scale, void* out, int out_dtype,
                     void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  AttnParams prm{};
  prm.k_codes = c.k_codes;
  prm.v_codes = c.v_codes;
  prm.k_scales = c.k_scales;
  prm.v_scales = c.v_scales;
  prm.k_g = c.k_gscale;
  prm.v_g = c.v_gscale;
  prm.k_mean = (c.flags & NVFP4KV_K_SMOOTH) ? c.k_mean : nullptr;
  prm.out = out;
  prm.part = static_cast<float*>(workspace);
  prm.status = c.status;
  prm.T = static_cast<int64_t>(c.capacity_chunks) * c.chunk_tokens;
  prm.B = c.batch;
  prm.H = c.heads;
  prm.Lq = q_tokens;
  prm.Lc = c.chunk_tokens;
  prm.C = c.capacity_chunks;
  prm.out_bf16 = out_dtype == NVFP4KV_OUT_BF16 ? 1 : 0;
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(D));
  prm.scale_log2 = scale * 1.4426950408889634f;

  // The visible chunk slots (ascending, distinct), merged into runs of consecutive slots; KV
  // tiles never cross a run boundary.
  prm.n_runs = 0;
  prm.run_tile0[0] = 0;
  for (size_t i = 0; i < vis.size();) {
    size_t k = i;
    while (k + 1 < vis.size() && vis[k + 1] == vis[k] + 1) ++k;
    if (prm.n_runs == MAX_RUNS) return NVFP4KV_ERR_UNSUPPORTED;
    const int r = prm.n_runs++;
    prm.run_key0[r] = vis[i] * c.chunk_tokens;
    prm.run_key1[r] = (vis[k] + 1) * c.chunk_tokens;
    prm.run_tile0[r + 1] = prm.run_tile0[r] + (prm.run_key1[r] - prm.run_key0[r] + BN - 1) / BN;
    i = k + 1;
  }
  prm.n_tiles = prm.run_tile0[prm.n_runs];
  if (!attention_shape_supported(c, q_tokens, prm.n_tiles)) return NVFP4KV_ERR_UNSUPPORTED;

  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return NVFP4KV_ERR_CUDA;
  CUtensorMap tm;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(c.heads),
                              static_cast<cuuint64_t>(q_tokens), static_cast<cuuint64_t>(c.batch)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(q_stride) * 2,
                                 static_cast<cuuint64_t>(q_tokens) * q_stride * 2};
  const cuuint32_t box[4] = {64, 1, BM, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult cr = encode(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(q), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return NVFP4KV_ERR_CUDA;
  const int sms = current_sm_count();
  if (sms <= 0) return NVFP4KV_ERR_CUDA;
  prm.pl = make_plan(static_cast<int64_t>(c.batch) * c.heads, (q_tokens + BM - 1) / BM, prm.n_tiles, sms);
  const bool splits = plan_has_splits(prm.pl);
  if (splits && (!workspace || workspace_bytes < 2 * static_cast<size_t>(prm.pl.G) * slot_bytes()))
    return NVFP4KV_ERR_WORKSPACE;

  const cudaError_t ae = g_attn_attr.run([] {
    cudaError_t e = cudaFuncSetAttribute(attention_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attention_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    return e;
  });
  if (ae != cudaSuccess) return NVFP4KV_ERR_CUDA;
  if (prm.k_mean)
    attention_kernel<true><<<prm.pl.G, Cfg::kThreads, Cfg::kSmemBytes, stream>>>(tm, prm);
  else
    attention_kernel<false><<<prm.pl.G, Cfg::kThreads, Cfg::kSmemBytes, stream>>>(tm, prm);
  if (cudaGetLastError() != cudaSuccess) return NVFP4KV_ERR_CUDA;
  if (splits) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prm.pl.G - 1, QT * BM / kCombineRows, 1);
    cfg.blockDim = dim3(32 * kCombineRows / 4, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, combine_kernel, prm) != cudaSuccess) return NVFP4KV_ERR_CUDA;
  }
  return NVFP4KV_OK;
}

}  // namespace nvfp4kv
