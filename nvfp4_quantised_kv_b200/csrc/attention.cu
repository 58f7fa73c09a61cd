// attention.cu -- chunk attention over the NVFP4 KV cache on sm_100a.
//
// Method: "LongLive-2.0" paper page (paperpeel.com), section 1 and section 3.2 "Parallel KV
// Quantization": the cache stays in NVFP4 and is dequantised in parallel inside the
// attention kernel; section 4.2 "Inference with Multi-Shot Attention Sink": the query chunk
// attends to a permanent sink plus a sliding window of chunks (duplicates removed); section
// 2.1: a chunk sees its own tokens.  Reading note (yingwang.github.io), "The NVFP4
// quantization format": x_hat = E2M1 * E4M3 * FP32 scale.
//
// One CTA owns one or two query tiles of 128 rows of one (batch, head) and walks the visible
// KV tiles (128 keys each; tiles lie inside runs of consecutive visible chunks, so chunks
// outside the mask are never read).  A host planner chooses how many CTAs take two tiles.
// 512 threads, four warpgroups; warp roles:
//   softmax warps 0-3, 4-7    query tile 0 / 1: one query row per thread, online softmax over
//                             TMEM rows, epilogue (176 registers each, setmaxnreg)
//   producer warp 8           TMA: Q tiles (tensor map, 128B swizzle) and packed K/V tiles
//                             + E4M3 scales (1-D bulk copies) into a ring of smem slots
//   MMA warp 9                TMEM allocation; tcgen05.mma S = Q K^T (both operands in
//                             smem), O += P V (P from TMEM, V from smem), eight MMAs per asm
//                             block from one elected lane
//   dequant warps 10-15       E2M1 * E4M3 products, exact in fp16, written straight into the
//                             128B-swizzled UMMA operand layout: K (the B operand of Q K^T,
//                             K-major) and V (the B operand of P V, MN-major)
// With two tiles the softmax warpgroups alternate with the tensor core: PV(0, j), QK(0, j+1),
// PV(1, j), QK(1, j+1).  The FP32 scales stay out of the MMAs: g_K(chunk) multiplies S per
// column, and g_V(chunk) / max g_V multiplies P per column before P is rounded to fp16 (fp16
// P and V keep the P V product 8x finer than bf16).  Rows are rescaled lazily: the running
// max only moves when it grows by more than 2^8.
//
// Every mbarrier wait is bounded (%globaltimer); on a time-out the kernel ORs
// NVFP4KV_ERR_DEVICE_TIMEOUT into the status word, lets in-flight copies and MMAs finish,
// frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4kv {
namespace {

constexpr int BM = 128;  // query rows per tile (TMEM lanes)
constexpr int BN = 128;  // keys per KV tile
constexpr int D = kHeadDim;
constexpr int NST = 2;   // stages of dequantised K / V tiles
constexpr int NPK = 3;   // slots of packed data (K and V tiles alternate)
constexpr int NCT = 4;   // slots of per-tile column tables
constexpr int kMaxTabChunks = 256;  // chunk scales staged in shared memory up to this many slots
constexpr int PK_CODES = BN * kCodeBytes;               // 8192
constexpr int PK_BYTES = PK_CODES + BN * kScaleBytes;   // 9216
constexpr int TILE16 = BN * D * 2;                      // one 128 x 128 16-bit operand tile
constexpr int HALF16 = TILE16 / 2;                      // 128 rows x 64 elements (128 B rows)
constexpr int MAX_RUNS = kAttnMaxRuns;

template <int QT>
struct Cfg {
  static constexpr int kSoftmaxWarps = 4 * QT;
  static constexpr int kProducerWarp = kSoftmaxWarps;
  static constexpr int kMmaWarp = kSoftmaxWarps + 1;
  static constexpr int kDequantWarp0 = kSoftmaxWarps + 2;
  static constexpr int kDequantWarps = 6;  // 2 in the producer/MMA warpgroup + one full warpgroup
  static constexpr int kDequantThreads = 32 * kDequantWarps;
  static_assert(kDequantThreads % 64 == 0, "dequant_tile deals blocks to a multiple of 64 threads");
  static constexpr int kThreads = 32 * (kSoftmaxWarps + 2 + kDequantWarps);  // whole warpgroups
  static constexpr uint32_t kTmemCols = QT == 1 ? 256 : 512;
  // shared memory map (bytes from a 1024-aligned base)
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + QT * TILE16;
  static constexpr int oV = oK + NST * TILE16;
  static constexpr int oPK = oV + NST * TILE16;
  // Per-tile column tables colK[BN], colV[BN] (fp32) and int4 {n_valid, uniform}, in NCT slots:
  // the K stage of tile j is refilled once the QKs of tile j - NST are done, while the softmax
  // warps may still read the tables of tiles j - NST and j - NST + 1.
  static constexpr int oCol = oPK + NPK * PK_BYTES;
  static constexpr int oInfo = oCol + NCT * 2 * BN * 4;
  static constexpr int oRed = oInfo + NCT * 16;          // per Q tile: 4 warp maxima
  static constexpr int oTab = oRed + QT * 16;            // per chunk slot: {g_K * scale, g_V / max g_V}
  static constexpr int oBar = oTab + kMaxTabChunks * 8;
  // barrier indices
  static constexpr int bQFull = 0;
  static constexpr int bQReady = 1;
  static constexpr int bPkFull = 2;
  static constexpr int bPkEmpty = bPkFull + NPK;
  static constexpr int bKFull = bPkEmpty + NPK;
  static constexpr int bVFull = bKFull + NST;
  static constexpr int bKEmpty = bVFull + NST;  // K stage read by every QK of its tile
  static constexpr int bVEmpty = bKEmpty + NST;  // V stage read by every PV of its tile
  static constexpr int bSFull = bVEmpty + NST;
  static constexpr int bPFull = bSFull + QT;
  static constexpr int bODone = bPFull + QT;
  static constexpr int bDrain = bODone + QT;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int oMisc = oBar + kNumBars * 8;  // [0] TMEM base, [1] abort flag
  static constexpr int kSmemBytes = oMisc + 16 + 1024;  // + slack for 1024-B alignment
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct AttnParams {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint8_t* k_scales;
  const uint8_t* v_scales;
  const float* k_g;
  const float* v_g;
  void* out;
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
  // Work list: every (b, h) has n_qt query tiles of 128 rows; the first pp + 1 (for (b, h) <
  // pr) or pp of its tile pairs go to two-tile CTAs, the rest of its tiles to one-tile CTAs.
  // CTAs [0, n_pair_ctas) take pairs, the others single tiles.
  int n_qt, pp, pr, n_pair_ctas;
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
  constexpr int KS = NT / 8;               // keys per pass: 24 for 192 threads, 40 for 320
  constexpr int kIt = (BN + KS - 1) / KS;  // passes; the last one may cover only part of the keys
  const int blk = dt & 7, kq = dt >> 3;
  const bool swap = blk >= 4;
  const int c0 = (blk & 3) * 2;
  const uint8_t* csrc = pk + kq * kCodeBytes + blk * 8;
  const uint8_t* ssrc = pk + PK_CODES + kq * kScaleBytes + blk;
  uint8_t* const row = dst + (blk >> 2) * HALF16 + kq * 128;
  uint8_t* const dA = row + (((c0 + (swap ? 1 : 0)) ^ (kq & 7)) << 4);  // first store
  uint8_t* const dB = row + (((c0 + (swap ? 0 : 1)) ^ (kq & 7)) << 4);
  const bool tail = kq + KS * (kIt - 1) < BN;  // this thread has a sixth key
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

// Work item of CTA c: every (b, h) has n_qt query tiles; (b, h) < pr gives its first pp + 1 tile
// pairs to two-tile CTAs, the others their first pp; CTAs [0, n_pair_ctas) take those pairs in
// (b, h) order, the rest take the remaining tiles one by one, also in (b, h) order.  Shared by the
// kernel and the host diagnostic that checks the split.
struct WorkItem {
  int bhi, m0, nq;
};

__host__ __device__ inline WorkItem work_item(int c, int n_qt, int pp, int pr, int n_pair_ctas) {
  WorkItem w;
  if (c < n_pair_ctas) {
    const int big = pr * (pp + 1);
    int idx;
    if (c < big || pp == 0) {
      w.bhi = c / (pp + 1);
      idx = c % (pp + 1);
    } else {
      w.bhi = pr + (c - big) / pp;
      idx = (c - big) % pp;
    }
    w.m0 = idx * 2 * BM;
    w.nq = 2;
  } else {
    const int c2 = c - n_pair_ctas;
    const int s_big = n_qt - 2 * (pp + 1), s_small = n_qt - 2 * pp;
    const int big = s_big > 0 ? pr * s_big : 0;
    int idx, pairs;
    if (c2 < big || s_small <= 0) {
      w.bhi = s_big > 0 ? c2 / s_big : 0;
      idx = s_big > 0 ? c2 % s_big : 0;
      pairs = pp + 1;
    } else {
      w.bhi = pr + (c2 - big) / s_small;
      idx = (c2 - big) % s_small;
      pairs = pp;
    }
    w.m0 = (2 * pairs + idx) * BM;
    w.nq = 1;
  }
  return w;
}

template <int QT>
__global__ void __launch_bounds__(Cfg<QT>::kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ AttnParams p) {
  using C = Cfg<QT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // This CTA's work item: (b, h), first query row m0 and nq query tiles.
  const WorkItem wi = work_item(blockIdx.x, p.n_qt, p.pp, p.pr, p.n_pair_ctas);
  const int bhi = wi.bhi, m0 = wi.m0, nq = wi.nq;
  const int h = bhi % p.H, b = bhi / p.H;
  const int64_t bh = static_cast<int64_t>(b) * p.H + h;
  const int n_dq_warps = C::kDequantWarps;

  const uint32_t sbase = ptx::smem_u32(smem);
  auto bar = [&](int i) { return sbase + C::oBar + 8 * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::oMisc);
  volatile uint32_t* abort_flag = misc + 1;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(C::bQFull), 1);
    ptx::mbar_init(bar(C::bQReady), 4 * nq);
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
    for (int q = 0; q < QT; ++q) {
      ptx::mbar_init(bar(C::bSFull + q), 1);
      ptx::mbar_init(bar(C::bPFull + q), 4);
      ptx::mbar_init(bar(C::bODone + q), 1);
    }
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
  // Registers move from the producer/MMA/dequant warpgroups (80 each) to the two softmax
  // warpgroups (176 each), which hold a whole 128-column S row: 2*128*176 + 2*128*80 = 65536,
  // exactly what the 512-thread block was launched with.  Each role branch starts with its
  // warpgroup's budget change.
  static_assert(QT == 1 || C::kThreads == 512, "register split assumes four warpgroups");

  // Dequantiser role: thread dt of the nthreads threads of the dequant warps.
  auto dequant_role = [&](int dt) {
    const int nthreads = 32 * n_dq_warps;
    const float inv_gv = 1.0f / max_visible_gv(p, bh);
    // The per-chunk FP32 scales of this (b, h), staged once, so the per-tile column tables are
    // built from shared memory.
    const float2* gtab = reinterpret_cast<const float2*>(smem + C::oTab);
    const bool use_tab = p.C <= kMaxTabChunks;
    if (use_tab)
      for (int c = dt; c < p.C; c += nthreads)
        reinterpret_cast<float2*>(smem + C::oTab)[c] =
            make_float2(p.k_g[bh * p.C + c] * p.scale_log2, p.v_g[bh * p.C + c] * inv_gv);
    ptx::named_bar(3, nthreads);
    bool ok = true;
    for (int j = 0; j < p.n_tiles && ok; ++j) {
      const int st = j % NST;
      int key0, n;
      tile_keys(p, j, key0, n);
      for (int t = 0; t < 2 && ok; ++t) {
        // the stage's previous tile (j - NST) is done with it: K after its QKs, V after its PVs
        if (j >= NST) ok = waitw(bar((t == 0 ? C::bKEmpty : C::bVEmpty) + st), ((j / NST) - 1) & 1, abort_flag, p.status);
        if (!ok) break;
        const int pk = 2 * j + t;
        const int slot = pk % NPK;
        ok = waitw(bar(C::bPkFull + slot), (pk / NPK) & 1, abort_flag, p.status);
        if (!ok) break;
        const uint8_t* src = smem + C::oPK + slot * PK_BYTES;
        uint8_t* dst = smem + (t == 0 ? C::oK : C::oV) + st * TILE16;
        if (n == BN) dequant_tile<C::kDequantThreads, true>(src, dst, n, dt);
        else dequant_tile<C::kDequantThreads, false>(src, dst, n, dt);
        if (t == 0 && dt < BN) {  // per-column tables: one thread per key of the tile
          float* colK = reinterpret_cast<float*>(smem + C::oCol + (j % NCT) * 2 * BN * 4);
          const bool valid = dt < n;
          const int c = valid ? (key0 + dt) / p.Lc : 0;
          const float2 g = !valid ? make_float2(0.0f, 0.0f)
                           : use_tab ? gtab[c]
                                     : make_float2(p.k_g[bh * p.C + c] * p.scale_log2, p.v_g[bh * p.C + c] * inv_gv);
          colK[dt] = g.x;
          colK[BN + dt] = g.y;
          if (dt == 0) {
            const int uniform = (n == BN) && (key0 / p.Lc == (key0 + BN - 1) / p.Lc);
            *reinterpret_cast<int4*>(smem + C::oInfo + 16 * (j % NCT)) = make_int4(n, uniform, 0, 0);
          }
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(bar(C::bPkEmpty + slot));
          ptx::mbar_arrive(bar(t == 0 ? C::bKFull + st : C::bVFull + st));
        }
      }
    }
  };

  if (warp < C::kSoftmaxWarps) {
    // ============================================================ softmax + epilogue
    if constexpr (QT == 2) ptx::setmaxnreg_inc<176>();
    const int qt = warp >> 2;
    if (qt < nq) {
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + qt * BN;
    const uint32_t tO = tmem + lane_off + QT * BN + qt * D;
    const float gv_ref = max_visible_gv(p, bh);
    bool ok = waitw(bar(C::bQFull), 0, abort_flag, p.status);
    float pre_scale = 1.0f;

    // ---- Q tile: bf16 -> fp16 in place, exact, after a power-of-two prescale 2^-e that keeps
    // the tile's largest |q| below 2^15; S is scaled back by 2^e with the logit factor.
    float q_unscale = 1.0f;
    uint8_t* qrow = smem + C::oQ + qt * TILE16 + row * 128;
    {
      uint32_t mb = 0;
      if (ok) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(qrow + (i >> 3) * HALF16 + (((i + lane) & 7) << 4));
          mb = __vmaxu2(mb, __vmaxu2(absmax_bf16x2(v.x, v.y), absmax_bf16x2(v.z, v.w)));
        }
      }
      mb = max(mb & 0xFFFFu, mb >> 16);
      mb = __reduce_max_sync(0xFFFFFFFFu, mb);
      uint32_t* red = reinterpret_cast<uint32_t*>(smem + C::oRed + qt * 16);
      if (lane == 0) red[warp & 3] = mb;
      ptx::named_bar(1 + qt, 128);  // reached by all four warps of the tile, on every path
      mb = max(max(red[0], red[1]), max(red[2], red[3]));
      const int ex = static_cast<int>((mb >> 7) & 0xFF) - 127;  // floor(log2 max|q|)
      const int e = ex > 14 ? ex - 14 : 0;
      q_unscale = __int_as_float((127 + e) << 23);  // 2^e
      pre_scale = __int_as_float((127 - e) << 23);  // 2^-e
    }
    if (ok) {
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
      if (lane == 0) ptx::mbar_arrive(bar(C::bQReady));
    }

    float m_run = -INFINITY, l_run = 0.0f;
    for (int j = 0; j < p.n_tiles && ok; ++j) {
      const int st = j % NST;
      ok = waitw(bar(C::bSFull + qt), j & 1, abort_flag, p.status) &&
           waitw(bar(C::bKFull + st), (j / NST) & 1, abort_flag, p.status);
      if (!ok) break;
      ptx::tc_fence_after();
      const int ct = j % NCT;
      const int4 info = *reinterpret_cast<const int4*>(smem + C::oInfo + 16 * ct);
      const float* colK = reinterpret_cast<const float*>(smem + C::oCol + ct * 2 * BN * 4);
      const float* colV = colK + BN;
      const float ck = colK[0] * q_unscale;
      // A tile inside one chunk with every key valid and a nonzero V scale takes the uniform path
      // (one logit factor, one cv); any other tile works per column.
      const bool uni = info.y && colV[0] > 0.0f;

      // The whole 128-column S row: four loads in flight, one wait.
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tS + 32 * c, sr[c]);
      ptx::tc_wait_ld_regs(sr[0]);
      ptx::reg_fence32(sr[1]);
      ptx::reg_fence32(sr[2]);
      ptx::reg_fence32(sr[3]);

      // Row maximum of x = S * g_K(chunk) * scale * log2(e) (masked keys -inf).
      float mx;
      if (uni) {
        float m8[8];  // eight independent max chains
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            m8[2 * c] = ptx::fmax3(m8[2 * c], __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]));
            m8[2 * c + 1] =
                ptx::fmax3(m8[2 * c + 1], __uint_as_float(sr[c][i + 2]), __uint_as_float(sr[c][i + 3]));
          }
        mx = fmaxf(ptx::fmax3(m8[0], m8[1], m8[2]), ptx::fmax3(m8[3], m8[4], ptx::fmax3(m8[5], m8[6], m8[7]))) *
             ck;
      } else {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int jj = 32 * c + i;
            m4[c] = fmaxf(m4[c], jj < info.x ? __uint_as_float(sr[c][i]) * colK[jj] * q_unscale : -INFINITY);
          }
        mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      }
      // Lazy rescale: the reference m only moves (to a whole number, so the rescale is an exact
      // power of two) when the row maximum exceeds it by more than 2^8.  The O rescale uses
      // warp-collective TMEM accesses, so it runs for the whole warp when any row moved
      // (alpha = 1 for the rows that did not).
      const bool grow = mx > m_run + 8.0f;
      if (__any_sync(0xFFFFFFFFu, grow)) {
        const float m_new = grow ? ceilf(mx) : m_run;
        const float alpha = grow ? ptx::ex2(m_run - m_new) : 1.0f;  // 0 while m is -inf
        l_run *= alpha;
        m_run = m_new;
        if (j > 0) {  // O holds tiles < j; PV(j - 1) is complete (it precedes QK(j))
          ok = waitw(bar(C::bODone + qt), (j - 1) & 1, abort_flag, p.status);
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

      // P~ = 2^(x - m) * cv (cv = g_V(chunk) / max g_V), rounded to fp16 pairs and stored over
      // S's first 64 columns (chunk c -> P columns [16c, 16c + 16)).  The row sum adds the same
      // rounded values divided by cv, so the rounding largely cancels in O / l; a key of an
      // all-zero V chunk (cv = 0) adds 0 to O and its p to l.
      float la = 0.0f, lb = 0.0f;
      if (uni) {
        // x = S * ck + log2(cv) - m in packed pairs; eight independent row-sum chains.
        const float mneg = log2f(colV[0]) - m_run;
        float l8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) l8[k] = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
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
        la = (l8[0] + l8[1]) + (l8[2] + l8[3]);
        lb = (l8[4] + l8[5]) + (l8[6] + l8[7]);
        l_run += (la + lb) / colV[0];
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int j0 = 32 * c + 2 * i;
            const float x0 = j0 < info.x ? __uint_as_float(sr[c][2 * i]) * colK[j0] * q_unscale : -INFINITY;
            const float x1 =
                j0 + 1 < info.x ? __uint_as_float(sr[c][2 * i + 1]) * colK[j0 + 1] * q_unscale : -INFINITY;
            const float p0 = x0 == -INFINITY ? 0.0f : ptx::ex2(x0 - m_run);
            const float p1 = x1 == -INFINITY ? 0.0f : ptx::ex2(x1 - m_run);
            const float cv0 = colV[j0], cv1 = colV[j0 + 1];
            pk[i] = ptx::f32x2_to_f16x2(p0 * cv0, p1 * cv1);
            const float t0 = __half2float(__ushort_as_half(static_cast<uint16_t>(pk[i] & 0xFFFFu)));
            const float t1 = __half2float(__ushort_as_half(static_cast<uint16_t>(pk[i] >> 16)));
            la += cv0 > 0.0f ? t0 / cv0 : p0;
            lb += cv1 > 0.0f ? t1 / cv1 : p1;
          }
          ptx::tmem_st16p(tS + 16 * c, pk);
        }
        l_run += la + lb;
      }
      ptx::tc_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(C::bPFull + qt));
    }
    if (ok && p.n_tiles > 0) {
      ok = waitw(bar(C::bODone + qt), (p.n_tiles - 1) & 1, abort_flag, p.status);
      if (ok) {
        ptx::tc_fence_after();
        const float inv = gv_ref / l_run;
        const int qrow = m0 + qt * BM + row;
        const bool store = qrow < p.Lq;
        const int64_t obase = ((static_cast<int64_t>(b) * p.Lq + qrow) * p.H + h) * D;
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
      }
    }
    }
  } else {
  if constexpr (QT == 2) ptx::setmaxnreg_dec<80>();
  if (warp == C::kProducerWarp) {
    // ============================================================ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_q);
      ptx::mbar_arrive_expect_tx(bar(C::bQFull), nq * TILE16);
      for (int q = 0; q < nq; ++q)
        for (int half = 0; half < 2; ++half)
          ptx::tma_load_4d(sbase + C::oQ + q * TILE16 + half * HALF16, &tmap_q, half * 64, h,
                           m0 + q * BM, b, bar(C::bQFull));
      const uint8_t* kc = p.k_codes + bh * p.T * kCodeBytes;
      const uint8_t* vc = p.v_codes + bh * p.T * kCodeBytes;
      const uint8_t* ks = p.k_scales + bh * p.T * kScaleBytes;
      const uint8_t* vs = p.v_scales + bh * p.T * kScaleBytes;
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < p.n_tiles && ok; ++j) {
        int key0, n;
        tile_keys(p, j, key0, n);
        for (int t = 0; t < 2; ++t) {
          const int pk = 2 * j + t;
          const int slot = pk % NPK;
          ok = wait1(bar(C::bPkEmpty + slot), ((pk / NPK) & 1) ^ 1, abort_flag, p.status);
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
      if (!ok) {  // let every copy already issued land before the CTA can exit
        wait_drain(bar(C::bQFull), 0, p.status);
        for (int pk = std::max(0, issued - NPK); pk < issued; ++pk)
          wait_drain(bar(C::bPkFull + pk % NPK), (pk / NPK) & 1, p.status);
      }
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ============================================================ MMA issuer
    // The whole warp runs this loop with warp-uniform values; one elected lane issues each
    // tcgen05 instruction.
    // kind::f16 instruction descriptors: fp16 x fp16 -> fp32; M = 128; N = 128.
    constexpr uint32_t kIdescQK = (1u << 4) |  // A = Q and B = K^ both K-major
                                  (static_cast<uint32_t>(BN >> 3) << 17) |
                                  (static_cast<uint32_t>(BM >> 4) << 24);
    constexpr uint32_t kIdescPV = (1u << 4) | (1u << 16) |  // B = V^ MN-major
                                  (static_cast<uint32_t>(D >> 3) << 17) |
                                  (static_cast<uint32_t>(BM >> 4) << 24);
    // Shared-memory descriptors are built once; a K step only advances the 14-bit start address
    // field (address >> 4).
    const uint64_t dQ0 = ptx::smem_desc_sw128(sbase + C::oQ, 16, 1024);
    const uint64_t dK0 = ptx::smem_desc_sw128(sbase + C::oK, 16, 1024);
    const uint64_t dV0 = ptx::smem_desc_sw128(sbase + C::oV, HALF16, 1024);
    auto issue_qk = [&](int q, int st) {
      const uint64_t dQ = dQ0 + static_cast<uint64_t>((q * TILE16) >> 4);
      const uint64_t dK = dK0 + static_cast<uint64_t>((st * TILE16) >> 4);
      const uint32_t tS = tmem + q * BN;
      // one asm block of eight MMAs: a rolled loop issued an MMA only every ~80 cycles
      ptx::mma_qk8_w(tS, dQ, dK, kIdescQK, 0u);
      ptx::mma_commit_w(bar(C::bSFull + q));
    };
    bool ok = waitw(bar(C::bQReady), 0, abort_flag, p.status) && p.n_tiles > 0 &&
              waitw(bar(C::bKFull + 0), 0, abort_flag, p.status);
    if (ok) {
      ptx::tc_fence_after();
      for (int q = 0; q < nq; ++q) issue_qk(q, 0);
      ptx::mma_commit_w(bar(C::bKEmpty + 0));
    }
    // Per KV tile j: PV(q, j) as soon as softmax q has written P(q, j), then QK(q, j + 1) into the
    // same S columns; the two query tiles alternate so the tensor core always has the other
    // tile's work while one softmax runs.
    for (int j = 0; j < p.n_tiles && ok; ++j) {
      const int st = j % NST;
      for (int q = 0; q < nq && ok; ++q) {
        ok = waitw(bar(C::bPFull + q), j & 1, abort_flag, p.status);
        if (ok && q == 0) ok = waitw(bar(C::bVFull + st), (j / NST) & 1, abort_flag, p.status);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint64_t dV = dV0 + static_cast<uint64_t>((st * TILE16) >> 4);
        const uint32_t tO = tmem + QT * BN + q * D, tP = tmem + q * BN;
        ptx::mma_pv8_w(tO, tP, dV, kIdescPV, j > 0 ? 1u : 0u);
        ptx::mma_commit_w(bar(C::bODone + q));
        if (q == nq - 1) ptx::mma_commit_w(bar(C::bVEmpty + st));
        if (j + 1 < p.n_tiles) {
          const int st1 = (j + 1) % NST;
          if (q == 0) {
            ok = waitw(bar(C::bKFull + st1), ((j + 1) / NST) & 1, abort_flag, p.status);
            if (!ok) break;
            ptx::tc_fence_after();
          }
          issue_qk(q, st1);
          if (q == nq - 1) ptx::mma_commit_w(bar(C::bKEmpty + st1));
        }
      }
    }
    // every MMA issued so far completes before the drain barrier's phase 0
    ptx::mma_commit_w(bar(C::bDrain));
    if (lane == 0) wait_drain(bar(C::bDrain), 0, p.status);
    __syncwarp();
  } else {
    // ============================================================ dequant warps
    dequant_role(threadIdx.x - C::kDequantWarp0 * 32);
  }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
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
template <int QT>
cudaError_t launch(const CUtensorMap& tm, const AttnParams& prm, int n_single_ctas, cudaStream_t stream) {
  using C = Cfg<QT>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(attention_kernel<QT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  attention_kernel<QT><<<prm.n_pair_ctas + n_single_ctas, C::kThreads, C::kSmemBytes, stream>>>(tm, prm);
  return cudaGetLastError();
}

// Makespan of p two-tile CTAs (cost `pair`) followed by s one-tile CTAs (cost `single`), each
// started on whichever of the g SMs frees first (one CTA per SM at a time).  Integer costs keep
// equal loads equal; machines are tracked per load level, so the cost is the number of levels the
// schedule passes through, not the number of CTAs.
int64_t makespan(int64_t p, int64_t s, int64_t g, int64_t pair, int64_t single) {
  std::map<int64_t, int64_t> level;  // load -> machines at that load
  level[(p / g) * pair] += g - p % g;
  if (p % g) level[(p / g + 1) * pair] += p % g;
  while (s > 0) {
    auto lo = level.begin();
    const int64_t take = std::min(lo->second, s);
    const int64_t load = lo->first;
    s -= take;
    if ((lo->second -= take) == 0) level.erase(lo);
    level[load + single] += take;
  }
  return level.rbegin()->first;
}

// Splits the n_qt query tiles of each of the bh (batch, head) pairs into tile pairs (two-tile CTAs,
// the two softmax warpgroups in ping-pong) and single tiles (one-tile CTAs) so that the launch
// finishes soonest on g SMs: e.g. 444 tiles on 148 SMs as 148 pairs + 148 singles (1.94 units)
// instead of 222 pairs in two waves (2 units).  Candidates: all pairs, no pairs, and the last
// three whole waves of pairs.  Plans are cached per (n_qt, bh, g).
void plan_work(int n_qt, int bh, int g, AttnParams& prm, int& n_single_ctas) {
  // Cost of a one-tile CTA relative to a two-tile one (94 : 100), measured on the 1.3B-class
  // layer: the per-KV-tile dequantisation and MMA chain, which do not shrink with one query tile,
  // dominate.
  constexpr int64_t kPair = 100, kSingle = 94;
  static std::mutex mu;
  static std::map<std::tuple<int, int, int>, int> cache;
  int best_p = -1;
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(std::make_tuple(n_qt, bh, g));
    if (it != cache.end()) best_p = it->second;
  }
  const int64_t max_p = static_cast<int64_t>(bh) * (n_qt / 2), total = static_cast<int64_t>(bh) * n_qt;
  if (best_p < 0) {
    std::vector<int64_t> cand = {0, max_p};
    for (int64_t k = max_p / g; k >= 1 && k >= max_p / g - 2; --k) cand.push_back(k * g);
    int64_t bp = max_p, best = makespan(max_p, total - 2 * max_p, g, kPair, kSingle);
    for (int64_t pc : cand) {
      const int64_t m = makespan(pc, total - 2 * pc, g, kPair, kSingle);
      if (m < best || (m == best && pc > bp)) {
        best = m;
        bp = pc;
      }
    }
    best_p = static_cast<int>(bp);
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() > 4096) cache.clear();
    cache[std::make_tuple(n_qt, bh, g)] = best_p;
  }
  prm.n_qt = n_qt;
  prm.pp = best_p / bh;
  prm.pr = best_p % bh;
  prm.n_pair_ctas = best_p;
  n_single_ctas = static_cast<int>(total - 2 * best_p);
}

}  // namespace

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

size_t attention_workspace_bytes(const nvfp4kv_cache&, int) { return 0; }

cudaError_t launch_wait_timeout_probe(uint32_t* status, cudaStream_t stream) {
  wait_timeout_probe<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

int attention_plan(const nvfp4kv_cache& c, int q_tokens, int n_sms, int cta, int out[4]) {
  AttnParams prm{};
  int n_single = 0;
  const int n_qt = (q_tokens + BM - 1) / BM;
  plan_work(n_qt, c.batch * c.heads, n_sms, prm, n_single);
  out[0] = prm.n_pair_ctas + n_single;
  out[1] = out[2] = out[3] = 0;
  if (cta < 0) return NVFP4KV_OK;
  if (cta >= out[0]) return NVFP4KV_ERR_INVALID_ARG;
  const WorkItem w = work_item(cta, prm.n_qt, prm.pp, prm.pr, prm.n_pair_ctas);
  out[1] = w.bhi;
  out[2] = w.m0;
  out[3] = w.nq;
  return NVFP4KV_OK;
}

int attention_runs(const std::vector<int>& vis) {
  int runs = 0;
  for (size_t i = 0; i < vis.size(); ++i)
    if (i == 0 || vis[i] != vis[i - 1] + 1) ++runs;
  return runs;
}

int launch_attention(const nvfp4kv_cache& c, const uint16_t* q, int q_tokens, int64_t q_stride,
                     const std::vector<int>& vis, float softmax_scale, void* out, int out_dtype, void*,
                     size_t, cudaStream_t stream) {
  AttnParams prm{};
  prm.k_codes = c.k_codes;
  prm.v_codes = c.v_codes;
  prm.k_scales = c.k_scales;
  prm.v_scales = c.v_scales;
  prm.k_g = c.k_gscale;
  prm.v_g = c.v_gscale;
  prm.out = out;
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
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return NVFP4KV_ERR_CUDA;
  int n_single_ctas = 0;
  plan_work((q_tokens + BM - 1) / BM, c.batch * c.heads, sms, prm, n_single_ctas);
  const cudaError_t e = launch<2>(tm, prm, n_single_ctas, stream);
  return e == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

}  // namespace nvfp4kv
