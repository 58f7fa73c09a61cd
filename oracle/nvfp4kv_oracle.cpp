/*
 * nvfp4kv_oracle.cpp -- CPU oracle for the NVFP4 KV-cache path.
 *
 * TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's CPU
 * baseline load this file's library; the CUDA library never does.  It is deliberately
 * plain and slow: one thread, scalar loops, no blocking or reordering beyond what the
 * definitions state.  Build with -O2 -ffp-contract=off and without fast-math so that
 * every fp32 operation below is one IEEE-754 round-to-nearest-even operation.
 *
 * What it computes (sources cited as in nvfp4kv_oracle.h):
 *
 *  NVFP4 quantisation of one K or V chunk of one head [P1 sec. 2.2], [N1], [N2]:
 *   The pages lose the equation itself; only its constants (16-element blocks,
 *   M_FP8 = 448, M_FP4 = 6) and the three factors of dequantisation survive.  The reading
 *   taken here, in fp32 with round-to-nearest-even at every step:
 *     A      = max |x| over the chunk (exact)
 *     g      = A / (448 * 6)                       (0 when A == 0)      -- FP32 scale
 *     for every token and every 16-element block b along the head dimension:
 *       a_b  = max |x| over the block
 *       s    = E4M3(a_b / (6 * g))                 (0 when a_b == 0 or g == 0) -- block scale
 *       r    = 1 / (decode(s) * g)
 *       q_i  = E2M1(x_i * r)                       (all 0 when decode(s) == 0 or r is not finite)
 *   E4M3() and E2M1() round to the nearest representable value, ties to the even code,
 *   and clamp to the largest finite magnitude.
 *  Dequantisation [N1]: x_hat = E2M1(q) * E4M3(s) * g, evaluated in fp64 (exact).
 *
 *  The pages' own recipe for the cache [N2]: "K-smoothing" of K and "adaptive scale selection"
 *  of V within each chunk, with the candidate scale targets {4, 6} [N3], [P1 sec. A.2].  The
 *  pages name both and define neither; the readings taken here:
 *   K-smoothing: mu_i = the channel mean of the chunk's keys of one head, (sum over t of x[t][i]) / L
 *     computed exactly (every bf16 value is a whole number of 2^-133) and rounded once to fp32,
 *     to nearest with ties to even; the chunk is quantised as above from
 *     x'[t][i] = x[t][i] - mu_i (one fp32 subtraction), and the key the cache stands for is
 *     x_hat' + mu (mu stored in fp32 beside the chunk).
 *   Adaptive scale (target T in {6, 4}): for every block both targets are tried,
 *       s_T = E4M3(a_b / (T * g)),  q_i = E2M1(x_i * 1 / (decode(s_T) * g)),
 *     and the one with the smaller squared error E_T = sum over the block's 16 elements, in
 *     order, of (x_i - E2M1(q_i) * E4M3(s_T) * g)^2 (fp64, each product, difference, square
 *     and sum rounded once) is kept; ties keep 6.  g is unchanged (A / (448 * 6)), so a block
 *     near the chunk maximum whose target-4 scale would exceed 448 saturates, and keeps 6 unless
 *     the saturated candidate is strictly better.
 *  Attention [P1' sec. 4.2], [P1'' sec. 2.1]: a query row of chunk t attends to the keys of
 *   the visible chunks V(t) = {c < n_sink} U {t - window < c <= t} (duplicates removed), in
 *   fp64: s_j = sigma * q . k_hat_j, p_j = exp(s_j - max_j s_j), o = sum p_j v_hat_j / sum p_j.
 */
#include "nvfp4kv_oracle.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>
#include <vector>
#include <xmmintrin.h>

namespace {

/* Keep subnormals: clear flush-to-zero and denormals-are-zero for the duration of a call. */
struct IeeeMode {
  unsigned saved;
  IeeeMode() : saved(_mm_getcsr()) { _mm_setcsr(saved & ~(0x8000u | 0x0040u)); }
  ~IeeeMode() { _mm_setcsr(saved); }
};

float bf16_bits_to_float(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

/* A non-negative integer as little-endian 32-bit digits: just enough arithmetic for the exact
 * channel mean (add a small value shifted left, compare, subtract, divide by a small value). */
struct BigNat {
  std::vector<uint32_t> dig;
  void add_shifted(uint32_t m, int shift) {
    size_t k = static_cast<size_t>(shift / 32);
    uint64_t carry = static_cast<uint64_t>(m) << (shift % 32);
    while (carry != 0) {
      if (dig.size() <= k) dig.resize(k + 1, 0u);
      const uint64_t t = static_cast<uint64_t>(dig[k]) + (carry & 0xFFFFFFFFu);
      dig[k] = static_cast<uint32_t>(t);
      carry = (carry >> 32) + (t >> 32);
      ++k;
    }
  }
  bool bit(int n) const {
    const size_t k = static_cast<size_t>(n / 32);
    return k < dig.size() && ((dig[k] >> (n % 32)) & 1u);
  }
  int bit_length() const {
    for (size_t k = dig.size(); k-- > 0;)
      if (dig[k] != 0)
        for (int j = 31; j >= 0; --j)
          if ((dig[k] >> j) & 1u) return static_cast<int>(k) * 32 + j + 1;
    return 0;
  }
};

int compare(const BigNat& a, const BigNat& b) {
  const size_t n = std::max(a.dig.size(), b.dig.size());
  for (size_t k = n; k-- > 0;) {
    const uint32_t x = k < a.dig.size() ? a.dig[k] : 0u, y = k < b.dig.size() ? b.dig[k] : 0u;
    if (x != y) return x < y ? -1 : 1;
  }
  return 0;
}

BigNat subtract(const BigNat& a, const BigNat& b) { /* a >= b */
  BigNat r;
  r.dig.resize(a.dig.size(), 0u);
  int64_t borrow = 0;
  for (size_t k = 0; k < a.dig.size(); ++k) {
    int64_t t = static_cast<int64_t>(a.dig[k]) - (k < b.dig.size() ? b.dig[k] : 0u) - borrow;
    borrow = t < 0 ? 1 : 0;
    if (t < 0) t += (int64_t(1) << 32);
    r.dig[k] = static_cast<uint32_t>(t);
  }
  return r;
}

/* fp32 nearest to (pos - neg) * 2^-133 / L, ties to even: the quotient is taken in units of 2^-149
 * (the smallest fp32 subnormal step) with its remainder, then rounded to 24 significant bits. */
float exact_mean_to_float(const BigNat& pos, const BigNat& neg, uint32_t L) {
  const int c = compare(pos, neg);
  if (c == 0) return 0.0f;
  BigNat mag = c > 0 ? subtract(pos, neg) : subtract(neg, pos);
  BigNat num;  /* mag * 2^16 */
  for (int n = mag.bit_length() - 1; n >= 0; --n)
    if (mag.bit(n)) num.add_shifted(1u, n + 16);
  /* long division by L, most significant digit first */
  BigNat q;
  q.dig.resize(num.dig.size(), 0u);
  uint64_t r = 0;
  for (size_t k = num.dig.size(); k-- > 0;) {
    const uint64_t cur = (r << 32) | num.dig[k];
    q.dig[k] = static_cast<uint32_t>(cur / L);
    r = cur % L;
  }
  const int n = q.bit_length();
  double v;
  if (n <= 24) { /* below 2^-125: every multiple of 2^-149 under 2^24 of them is an fp32 value */
    uint64_t k = 0;
    for (int j = n - 1; j >= 0; --j) k = (k << 1) | (q.bit(j) ? 1u : 0u);
    const bool up = 2 * r > L || (2 * r == L && (k & 1u));
    v = std::ldexp(static_cast<double>(k + (up ? 1 : 0)), -149);
  } else {
    const int sh = n - 24;
    uint64_t mant = 0;
    for (int j = n - 1; j >= sh; --j) mant = (mant << 1) | (q.bit(j) ? 1u : 0u);
    const bool guard = q.bit(sh - 1);
    bool lower = r != 0;
    for (int j = sh - 2; j >= 0 && !lower; --j) lower = q.bit(j);
    const bool up = guard && (lower || (mant & 1u));
    v = std::ldexp(static_cast<double>(mant + (up ? 1 : 0)), sh - 149);
  }
  return static_cast<float>(c > 0 ? v : -v); /* exact: v has at most 24 significant bits */
}

/* Nearest code among the ascending non-negative magnitudes dec(0) < dec(1) < ... <
 * dec(n-1); an exact tie goes to the even code; anything at or beyond the largest
 * magnitude takes the largest code. */
uint8_t nearest_magnitude_code(double a, int n, double (*dec)(uint8_t)) {
  const double top = dec(static_cast<uint8_t>(n - 1));
  if (a >= top) return static_cast<uint8_t>(n - 1);
  int best = 0;
  double best_d = std::fabs(a - dec(0));
  for (int c = 1; c < n; ++c) {
    const double dist = std::fabs(a - dec(static_cast<uint8_t>(c)));
    if (dist < best_d || (dist == best_d && (c % 2) == 0)) {
      best = c;
      best_d = dist;
    }
  }
  return static_cast<uint8_t>(best);
}

double e2m1_magnitude(uint8_t c) { return oracle_e2m1_decode(static_cast<uint8_t>(c & 7)); }
double e4m3_magnitude(uint8_t c) { return oracle_e4m3_decode(static_cast<uint8_t>(c & 0x7F)); }

}  // namespace

extern "C" {

/* E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa [N1 "The NVFP4
 * quantization format"]; exponent 0 is the subnormal 0.5 * m. */
double oracle_e2m1_decode(uint8_t code) {
  const int e = (code >> 1) & 3;
  const int m = code & 1;
  const double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return (code & 8) ? -mag : mag;
}

uint8_t oracle_e2m1_encode(float v) {
  const uint8_t sign = std::signbit(v) ? 8 : 0;
  /* 8 magnitudes (codes 0..7), largest 6 = M_FP4 [P1 sec. 2.2]. */
  return static_cast<uint8_t>(sign | nearest_magnitude_code(std::fabs(static_cast<double>(v)), 8,
                                                            e2m1_magnitude));
}

/* E4M3: bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa; exponent 0 is
 * subnormal (m * 2^-9); S.1111.111 is NaN, so the largest finite magnitude is
 * 1.75 * 2^8 = 448 = M_FP8 [P1 sec. 2.2]. */
double oracle_e4m3_decode(uint8_t code) {
  const int e = (code >> 3) & 15;
  const int m = code & 7;
  if (e == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
  const double mag = (e == 0) ? std::ldexp(static_cast<double>(m), -9)
                              : std::ldexp(1.0 + m / 8.0, e - 7);
  return (code & 0x80) ? -mag : mag;
}

uint8_t oracle_e4m3_encode(float v) {
  const uint8_t sign = std::signbit(v) ? 0x80 : 0;
  /* 127 finite magnitudes, codes 0x00..0x7E. */
  return static_cast<uint8_t>(sign | nearest_magnitude_code(std::fabs(static_cast<double>(v)), 127,
                                                            e4m3_magnitude));
}

void oracle_e2m1_encode_array(const float* x, int64_t n, uint8_t* out) {
  IeeeMode ieee;
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(x[i]);
}

void oracle_e4m3_encode_array(const float* x, int64_t n, uint8_t* out) {
  IeeeMode ieee;
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(x[i]);
}

int oracle_key_mean(const uint16_t* x, int32_t B, int32_t L, int32_t H, int32_t d,
                    int64_t token_stride, float* mean) {
  if (!x || !mean || B <= 0 || L <= 0 || L > (1 << 23) || H <= 0 || d <= 0 ||
      token_stride < static_cast<int64_t>(H) * d)
    return -1;
  for (int32_t b = 0; b < B; ++b)
    for (int32_t h = 0; h < H; ++h)
      for (int32_t i = 0; i < d; ++i) {
        /* the exact sum of the channel, as counts of 2^-133 (every bf16 value is a whole number of
         * them): positive and negative values kept apart, each a non-negative big integer */
        BigNat pos, neg;
        for (int32_t t = 0; t < L; ++t) {
          const uint16_t v = x[(static_cast<int64_t>(b) * L + t) * token_stride + static_cast<int64_t>(h) * d + i];
          const int e = (v >> 7) & 0xFF, f = v & 0x7F;
          /* |v| = f * 2^-133 (e == 0), else (128 + f) * 2^(e - 134) = ((128 + f) << (e - 1)) * 2^-133 */
          const uint32_t m = e == 0 ? static_cast<uint32_t>(f) : static_cast<uint32_t>(128 + f);
          const int shift = e == 0 ? 0 : e - 1;
          ((v & 0x8000) ? neg : pos).add_shifted(m, shift);
        }
        mean[(static_cast<int64_t>(b) * H + h) * d + i] = exact_mean_to_float(pos, neg, static_cast<uint32_t>(L));
      }
  return 0;
}

int oracle_quantize_chunk_ex(const uint16_t* x, int32_t B, int32_t L, int32_t H, int32_t d,
                             int64_t token_stride, const float* mean, int32_t adaptive_scale,
                             uint8_t* codes, uint8_t* scales, float* gscale) {
  if (!x || !codes || !scales || !gscale || B <= 0 || L <= 0 || H <= 0 || d <= 0 || d % 16 != 0 ||
      token_stride < static_cast<int64_t>(H) * d || (adaptive_scale != 0 && adaptive_scale != 1))
    return -1;
  IeeeMode ieee;
  const int nblk = d / 16;
  const float kFp8Max = 448.0f;  /* M_FP8 */
  const float kFp4Max = 6.0f;    /* M_FP4 */
  for (int32_t b = 0; b < B; ++b) {
    for (int32_t h = 0; h < H; ++h) {
      /* the element to quantise: the bf16 input, less the channel mean when K is smoothed */
      auto elem = [&](int32_t t, int32_t i) {
        const float v = bf16_bits_to_float(x[(static_cast<int64_t>(b) * L + t) * token_stride +
                                             static_cast<int64_t>(h) * d + i]);
        return mean ? v - mean[(static_cast<int64_t>(b) * H + h) * d + i] : v;
      };
      /* FP32 scale of this (chunk, head). */
      float A = 0.0f;
      for (int32_t t = 0; t < L; ++t)
        for (int32_t i = 0; i < d; ++i) A = std::fmax(A, std::fabs(elem(t, i)));
      const float g = (A == 0.0f) ? 0.0f : A / (kFp8Max * kFp4Max);
      gscale[static_cast<int64_t>(b) * H + h] = g;

      const int64_t row0 = (static_cast<int64_t>(b) * H + h) * L;
      for (int32_t t = 0; t < L; ++t) {
        uint8_t* crow = codes + (row0 + t) * (d / 2);
        uint8_t* srow = scales + (row0 + t) * nblk;
        std::memset(crow, 0, static_cast<size_t>(d / 2));
        for (int blk = 0; blk < nblk; ++blk) {
          float ab = 0.0f;
          for (int k = 0; k < 16; ++k) ab = std::fmax(ab, std::fabs(elem(t, blk * 16 + k)));
          /* one candidate per scale target: target 6, and target 4 when the scale is adaptive */
          uint8_t best_s = 0, best_q[16] = {0};
          double best_err = 0.0;
          const int n_targets = adaptive_scale ? 2 : 1;
          for (int cand = 0; cand < n_targets; ++cand) {
            const float target = cand == 0 ? kFp4Max : 4.0f;
            uint8_t s_code = 0, q[16] = {0};
            if (ab != 0.0f && g != 0.0f) {
              const float denom = target * g;
              const float s_raw = ab / denom;
              s_code = oracle_e4m3_encode(s_raw);
            }
            const float s = static_cast<float>(oracle_e4m3_decode(s_code));
            if (s != 0.0f) {
              const float sg = s * g;
              const float r = 1.0f / sg;
              if (std::isfinite(r)) /* else the scale product underflowed: codes stay 0 */
                for (int k = 0; k < 16; ++k) q[k] = oracle_e2m1_encode(elem(t, blk * 16 + k) * r);
            }
            double err = 0.0;
            if (adaptive_scale)
              for (int k = 0; k < 16; ++k) {
                const double xhat = oracle_e2m1_decode(q[k]) * oracle_e4m3_decode(s_code) * static_cast<double>(g);
                const double diff = static_cast<double>(elem(t, blk * 16 + k)) - xhat;
                const double sq = diff * diff;
                err = err + sq;
              }
            if (cand == 0 || err < best_err) { /* strictly smaller: ties keep target 6 */
              best_err = err;
              best_s = s_code;
              for (int k = 0; k < 16; ++k) best_q[k] = q[k];
            }
          }
          srow[blk] = best_s;
          for (int k = 0; k < 16; ++k) {
            const int i = blk * 16 + k;
            crow[i / 2] |= static_cast<uint8_t>((i % 2 == 0) ? best_q[k] : (best_q[k] << 4));
          }
        }
      }
    }
  }
  return 0;
}

int oracle_quantize_chunk(const uint16_t* x, int32_t B, int32_t L, int32_t H, int32_t d,
                          int64_t token_stride, uint8_t* codes, uint8_t* scales, float* gscale) {
  return oracle_quantize_chunk_ex(x, B, L, H, d, token_stride, nullptr, 0, codes, scales, gscale);
}

int oracle_dequantize(const uint8_t* codes, const uint8_t* scales, const float* gscale, int32_t B,
                      int32_t H, int32_t d, int32_t chunk_tokens, int32_t capacity, double* out) {
  if (!codes || !scales || !gscale || !out || B <= 0 || H <= 0 || d <= 0 || d % 16 != 0 ||
      chunk_tokens <= 0 || capacity <= 0)
    return -1;
  const int64_t T = static_cast<int64_t>(chunk_tokens) * capacity;
  for (int32_t b = 0; b < B; ++b)
    for (int32_t h = 0; h < H; ++h)
      for (int64_t t = 0; t < T; ++t) {
        const int64_t row = (static_cast<int64_t>(b) * H + h) * T + t;
        const double g = gscale[(static_cast<int64_t>(b) * H + h) * capacity + t / chunk_tokens];
        for (int32_t i = 0; i < d; ++i) {
          const uint8_t byte = codes[row * (d / 2) + i / 2];
          const uint8_t q = (i % 2 == 0) ? (byte & 0xF) : (byte >> 4);
          const double s = oracle_e4m3_decode(scales[row * (d / 16) + i / 16]);
          out[row * d + i] = oracle_e2m1_decode(q) * s * g;
        }
      }
  return 0;
}

int oracle_visible_chunks(int32_t q_chunk, int32_t n_sink, int32_t window, int32_t capacity,
                          int32_t* out) {
  if (!out || capacity <= 0 || q_chunk < 0 || q_chunk >= capacity || n_sink < 0 || window < 1)
    return -1;
  int n = 0;
  for (int32_t c = 0; c < capacity; ++c) {
    const bool in_sink = c < n_sink;                             /* A_g */
    const bool in_window = (c > q_chunk - window) && (c <= q_chunk); /* sliding window */
    if (in_sink || in_window) out[n++] = c;                      /* union: each chunk once */
  }
  return n;
}

int oracle_multishot_chunks(int32_t q_chunk, int32_t n_sink, int32_t window, int32_t shot_start,
                            int32_t shot_len, int32_t capacity, int32_t* out) {
  /* the shot sink is the start of the current shot: history, never past the query chunk */
  if (!out || capacity <= 0 || q_chunk < 0 || q_chunk >= capacity || n_sink < 0 || window < 1 ||
      shot_start < 0 || shot_len < 0 || shot_start + shot_len > q_chunk + 1)
    return -1;
  int n = 0;
  for (int32_t c = 0; c < capacity; ++c) {
    const bool global_sink = c < n_sink;                                  /* A_g */
    const bool shot_sink = c >= shot_start && c < shot_start + shot_len;  /* A_s = (start, len) */
    const bool in_window = (c > q_chunk - window) && (c <= q_chunk);      /* sliding window */
    if (global_sink || shot_sink || in_window) out[n++] = c;             /* union, each chunk once */
  }
  return n;
}

}  // extern "C"

namespace {

/* fp64 attention of the requested rows over the keys of the chunk slots vis[0..nvis) (ascending,
 * distinct): the plain definition, two passes per row. */
int attention_over_slots(const uint16_t* q, int32_t B, int32_t Lq, int32_t H, int32_t d,
                         int64_t q_token_stride,
                         const uint8_t* k_codes, const uint8_t* k_scales, const float* k_gscale,
                         const uint8_t* v_codes, const uint8_t* v_scales, const float* v_gscale,
                         int32_t chunk_tokens, int32_t capacity, const int32_t* vis, int nvis,
                         double softmax_scale, const int32_t* rows, int32_t n_rows, double* out,
                         const float* k_mean) {
  if (!q || !k_codes || !k_scales || !k_gscale || !v_codes || !v_scales || !v_gscale || !rows ||
      !out || B <= 0 || Lq <= 0 || H <= 0 || d <= 0 || d % 16 != 0 || chunk_tokens <= 0 ||
      capacity <= 0 || n_rows < 0 || q_token_stride < static_cast<int64_t>(H) * d || nvis < 0)
    return -1;
  const double sigma = softmax_scale > 0.0 ? softmax_scale : 1.0 / std::sqrt(static_cast<double>(d));
  const int64_t T = static_cast<int64_t>(chunk_tokens) * capacity;

  /* x_hat of one cached token (fp64, exact). */
  auto dequant_row = [&](const uint8_t* codes, const uint8_t* scales, const float* gs, int32_t b,
                         int32_t h, int64_t t, double* dst) {
    const int64_t row = (static_cast<int64_t>(b) * H + h) * T + t;
    const double g = gs[(static_cast<int64_t>(b) * H + h) * capacity + t / chunk_tokens];
    for (int32_t i = 0; i < d; ++i) {
      const uint8_t byte = codes[row * (d / 2) + i / 2];
      const uint8_t c = (i % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      dst[i] = oracle_e2m1_decode(c) * oracle_e4m3_decode(scales[row * (d / 16) + i / 16]) * g;
    }
  };
  /* a smoothed key is x_hat' + mu of its chunk (mu: [B][H][capacity][d] fp32) */
  auto add_mean = [&](int32_t b, int32_t h, int64_t t, double* dst) {
    if (!k_mean) return;
    const float* mu = k_mean + ((static_cast<int64_t>(b) * H + h) * capacity + t / chunk_tokens) * d;
    for (int32_t i = 0; i < d; ++i) dst[i] += static_cast<double>(mu[i]);
  };

  /* The visible keys of one (b, h), dequantised once and reused for every requested row of
   * that (b, h); the arithmetic per row is unchanged. */
  std::vector<int64_t> keys;
  for (int n = 0; n < nvis; ++n)
    for (int32_t j = 0; j < chunk_tokens; ++j)
      keys.push_back(static_cast<int64_t>(vis[n]) * chunk_tokens + j);
  const size_t nk = keys.size();
  std::vector<double> khat(nk * d), vhat(nk * d);
  int32_t cached_b = -1, cached_h = -1;

  std::vector<double> qrow(static_cast<size_t>(d)), o(static_cast<size_t>(d)), s(nk);
  for (int32_t r = 0; r < n_rows; ++r) {
    const int32_t b = rows[3 * r + 0], h = rows[3 * r + 1], i = rows[3 * r + 2];
    if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= Lq) return -1;
    if (b != cached_b || h != cached_h) {
      for (size_t k = 0; k < nk; ++k) {
        dequant_row(k_codes, k_scales, k_gscale, b, h, keys[k], &khat[k * d]);
        add_mean(b, h, keys[k], &khat[k * d]);
        dequant_row(v_codes, v_scales, v_gscale, b, h, keys[k], &vhat[k * d]);
      }
      cached_b = b;
      cached_h = h;
    }
    for (int32_t e = 0; e < d; ++e)
      qrow[e] = bf16_bits_to_float(q[(static_cast<int64_t>(b) * Lq + i) * q_token_stride +
                                     static_cast<int64_t>(h) * d + e]);
    /* pass 1: logits over every visible key */
    double smax = -std::numeric_limits<double>::infinity();
    for (size_t k = 0; k < nk; ++k) {
      double dot = 0.0;
      for (int32_t e = 0; e < d; ++e) dot += qrow[e] * khat[k * d + e];
      s[k] = sigma * dot;
      smax = std::fmax(smax, s[k]);
    }
    /* pass 2: weights and the weighted sum of values */
    double denom = 0.0;
    for (int32_t e = 0; e < d; ++e) o[e] = 0.0;
    for (size_t k = 0; k < nk; ++k) {
      const double p = std::exp(s[k] - smax);
      denom += p;
      for (int32_t e = 0; e < d; ++e) o[e] += p * vhat[k * d + e];
    }
    for (int32_t e = 0; e < d; ++e) out[static_cast<int64_t>(r) * d + e] = o[e] / denom;
  }
  return 0;
}

}  // namespace

extern "C" {

int oracle_attention_rows(const uint16_t* q, int32_t B, int32_t Lq, int32_t H, int32_t d,
                          int64_t q_token_stride,
                          const uint8_t* k_codes, const uint8_t* k_scales, const float* k_gscale,
                          const uint8_t* v_codes, const uint8_t* v_scales, const float* v_gscale,
                          int32_t chunk_tokens, int32_t capacity,
                          int32_t q_chunk, int32_t n_sink, int32_t window, double softmax_scale,
                          const int32_t* rows, int32_t n_rows, double* out) {
  if (capacity <= 0) return -1;
  std::vector<int32_t> vis(static_cast<size_t>(capacity));
  const int nvis = oracle_visible_chunks(q_chunk, n_sink, window, capacity, vis.data());
  if (nvis < 0) return -1;
  return attention_over_slots(q, B, Lq, H, d, q_token_stride, k_codes, k_scales, k_gscale, v_codes,
                              v_scales, v_gscale, chunk_tokens, capacity, vis.data(), nvis,
                              softmax_scale, rows, n_rows, out, nullptr);
}

int oracle_attention_rows_slots_kmean(const uint16_t* q, int32_t B, int32_t Lq, int32_t H, int32_t d,
                                      int64_t q_token_stride,
                                      const uint8_t* k_codes, const uint8_t* k_scales, const float* k_gscale,
                                      const float* k_mean,
                                      const uint8_t* v_codes, const uint8_t* v_scales, const float* v_gscale,
                                      int32_t chunk_tokens, int32_t capacity, const int32_t* slots,
                                      int32_t n_slots, double softmax_scale, const int32_t* rows,
                                      int32_t n_rows, double* out) {
  if (capacity <= 0 || !slots || n_slots < 1) return -1;
  std::vector<char> listed(static_cast<size_t>(capacity), 0);  /* the union of the listed slots */
  for (int32_t i = 0; i < n_slots; ++i) {
    if (slots[i] < 0 || slots[i] >= capacity) return -1;
    listed[static_cast<size_t>(slots[i])] = 1;
  }
  std::vector<int32_t> vis;
  for (int32_t c = 0; c < capacity; ++c)
    if (listed[static_cast<size_t>(c)]) vis.push_back(c);
  return attention_over_slots(q, B, Lq, H, d, q_token_stride, k_codes, k_scales, k_gscale, v_codes,
                              v_scales, v_gscale, chunk_tokens, capacity, vis.data(),
                              static_cast<int>(vis.size()), softmax_scale, rows, n_rows, out, k_mean);
}

int oracle_attention_rows_slots(const uint16_t* q, int32_t B, int32_t Lq, int32_t H, int32_t d,
                                int64_t q_token_stride,
                                const uint8_t* k_codes, const uint8_t* k_scales, const float* k_gscale,
                                const uint8_t* v_codes, const uint8_t* v_scales, const float* v_gscale,
                                int32_t chunk_tokens, int32_t capacity, const int32_t* slots,
                                int32_t n_slots, double softmax_scale, const int32_t* rows,
                                int32_t n_rows, double* out) {
  return oracle_attention_rows_slots_kmean(q, B, Lq, H, d, q_token_stride, k_codes, k_scales, k_gscale,
                                           nullptr, v_codes, v_scales, v_gscale, chunk_tokens, capacity,
                                           slots, n_slots, softmax_scale, rows, n_rows, out);
}

}  // extern "C"
