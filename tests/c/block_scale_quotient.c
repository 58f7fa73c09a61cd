/* Host check of the quantiser's block-scale quotient shortcut.  For a chunk maximum A (a bf16
 * value), d = RN(T * RN(A / 2688)) for the scale target T (6, or 4 for the adaptive candidate);
 * the kernel takes q = RN(a * y) with y = RN(1 / d), then q' = RN(q + RN(a - q * d) * y) (two
 * FMAs), instead of RN(a / d), whenever d and y are normal and a >= 2^-100.  Only the E4M3 code
 * of the quotient is stored, so the check compares codes: E4M3 round-to-nearest-even with
 * saturation at 448, found by nearest-value search.
 * Usage: block_scale_quotient N_CHUNK_MAXIMA GUARD(0|1) [T]; N_CHUNK_MAXIMA = 0 takes every
 * positive finite bf16 chunk maximum; prints "tested T mismatches M". */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static double e4m3_value(int c) { /* positive codes 0..126 */
  int e = (c >> 3) & 15, m = c & 7;
  return e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
}

static int e4m3_rne(float q) {
  int best = 0;
  double bd = 1e300;
  for (int c = 0; c <= 126; ++c) {
    double dd = fabs((double)q - e4m3_value(c));
    if (dd < bd || (dd == bd && (c & 1) == 0)) {
      bd = dd;
      best = c;
    }
  }
  return best;
}

int main(int argc, char** argv) {
  const int n_arg = argc > 1 ? atoi(argv[1]) : 600;
  const int guard = argc > 2 ? atoi(argv[2]) : 1;
  const float target = argc > 3 ? (float)atof(argv[3]) : 6.0f;
  const int all = n_arg == 0;
  const int n_max = all ? 0x7F7F : n_arg;
  long tested = 0, mism = 0;
  uint64_t st = 88172645463325252ull;
  for (int ai = 0; ai < n_max; ++ai) {
    st ^= st << 13;
    st ^= st >> 7;
    st ^= st << 17;
    uint16_t abits = (uint16_t)(st % 0x7F80u);
    if (ai < 64) abits = (uint16_t)(0x0001 + ai * 0x01FF); /* the small end, subnormals included */
    if (all) abits = (uint16_t)(ai + 1);                     /* 0x0001 .. 0x7F7F: every one */
    const float A = bf16(abits);
    if (A == 0.0f) continue;
    const float g = A / 2688.0f;
    const float d = target * g;
    const float y = 1.0f / d;
    if (!isnormal(d) || !isnormal(y)) continue; /* the kernel divides for these chunks */
    for (uint32_t b = 1; b <= abits; ++b) {
      const float a = bf16((uint16_t)b);
      if (guard && a < 0x1p-100f) continue; /* the kernel divides for these blocks */
      const float q0 = a / d;
      const float q = a * y;
      const float r = fmaf(-q, d, a);
      const float q1 = fmaf(r, y, q);
      ++tested;
      if (q0 != q1 && e4m3_rne(q0) != e4m3_rne(q1)) ++mism;
    }
  }
  printf("tested %ld mismatches %ld\n", tested, mism);
  return 0;
}
