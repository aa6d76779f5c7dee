/*
 * Test-only check of the FMA division sequence the FP8 quantiser uses for x / s
 * (P. Markstein, "IA-64 and Elementary Functions", 2000, chapter 8; Muller et al.,
 * "Handbook of Floating-Point Arithmetic", division with an FMA):
 *
 *     r = RN(1 / s),  y = RN(x * r),  e = RN(x - y * s) (one FMA),  q = RN(y + e * r) (one FMA),
 *
 * with the sign of x ORed back into q, against the IEEE quotient RN(x / s). The
 * quantiser takes this path only when the scale's significand is not all ones and
 * 2^-90 <= s < infinity; the claim checked here is that, under those conditions, q
 * equals the IEEE quotient bit for bit whenever |x / s| > 2^-11, and that smaller
 * quotients (which E4M3 rounds to a signed zero) stay at or below 2^-10 with the
 * sign of x, so the E4M3 code is the same either way.
 *
 * Plain C, IEEE single precision with round-to-nearest-even: fmaf is the C library's
 * correctly rounded fused multiply-add and '/' the hardware's IEEE division. Build:
 * gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (the test compiles it).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float from_bits(uint32_t b) {
  float f;
  memcpy(&f, &b, 4);
  return f;
}

static uint32_t to_bits(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  return b;
}

/* mode 0: the sequence above. mode 1: the reciprocal product y alone (no residual
 * step), a deliberately wrong variant that shows the check can fail. */
static float fma_div(float x, float s, float r, int mode) {
  const float y = x * r;
  if (mode == 1) return y;
  const float e = fmaf(-y, s, x);
  const float q = fmaf(e, r, y);
  return from_bits(to_bits(q) | (to_bits(x) & 0x80000000u));
}

/* 1 if the sequence disagrees with IEEE division in a way that could change the code. */
static int disagrees(float x, float s, float r, int mode) {
  const float qi = x / s;
  const float qm = fma_div(x, s, r, mode);
  if (fabsf(qi) > 0x1p-11f) return to_bits(qi) != to_bits(qm);
  return !(fabsf(qm) <= 0x1p-10f && signbit(qm) == signbit(qi));
}

/* Every significand of x in the binade [2^x_exp, 2^(x_exp+1)), both signs, for one
 * scale s. Returns the number of disagreements; *first gets the bits of the smallest
 * disagreeing x of that binade (0 if none). */
int64_t mk_binade(float s, int x_exp, int mode, uint32_t* first) {
  const float r = 1.0f / s;
  int64_t bad = 0;
  uint32_t first_bad = 0;
  const uint32_t base = (uint32_t)(x_exp + 127) << 23;
#pragma omp parallel for reduction(+ : bad) schedule(static)
  for (int64_t m = 0; m < (1 << 23); ++m) {
    const float x = from_bits(base | (uint32_t)m);
    const int d = disagrees(x, s, r, mode) + disagrees(-x, s, r, mode);
    if (d) {
      bad += d;
#pragma omp critical
      if (first_bad == 0 || (uint32_t)m < (first_bad & 0x7fffffu)) first_bad = base | (uint32_t)m;
    }
  }
  *first = first_bad;
  return bad;
}

/* n pseudo-random x per quotient binade for quotients 2^-12 .. 2^9 (every binade a
 * group can produce, with amax / s <= 448 * (1 + 2^-23)), for each of the ns scales.
 * x is drawn as (random significand) * 2^e * s rounded to float, so it covers the
 * whole significand range relative to s. Returns the number of disagreements. */
int64_t mk_scales(const float* s_list, int64_t ns, int64_t n_per_binade, uint64_t seed) {
  int64_t bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(dynamic)
  for (int64_t i = 0; i < ns; ++i) {
    const float s = s_list[i];
    const float r = 1.0f / s;
    uint64_t st = seed ^ (0x9E3779B97F4A7C15ull * (uint64_t)(i + 1));
    for (int e = -12; e <= 9; ++e) {
      for (int64_t j = 0; j < n_per_binade; ++j) {
        st ^= st << 13;
        st ^= st >> 7;
        st ^= st << 17;
        const float frac = from_bits(0x3f800000u | (uint32_t)(st & 0x7fffffu));  /* [1, 2) */
        const float x = (float)((double)frac * ldexp(1.0, e) * (double)s);
        if (!isfinite(x) || fabsf(x) > 448.0f * s * (1.0f + 0x1p-23f)) continue;
        bad += disagrees(x, s, r, 0) + disagrees(-x, s, r, 0);
      }
    }
  }
  return bad;
}
