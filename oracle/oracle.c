/*
 * CPU oracle for the GEMM library. TEST INFRASTRUCTURE ONLY: only the tests,
 * the smoke check and the bench's CPU-baseline leg may load it. The product path
 * never calls it, and it shares no code with the CUDA kernels.
 *
 * What it computes, with the passage each function follows:
 *
 *  - orc_gemm: C[i,j] = cast_out(act(sum_k a[i,k]*b[k,j] + bias[j])), the plain
 *    triple loop that "DeepGEMM kernel-library walkthrough" (zwxr.cn), section 3.2
 *    names the golden reference, with a double accumulator in ascending k, the
 *    activation in double, and ONE round-to-nearest-even from double to the
 *    output type. FP32 accumulation of low-precision inputs: same page, section 2.4.
 *    Linear = GEMM + bias add, then activation: "为什么我们要死磕GEMM" (kwkr.cn),
 *    sections 2.1 and 5.1; fused epilogue: walkthrough section 5.1.
 *  - orc_e4m3_encode / orc_e4m3_decode: the OCP FP8 E4M3 ("FN") format (bias 7,
 *    3 mantissa bits, max finite 448, no infinity, S.1111.111 = NaN), round to
 *    nearest even, saturating to +-448.
 *  - orc_quant_1x128 / orc_quant_128x128: group-scaled FP8 quantisation,
 *    walkthrough section 2.4: one FP32 scale per 1x128 row group (activations) or
 *    per 128x128 block (weights), scale = amax / 448, code = E4M3(x / scale).
 *  - orc_gemm_fp8: C[i,j] = cast_out(act(sum_kb sa[kb,i]*sb[kb,j/128] *
 *    sum_{k in kb} dec(qa[i,k])*dec(qb[j,k]) + bias[j])), in double, from the same
 *    quantised operands; walkthrough section 2.4 (accumulate high, rescale).
 *
 * Readings where the pages are silent: an all-zero group gets scale 1.0 (it avoids
 * 0/0, gives all-zero codes and dequantises to exactly 0); amax covers only the
 * elements present in a partial group, and the missing elements take no part in the
 * GEMM; x/scale is an IEEE float division (not a reciprocal multiply), and the scale
 * amax/448 is an FP32 division, not rounded to a power of two; rounding to zero keeps
 * the sign (code 0x80 for negative inputs); GeLU is the tanh form with sqrt(2/pi) and
 * 0.044715 (Hendrycks & Gimpel), SiLU is x*sigmoid(x); the bias is added to the
 * exact sum and the activation applied before the single rounding to the output type.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (no fast-math: every
 * float operation here is IEEE with round-to-nearest-even).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F16 = 2, ORC_E4M3 = 3, ORC_F64 = 4 };
enum { ORC_ACT_NONE = 0, ORC_ACT_GELU_TANH = 1, ORC_ACT_SILU = 2 };

/* ---------------------------------------------------------------- element decoding */

static double f16_bits_to_double(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  double v;
  if (e == 0) v = ldexp((double)m, -24);                 /* subnormal: m * 2^-14 * 2^-10 */
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp((double)(m | 0x400), e - 25);           /* (1024+m) * 2^(e-15-10) */
  return s ? -v : v;
}

static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

double orc_load(const void* p, int dtype, int64_t idx) {
  switch (dtype) {
    case ORC_F32: return (double)((const float*)p)[idx];
    case ORC_BF16: return bf16_bits_to_double(((const uint16_t*)p)[idx]);
    case ORC_F16: return f16_bits_to_double(((const uint16_t*)p)[idx]);
    case ORC_F64: return ((const double*)p)[idx];
    default: return NAN;
  }
}

/* ---------------------------------------------------------------- rounding to a format */

/* Round x to the nearest value with `prec` significand bits, minimum normal exponent
 * `emin` (so the subnormal quantum is 2^(emin-prec+1)), ties to even. Overflow of the
 * largest finite value `maxv` follows IEEE round-to-nearest: a result whose rounded
 * magnitude exceeds maxv becomes infinity. The division and multiplication by the
 * power-of-two quantum are exact; nearbyint rounds ties to even in the default mode. */
static double round_generic(double x, int prec, int emin, double maxv) {
  if (x == 0.0 || isnan(x) || isinf(x)) return x;
  int e2;
  frexp(fabs(x), &e2);                 /* |x| = f * 2^e2, f in [0.5, 1): leading bit 2^(e2-1) */
  int lead = e2 - 1;
  if (lead < emin) lead = emin;
  double quantum = ldexp(1.0, lead - (prec - 1));
  double r = nearbyint(x / quantum) * quantum;
  if (fabs(r) > maxv) return x > 0 ? INFINITY : -INFINITY;
  return r;
}

double orc_round_to(double x, int dtype) {
  switch (dtype) {
    case ORC_F32: return round_generic(x, 24, -126, 3.4028234663852886e38);
    case ORC_BF16: return round_generic(x, 8, -126, 3.3895313892515355e38);
    case ORC_F16: return round_generic(x, 11, -14, 65504.0);
    case ORC_F64: return x;
    default: return NAN;
  }
}

void orc_round_array(const double* x, int64_t n, int dtype, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_round_to(x[i], dtype);
}

/* ---------------------------------------------------------------- activations (double) */

/* sigmoid(z) = 1 / (1 + e^-z), written so that no step overflows or cancels: for z < 0
 * it is e^z / (1 + e^z) with e^z <= 1. */
static double orc_sigmoid(double z) {
  if (z >= 0.0) return 1.0 / (1.0 + exp(-z));
  const double e = exp(z);
  return e / (1.0 + e);
}

double orc_act(double x, int act) {
  switch (act) {
    case ORC_ACT_NONE: return x;
    case ORC_ACT_GELU_TANH: {
      /* GeLU, tanh form: 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3).
       * Since 1 + tanh(u) = 2 / (1 + e^(-2u)), this is x * sigmoid(2u); it is evaluated
       * in that form because 1 + tanh(u) cancels to nothing in double once u < -19
       * (x < -7), where the true value is still far above the smallest output values. */
      const double c = sqrt(2.0 / M_PI);
      const double u = c * (x + 0.044715 * x * x * x);
      return x * orc_sigmoid(2.0 * u);
    }
    case ORC_ACT_SILU:
      /* SiLU (Swish-1): x * sigmoid(x) = x / (1 + e^-x) */
      return x * orc_sigmoid(x);
    default: return NAN;
  }
}

/* ---------------------------------------------------------------- FP8 E4M3 codec */

double orc_e4m3_decode(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);                  /* m/8 * 2^(1-7) */
  else v = ldexp((double)(8 + m), e - 10);              /* (1 + m/8) * 2^(e-7) */
  return s ? -v : v;
}

uint8_t orc_e4m3_encode(float y) {
  if (isnan(y)) return 0x7F;
  uint8_t sign = signbit(y) ? 0x80 : 0x00;
  double a = fabs((double)y);
  if (a >= 448.0) return sign | 0x7E;                    /* saturate (satfinite) */
  /* E4M3: 4 significand bits (1 implicit + 3), minimum normal exponent -6. */
  double r = round_generic(a, 4, -6, 448.0);
  if (r == 0.0) return sign;                             /* keeps the sign: 0x80 for -0 */
  if (r < ldexp(1.0, -6)) return sign | (uint8_t)(r / ldexp(1.0, -9));   /* subnormal m */
  int e2;
  double f = frexp(r, &e2);                              /* r = f * 2^e2, f in [0.5,1) */
  int e = (e2 - 1) + 7;                                  /* biased exponent */
  int m = (int)((f * 2.0 - 1.0) * 8.0);                  /* exact: r has 4 significant bits */
  return sign | (uint8_t)((e << 3) | m);
}

void orc_e4m3_encode_array(const float* y, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(y[i]);
}

void orc_e4m3_decode_array(const uint8_t* c, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(c[i]);
}

/* ---------------------------------------------------------------- FP8 group quantiser */

/* The scale of one group from its amax: amax / 448 as an IEEE float division;
 * an all-zero group gets 1.0 (reading: the pages are silent; this avoids 0/0). */
static float group_scale(float amax) {
  if (amax == 0.0f) return 1.0f;
  volatile float s = amax / 448.0f;
  return s;
}

/* 1x128 groups along the columns of X[rows, cols], X[r,c] = X[r*rs + c*cs].
 * Q[r*cols + c] = E4M3(X[r,c] / S[kb*rows + r]) with kb = c / 128. */
void orc_quant_1x128(const float* X, int64_t rows, int64_t cols, int64_t rs, int64_t cs,
                     uint8_t* Q, float* S) {
  int64_t kb_n = (cols + 127) / 128;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t kb = 0; kb < kb_n; ++kb) {
      int64_t c0 = kb * 128, c1 = c0 + 128 < cols ? c0 + 128 : cols;
      float amax = 0.0f;
      for (int64_t c = c0; c < c1; ++c) {
        float v = fabsf(X[r * rs + c * cs]);
        if (v > amax) amax = v;
      }
      float s = group_scale(amax);
      S[kb * rows + r] = s;
      for (int64_t c = c0; c < c1; ++c) {
        volatile float y = X[r * rs + c * cs] / s;
        Q[r * cols + c] = orc_e4m3_encode(y);
      }
    }
  }
}

/* 128x128 blocks of the weight X[K, N], X[k,n] = X[k*rs + n*cs]. Codes are written
 * transposed, Q[n*K + k] (K contiguous), scales S[kb*NB + nb], NB = ceil(N/128). */
void orc_quant_128x128(const float* X, int64_t K, int64_t N, int64_t rs, int64_t cs,
                       uint8_t* Q, float* S) {
  int64_t kb_n = (K + 127) / 128, nb_n = (N + 127) / 128;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t kb = 0; kb < kb_n; ++kb) {
    for (int64_t nb = 0; nb < nb_n; ++nb) {
      int64_t k0 = kb * 128, k1 = k0 + 128 < K ? k0 + 128 : K;
      int64_t n0 = nb * 128, n1 = n0 + 128 < N ? n0 + 128 : N;
      float amax = 0.0f;
      for (int64_t k = k0; k < k1; ++k)
        for (int64_t n = n0; n < n1; ++n) {
          float v = fabsf(X[k * rs + n * cs]);
          if (v > amax) amax = v;
        }
      float s = group_scale(amax);
      S[kb * nb_n + nb] = s;
      for (int64_t k = k0; k < k1; ++k)
        for (int64_t n = n0; n < n1; ++n) {
          volatile float y = X[k * rs + n * cs] / s;
          Q[n * K + k] = orc_e4m3_encode(y);
        }
    }
  }
}

/* ---------------------------------------------------------------- GEMM (FP64) */

/* Selected outputs C[rows[r], cols[c]] -> out[r*ncols + c]; also absacc = sum_k |a||b|
 * (the scale of the tolerance bound) when absacc != NULL. The operands are first
 * copied into double scratch rows (A rows, B columns as K-contiguous rows) so the
 * inner loop is contiguous; the arithmetic is the plain ascending-k double sum. */
int orc_gemm(int64_t M, int64_t N, int64_t K,
             const void* A, int a_dtype, int64_t a_rs, int64_t a_cs,
             const void* B, int b_dtype, int64_t b_rs, int64_t b_cs,
             const void* bias, int bias_dtype, int act, int out_dtype,
             const int64_t* rows, int64_t nrows, const int64_t* cols, int64_t ncols,
             double* out, double* absacc) {
  (void)M; (void)N;
  double* arow = (double*)malloc(sizeof(double) * (size_t)(nrows * (K > 0 ? K : 1)));
  double* bcol = (double*)malloc(sizeof(double) * (size_t)(ncols * (K > 0 ? K : 1)));
  if (!arow || !bcol) { free(arow); free(bcol); return 1; }
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r)
    for (int64_t k = 0; k < K; ++k) arow[r * K + k] = orc_load(A, a_dtype, rows[r] * a_rs + k * a_cs);
#pragma omp parallel for schedule(static)
  for (int64_t c = 0; c < ncols; ++c)
    for (int64_t k = 0; k < K; ++k) bcol[c * K + k] = orc_load(B, b_dtype, k * b_rs + cols[c] * b_cs);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < nrows; ++r) {
    for (int64_t c = 0; c < ncols; ++c) {
      const double* a = arow + r * K;
      const double* b = bcol + c * K;
      double sum = 0.0, asum = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        sum += a[k] * b[k];
        asum += fabs(a[k]) * fabs(b[k]);
      }
      double x = sum;
      if (bias) x += orc_load(bias, bias_dtype, cols[c]);
      out[r * ncols + c] = orc_round_to(orc_act(x, act), out_dtype);
      if (absacc) absacc[r * ncols + c] = asum;
    }
  }
  free(arow);
  free(bcol);
  return 0;
}

/* FP8 block-scaled GEMM from codes: qa[M][K] (K contiguous), sa[kb*M + i],
 * qb[N][K] (K contiguous), sb[kb*NB + j/128]. absacc = sum_k |a^||b^| of the
 * dequantised operands a^ = dec(qa)*sa, b^ = dec(qb)*sb. */
int orc_gemm_fp8(int64_t M, int64_t N, int64_t K,
                 const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                 const void* bias, int bias_dtype, int act, int out_dtype,
                 const int64_t* rows, int64_t nrows, const int64_t* cols, int64_t ncols,
                 double* out, double* absacc) {
  int64_t kb_n = (K + 127) / 128, nb_n = (N + 127) / 128;
  double dec[256];
  for (int i = 0; i < 256; ++i) dec[i] = orc_e4m3_decode((uint8_t)i);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t i = rows[r];
    for (int64_t c = 0; c < ncols; ++c) {
      int64_t j = cols[c];
      double total = 0.0, asum = 0.0;
      for (int64_t kb = 0; kb < kb_n; ++kb) {
        int64_t k0 = kb * 128, k1 = k0 + 128 < K ? k0 + 128 : K;
        double part = 0.0, apart = 0.0;
        for (int64_t k = k0; k < k1; ++k) {
          double a = dec[qa[i * K + k]], b = dec[qb[j * K + k]];
          part += a * b;
          apart += fabs(a) * fabs(b);
        }
        double scale = (double)sa[kb * M + i] * (double)sb[kb * nb_n + j / 128];
        total += scale * part;
        asum += fabs(scale) * apart;
      }
      double x = total;
      if (bias) x += orc_load(bias, bias_dtype, j);
      out[r * ncols + c] = orc_round_to(orc_act(x, act), out_dtype);
      if (absacc) absacc[r * ncols + c] = asum;
    }
  }
  return 0;
}
