// Fused GEMM epilogue: FP32 accumulator + bias[n] -> activation -> one round-to-
// nearest-even cast to the output type -> store. The bias add and activation run in
// registers before the single write-back, as the DeepGEMM kernel-library walkthrough
// (zwxr.cn), section 5.1 recommends; "为什么我们要死磕GEMM" (kwkr.cn), section 2.1
// defines the linear layer as GEMM + bias add.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "fp8_codec.cuh"

namespace smg {

struct EpiArgs {
  int M, N;            // output C is M x N, row-major
  const void* bias;    // nullable, N entries
  int bias_dtype;      // kF32 / kBF16 / kF16
  int act;             // kActNone / kActGeluTanh / kActSilu
  void* C;
  int c_dtype;         // kF32 / kBF16 / kF16, or 3 = E4M3 codes with per-1x128 scales
  long long ldc;
  float* scales;       // E4M3 output only: [ceil(N/128)][M] group scales
};

// Activations. Both are x * sigmoid(z): SiLU with z = x, and the tanh-form GeLU with
// z = 2u, u = sqrt(2/pi) (x + 0.044715 x^3), because 0.5 x (1 + tanh(u)) = x / (1 + e^(-2u)).
// The sigmoid is taken as 1 / (1 + e) for z >= 0 and e / (1 + e) for z < 0, with
// e = e^(-|z|) <= 1: nothing overflows and nothing cancels, so the result keeps its
// relative accuracy far out in the negative tail, where 1 + tanh(u) would round to
// nothing (x < -5 in FP32).
//
// 16-bit and FP8 outputs use the FP32 form below: e^(-a) = 2^(-a log2 e) on the
// special-function unit (ex2.approx.f32, results down to the subnormal range kept) and
// an approximate reciprocal of 1 + e in [1, 2]. Its relative error is below 2^-16 for
// every input (the rounding of a log2 e, |a| log2 e <= 150, is the largest term),
// against the 2^-8 (BF16) and 2^-11 (FP16) spacing of the outputs, and the GeLU/SiLU
// arithmetic stays a dozen instructions per element, so the epilogue warps keep pace
// with the tensor cores. FP32 outputs add the bias and evaluate the activation in
// double precision (libm exp) and round once, so they are within one FP32 ulp of the
// exact value even where the accumulator contributes nothing.
__device__ __forceinline__ float exp2_sfu(float y) {
  float r;
  asm("ex2.approx.f32 %0, %1;" : "=f"(r) : "f"(y));
  return r;
}

__device__ __forceinline__ float rcp_sfu(float d) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
  return r;
}

// x * sigmoid(z) in FP32. Below 2^-120, e = 2^t is formed as 2^(t + 64) * 2^-64, so the
// final multiply (IEEE, subnormals kept) rounds it into the subnormal range correctly
// whatever the special-function unit does with subnormal results.
__device__ __forceinline__ float x_sigmoid_f32(float x, float z) {
  const float t = -fabsf(z) * 1.4426950408889634f;  // log2(e)
  const bool tiny = t < -120.0f;
  float e = exp2_sfu(tiny ? t + 64.0f : t);
  if (tiny) e *= 5.421010862427522e-20f;           // 2^-64
  const float r = rcp_sfu(1.0f + e);
  return z >= 0.0f ? x * r : (x * e) * r;
}

// GeLU's z = 2 sqrt(2/pi) (x + 0.044715 x^3) = x (kGeluA + kGeluB x^2).
constexpr float kGeluA = 1.5957691216057308f;   // 2 sqrt(2/pi)
constexpr float kGeluB = 0.07135481627260025f;  // 2 sqrt(2/pi) 0.044715

__device__ __forceinline__ float act_apply(float x, int act) {
  if (act == 1) return x_sigmoid_f32(x, x * fmaf(kGeluB, x * x, kGeluA));
  if (act == 2) return x_sigmoid_f32(x, x);
  return x;
}

// The same for two elements: the FP32 arithmetic as packed FP32x2 operations (each half
// rounded exactly like the scalar operation, so results equal act_apply's), the
// exponential and the reciprocal on the special-function unit one element at a time.
__device__ __forceinline__ float2 x_sigmoid_f32x2(float2 x, float2 z) {
  const float2 t = __fmul2_rn(make_float2(fabsf(z.x), fabsf(z.y)),
                              make_float2(-1.4426950408889634f, -1.4426950408889634f));
  const bool tiny0 = t.x < -120.0f, tiny1 = t.y < -120.0f;
  float e0 = exp2_sfu(tiny0 ? t.x + 64.0f : t.x);
  float e1 = exp2_sfu(tiny1 ? t.y + 64.0f : t.y);
  if (tiny0) e0 *= 5.421010862427522e-20f;  // 2^-64
  if (tiny1) e1 *= 5.421010862427522e-20f;
  const float2 d = __fadd2_rn(make_float2(1.0f, 1.0f), make_float2(e0, e1));
  const float2 r = make_float2(rcp_sfu(d.x), rcp_sfu(d.y));
  // x * r for z >= 0, (x * e) * r below (x * 1 is exact).
  const float2 xe = __fmul2_rn(x, make_float2(z.x >= 0.0f ? 1.0f : e0, z.y >= 0.0f ? 1.0f : e1));
  return __fmul2_rn(xe, r);
}

__device__ __forceinline__ float2 act_apply2(float2 x, int act) {
  if (act == 1) {
    const float2 p = __ffma2_rn(make_float2(kGeluB, kGeluB), __fmul2_rn(x, x), make_float2(kGeluA, kGeluA));
    return x_sigmoid_f32x2(x, __fmul2_rn(x, p));
  }
  if (act == 2) return x_sigmoid_f32x2(x, x);
  return x;
}

__device__ __forceinline__ double x_sigmoid_f64(double x, double z) {
  const double e = exp(-fabs(z));
  const double r = 1.0 / (1.0 + e);
  return z >= 0.0 ? x * r : (x * e) * r;
}

__device__ __forceinline__ double act_apply_f64(double x, int act) {
  if (act == 1) {
    const double u = 0.79788456080286535588 * (x + 0.044715 * x * x * x);
    return x_sigmoid_f64(x, 2.0 * u);
  }
  if (act == 2) return x_sigmoid_f64(x, x);
  return x;
}

__device__ __forceinline__ float load_bias(const void* bias, int dtype, int idx) {
  if (dtype == 0) return static_cast<const float*>(bias)[idx];
  if (dtype == 1) return __bfloat162float(static_cast<const __nv_bfloat16*>(bias)[idx]);
  return __half2float(static_cast<const __half*>(bias)[idx]);
}

__device__ __forceinline__ void store_one(void* C, int dtype, long long off, float x) {
  if (dtype == 0) static_cast<float*>(C)[off] = x;
  else if (dtype == 1) static_cast<__nv_bfloat16*>(C)[off] = __float2bfloat16_rn(x);
  else static_cast<__half*>(C)[off] = __float2half_rn(x);
}

// In-place bias add and activation over 32 values. Every branch is taken once per
// chunk, outside the per-element loops, so the common plain path jumps over these
// blocks in one step and stays a short, straight run of instructions (the epilogue
// warps share instruction caches with the producer and MMA-issuer warps).
// bias[col0 .. col0 + 32) added to v with 16-byte loads (two 16-bit values per word);
// one branch on the bias type and alignment per chunk, none per element. kPacked: the
// adds as packed FP32x2 operations (same results, half the instructions; the FP8
// promotion kernels, short of registers, keep the scalar form).
template <bool kPacked = true>
__device__ __forceinline__ void add_bias32_vec(const EpiArgs& e, int col0, float (&v)[32]) {
  if (e.bias_dtype == 0) {
    const float4* b4 = reinterpret_cast<const float4*>(static_cast<const float*>(e.bias) + col0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 b = __ldg(b4 + q);
      if constexpr (kPacked) {
        const float2 lo = __fadd2_rn(make_float2(v[4 * q], v[4 * q + 1]), make_float2(b.x, b.y));
        const float2 hi = __fadd2_rn(make_float2(v[4 * q + 2], v[4 * q + 3]), make_float2(b.z, b.w));
        v[4 * q] = lo.x;
        v[4 * q + 1] = lo.y;
        v[4 * q + 2] = hi.x;
        v[4 * q + 3] = hi.y;
      } else {
        v[4 * q] += b.x;
        v[4 * q + 1] += b.y;
        v[4 * q + 2] += b.z;
        v[4 * q + 3] += b.w;
      }
    }
  } else {
    const uint4* b4 = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(e.bias) + col0);
    const bool is_bf16 = e.bias_dtype == 1;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 b = __ldg(b4 + q);
      const uint32_t w[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float2 f;
        if (is_bf16) {
          f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[h]));
        } else {
          f = __half22float2(*reinterpret_cast<const __half2*>(&w[h]));
        }
        if constexpr (kPacked) {
          const float2 y = __fadd2_rn(make_float2(v[8 * q + 2 * h], v[8 * q + 2 * h + 1]), f);
          v[8 * q + 2 * h] = y.x;
          v[8 * q + 2 * h + 1] = y.y;
        } else {
          v[8 * q + 2 * h] += f.x;
          v[8 * q + 2 * h + 1] += f.y;
        }
      }
    }
  }
}

// FP32 output with an activation: bias add and activation in double, one rounding.
// The loop is not unrolled (one copy of the double-precision code) and always works
// on v[0], rotating the array by one after each element, so v stays in registers.
__device__ __forceinline__ void epi_bias_act32_f64(const EpiArgs& e, int col0, float (&v)[32]) {
#pragma unroll 1
  for (int j = 0; j < 32; ++j) {
    double x = static_cast<double>(v[0]);
    if (e.bias != nullptr && col0 + j < e.N) x += static_cast<double>(load_bias(e.bias, e.bias_dtype, col0 + j));
    const float y = __double2float_rn(act_apply_f64(x, e.act));
#pragma unroll
    for (int k = 0; k < 31; ++k) v[k] = v[k + 1];
    v[31] = y;
  }
}

template <bool kPacked = true>
__device__ __forceinline__ void epi_bias_act32(const EpiArgs& e, int col0, float (&v)[32]) {
  if (e.act != 0 && e.c_dtype == 0) {
    epi_bias_act32_f64(e, col0, v);
    return;
  }
  if (e.bias != nullptr) {
    const int esz = e.bias_dtype == 0 ? 4 : 2;
    const bool aligned = ((reinterpret_cast<uintptr_t>(e.bias) + static_cast<uintptr_t>(col0) * esz) & 15u) == 0;
    if (col0 + 32 <= e.N && aligned) {
      add_bias32_vec<kPacked>(e, col0, v);
    } else if (col0 + 32 <= e.N) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += load_bias(e.bias, e.bias_dtype, col0 + j);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < e.N) v[j] += load_bias(e.bias, e.bias_dtype, col0 + j);
    }
  }
  if constexpr (kPacked) {
    if (e.act == 1) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 y = act_apply2(make_float2(v[2 * j], v[2 * j + 1]), 1);
        v[2 * j] = y.x;
        v[2 * j + 1] = y.y;
      }
    } else if (e.act == 2) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 y = act_apply2(make_float2(v[2 * j], v[2 * j + 1]), 2);
        v[2 * j] = y.x;
        v[2 * j + 1] = y.y;
      }
    }
  } else {
    if (e.act == 1) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = act_apply(v[j], 1);
    } else if (e.act == 2) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = act_apply(v[j], 2);
    }
  }
}

// Stores 32 finished values of one output row (vector stores when the chunk is whole;
// the host guarantees 16-byte aligned C and ldc*elem_size).
__device__ __forceinline__ void epi_store_row32(const EpiArgs& e, int row, int col0, const float (&v)[32]) {
  if (row >= e.M) return;
  const long long base = static_cast<long long>(row) * e.ldc + col0;
  if (col0 + 32 <= e.N) {
    if (e.c_dtype == 1) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(e.C) + base);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          __nv_bfloat162 t = __floats2bfloat162_rn(v[8 * j + 2 * h], v[8 * j + 2 * h + 1]);
          w[h] = *reinterpret_cast<uint32_t*>(&t);
        }
        dst[j] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else if (e.c_dtype == 0) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(e.C) + base);
#pragma unroll
      for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(e.C) + base);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          __half2 t = __floats2half2_rn(v[8 * j + 2 * h], v[8 * j + 2 * h + 1]);
          w[h] = *reinterpret_cast<uint32_t*>(&t);
        }
        dst[j] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j < e.N) store_one(e.C, e.c_dtype, base + j, v[j]);
  }
}

// 32 consecutive columns col0.. of one output row: bias, activation, cast, store.
template <bool kPacked = true>
__device__ __forceinline__ void epi_row32(const EpiArgs& e, int row, int col0, float (&v)[32]) {
  if (e.bias != nullptr || e.act != 0) epi_bias_act32<kPacked>(e, col0, v);
  epi_store_row32(e, row, col0, v);
}

// 32 codes of v / s, four per word.
template <class Div>
__device__ __forceinline__ void encode32(const Div& div, const float (&v)[32], uint32_t (&w)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float x[4] = {v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]};
    w[q] = pack4(div, x);
  }
}

// FP8 output: the 128 columns col0.. of one row form one 1x128 group, quantised as the
// group quantiser does (group_scale, correctly rounded x / s, RN satfinite E4M3), after
// bias and activation. g holds the group's 128 raw accumulators (registers); bias and
// activation are applied in place. Columns past N take no part in the amax and are not
// written; the codes leave as 16-byte stores (ldc and the code pointer are 16-byte
// aligned), the scale as one float at scales[(col0 / 128) * M + row].
__device__ __forceinline__ void epi_group_fp8_regs(const EpiArgs& e, int row, int col0, float (&g)[128]) {
  if (row >= e.M || col0 >= e.N) return;
  const bool full = col0 + 128 <= e.N;
  float amax = 0.0f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float (&v)[32] = *reinterpret_cast<float(*)[32]>(g + 32 * c);
    if (e.bias != nullptr || e.act != 0) epi_bias_act32(e, col0 + 32 * c, v);
    if (full) {
#pragma unroll
      for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + 32 * c + j < e.N) amax = fmaxf(amax, fabsf(v[j]));
    }
  }
  const float sc = group_scale(amax);
  uint8_t* dst = static_cast<uint8_t*>(e.C) + static_cast<long long>(row) * e.ldc + col0;
  const bool fast = markstein_ok(sc);
  const MarksteinDiv md = markstein_div(sc);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float (&v)[32] = *reinterpret_cast<const float(*)[32]>(g + 32 * c);
    uint32_t w[8];
    if (fast) encode32(md, v, w);
    else encode32(ExactDiv{sc}, v, w);
    if (full) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
      d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
      d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + 32 * c + j < e.N) dst[32 * c + j] = static_cast<uint8_t>(w[j >> 2] >> (8 * (j & 3)));
    }
  }
  e.scales[static_cast<long long>(col0 / 128) * e.M + row] = sc;
}

// FP8 output in two passes over a 1x128 group of one row, 32 columns at a time, so the
// code stays one loop body per pass (the group is not held in registers): pass 1 loads
// each raw chunk (load(c, v): c = 0..3), applies bias and activation, folds the chunk
// into the group's amax and hands it back (keep(c, v), e.g. a store to TMEM, which then
// serves the chunk to pass 2); pass 2 fetches the finished chunk again (again(c, v)),
// divides by the group scale and stores the codes. Same encoding as epi_group_fp8_regs.
template <class Load, class Keep, class Again>
__device__ __forceinline__ void epi_group_fp8_2pass(const EpiArgs& e, int row, int col0, Load load, Keep keep,
                                                    Again again) {
  const bool full = col0 + 128 <= e.N;
  float amax = 0.0f;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    float v[32];
    load(c, v);
    if (e.bias != nullptr || e.act != 0) epi_bias_act32(e, col0 + 32 * c, v);
    if (full) {
#pragma unroll
      for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + 32 * c + j < e.N) amax = fmaxf(amax, fabsf(v[j]));
    }
    keep(c, v);
  }
  const float sc = group_scale(amax);
  const bool fast = markstein_ok(sc);
  const MarksteinDiv md = markstein_div(sc);
  const bool live = row < e.M && col0 < e.N;
  uint8_t* dst = static_cast<uint8_t*>(e.C) + static_cast<long long>(row) * e.ldc + col0;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    float v[32];
    again(c, v);
    uint32_t w[8];
    if (fast) encode32(md, v, w);
    else encode32(ExactDiv{sc}, v, w);
    if (!live) continue;
    if (full) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
      d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
      d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + 32 * c + j < e.N) dst[32 * c + j] = static_cast<uint8_t>(w[j >> 2] >> (8 * (j & 3)));
    }
  }
  if (live) e.scales[static_cast<long long>(col0 / 128) * e.M + row] = sc;
}

// CNT consecutive output rows row0.. of one column (transposed accumulator tiles).
template <int CNT>
__device__ __forceinline__ void epi_col(const EpiArgs& e, int col, int row0, const float* v) {
  if (col >= e.N) return;
  const float b = e.bias != nullptr ? load_bias(e.bias, e.bias_dtype, col) : 0.0f;
  if (e.act != 0 && e.c_dtype == 0) {
    // FP32 output with an activation: in double, one element per iteration from w[0]
    // with the copy rotated after each (w stays in registers; see epi_bias_act32_f64).
    float w[CNT];
#pragma unroll
    for (int j = 0; j < CNT; ++j) w[j] = v[j];
#pragma unroll 1
    for (int j = 0; j < CNT; ++j) {
      const int row = row0 + j;
      if (row < e.M)
        static_cast<float*>(e.C)[static_cast<long long>(row) * e.ldc + col] =
            __double2float_rn(act_apply_f64(static_cast<double>(w[0]) + static_cast<double>(b), e.act));
#pragma unroll
      for (int k = 0; k + 1 < CNT; ++k) w[k] = w[k + 1];
    }
    return;
  }
  // Bias and activation over the whole column first, then one store loop per output
  // type: each branch is taken once per call, so the plain path is one straight run of
  // instructions. (With the activation and the type switch inlined per element, the
  // executed instructions sat between the skipped ones and a lone CTA's first pass over
  // them, cold in the instruction cache, took ~7 us for a 32 x 32 chunk pair.)
  float w[CNT];
#pragma unroll
  for (int j = 0; j < CNT; ++j) w[j] = v[j] + b;
  if (e.act == 1) {
#pragma unroll
    for (int j = 0; j < CNT; ++j) w[j] = act_apply(w[j], 1);
  } else if (e.act == 2) {
#pragma unroll
    for (int j = 0; j < CNT; ++j) w[j] = act_apply(w[j], 2);
  }
  const int rows = e.M - row0 < CNT ? e.M - row0 : CNT;
  const long long off = static_cast<long long>(row0) * e.ldc + col;
  if (e.c_dtype == 0) {
    float* c = static_cast<float*>(e.C) + off;
#pragma unroll
    for (int j = 0; j < CNT; ++j)
      if (j < rows) c[static_cast<long long>(j) * e.ldc] = w[j];
  } else if (e.c_dtype == 1) {
    __nv_bfloat16* c = static_cast<__nv_bfloat16*>(e.C) + off;
#pragma unroll
    for (int j = 0; j < CNT; ++j)
      if (j < rows) c[static_cast<long long>(j) * e.ldc] = __float2bfloat16_rn(w[j]);
  } else {
    __half* c = static_cast<__half*>(e.C) + off;
#pragma unroll
    for (int j = 0; j < CNT; ++j)
      if (j < rows) c[static_cast<long long>(j) * e.ldc] = __float2half_rn(w[j]);
  }
}

}  // namespace smg
