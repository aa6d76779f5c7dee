// FP32 -> FP8 E4M3 group quantiser (1x128 row groups for activations, 128x128 blocks
// for weights), the memory-bound producer of the operands of the block-scaled GEMM.
//
// Per group, following the DeepGEMM kernel-library walkthrough (zwxr.cn),
// section 2.4: amax = max|x| over the group's elements, scale s = amax / 448 (FP32,
// correctly rounded division; 1.0 for an all-zero group), code = E4M3(x / s) with a
// correctly rounded division and the hardware's round-to-nearest-even, saturating
// conversion (cvt.rn.satfinite.e4m3x2.f32). The result is bit-exact with a plain
// sequential implementation: the max is order-independent and every other step is
// a single correctly rounded operation (GroupDivider below gives the correctly
// rounded quotient at a few instructions per element).
//
// Plus two small kernels: the K == 0 epilogue fill, and the bounded-wait self-test.
#include <cuda_fp8.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace smg {

namespace {

__device__ __forceinline__ float group_scale(float amax) {
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
}

// Correctly rounded x / s for every element of a group that shares the scale s.
// Markstein's FMA division (P. Markstein, "IA-64 and Elementary Functions", 2000,
// chapter 8; also Muller et al., "Handbook of Floating-Point Arithmetic", the
// section on division with an FMA): with r = RN(1/s), y = RN(x r) and the residual
// e = x - y s (exact in one FMA), RN(y + e r) is the correctly rounded quotient
// provided r is the correctly rounded reciprocal and the significand of s is not
// all ones. The residual is exact only while x - y s stays out of the subnormal
// range, which holds for every quotient E4M3 can tell from zero (|x/s| > 2^-11)
// once s >= 2^-90; smaller quotients become a signed zero code either way, and
// the sign survives every step. A group whose scale fails a condition (all-ones
// significand, s < 2^-90, s not finite) divides with __fdiv_rn instead
// (ExactDiv); the choice is made once per group, outside the element loops.
__device__ __forceinline__ bool markstein_ok(float s) {
  const uint32_t b = __float_as_uint(s);
  const uint32_t ex = (b >> 23) & 0xffu;
  return ex >= 127u - 90u && ex < 255u && (b & 0x7fffffu) != 0x7fffffu;
}

struct MarksteinDiv {
  float s, r;  // r = RN(1 / s)
  __device__ __forceinline__ float operator()(float x) const {
    const float y = __fmul_rn(x, r);
    const float e = __fmaf_rn(-y, s, x);
    return e == 0.0f ? y : __fmaf_rn(e, r, y);  // e == 0 keeps the sign of a zero x
  }
};

struct ExactDiv {
  float s;
  __device__ __forceinline__ float operator()(float x) const { return __fdiv_rn(x, s); }
};

__device__ __forceinline__ MarksteinDiv markstein_div(float s) { return MarksteinDiv{s, __frcp_rn(s)}; }

// Two codes packed little-endian: x0 -> low byte, x1 -> high byte.
__device__ __forceinline__ uint32_t e4m3x2(float x0, float x1) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3));
}

// Four codes of x[0..3] / s, little-endian in one word.
template <class Div>
__device__ __forceinline__ uint32_t pack4(const Div& div, const float (&x)[4]) {
  return e4m3x2(div(x[0]), div(x[1])) | (e4m3x2(div(x[2]), div(x[3])) << 16);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Row-major X (element (r, c) at r*ldx + c): each warp quantises kGroupsPerWarp
// consecutive 1x128 groups; every lane issues all of its 16-byte loads before using
// any, so enough bytes are in flight to keep HBM busy.
constexpr int kGroupsPerWarp = 4;
__global__ void __launch_bounds__(256) quant_1x128_rows_kernel(const float* __restrict__ X, long long rows,
                                                               long long cols, long long ldx,
                                                               uint8_t* __restrict__ Q, float* __restrict__ S) {
  const long long kbn = (cols + 127) / 128;
  const long long total = rows * kbn;
  const long long g0 = (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * kGroupsPerWarp;
  if (g0 >= total) return;
  const int lane = threadIdx.x & 31;
  const bool vec_ld = (ldx & 3) == 0;
  // (row, group) of each of the warp's groups: one division, then carries.
  long long gr[kGroupsPerWarp], gk[kGroupsPerWarp];
  gr[0] = g0 / kbn;
  gk[0] = g0 - gr[0] * kbn;
#pragma unroll
  for (int i = 1; i < kGroupsPerWarp; ++i) {
    gr[i] = gr[i - 1];
    gk[i] = gk[i - 1] + 1;
    if (gk[i] == kbn) {
      gk[i] = 0;
      ++gr[i];
    }
  }
  float v[kGroupsPerWarp][4];
#pragma unroll
  for (int i = 0; i < kGroupsPerWarp; ++i) {
    const bool live = g0 + i < total;
    const long long c0 = gk[i] * 128 + lane * 4;
    const float* src = X + gr[i] * ldx;
    if (live && vec_ld && gk[i] * 128 + 128 <= cols) {
      const float4 t = __ldcs(reinterpret_cast<const float4*>(src + c0));
      v[i][0] = t.x; v[i][1] = t.y; v[i][2] = t.z; v[i][3] = t.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[i][j] = (live && c0 + j < cols) ? src[c0 + j] : 0.0f;
    }
  }
#pragma unroll
  for (int i = 0; i < kGroupsPerWarp; ++i) {
    if (g0 + i >= total) break;
    const long long r = gr[i], kb = gk[i];
    const long long c0 = kb * 128 + lane * 4;
    float amax = fmaxf(fmaxf(fabsf(v[i][0]), fabsf(v[i][1])), fmaxf(fabsf(v[i][2]), fabsf(v[i][3])));
    amax = warp_max(amax);
    const float sc = group_scale(amax);
    const uint32_t w = markstein_ok(sc) ? pack4(markstein_div(sc), v[i]) : pack4(ExactDiv{sc}, v[i]);
    uint8_t* dst = Q + r * cols + c0;
    if (kb * 128 + 128 <= cols && (cols & 3) == 0) {
      *reinterpret_cast<uint32_t*>(dst) = w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (c0 + j < cols) dst[j] = static_cast<uint8_t>(w >> (8 * j));
    }
    if (lane == 0) S[kb * rows + r] = sc;
  }
}

// Codes of one row's group [c0, c1) of a column-major X, two columns at a time.
template <class Div>
__device__ __forceinline__ void quant_col_group(const Div& div, const float* __restrict__ X, long long ldx,
                                                long long r, long long c0, long long c1, uint8_t* dst) {
  for (long long c = c0; c < c1; c += 2) {
    const float x0 = X[c * ldx + r];
    const float x1 = (c + 1 < c1) ? X[(c + 1) * ldx + r] : 0.0f;
    const uint32_t w = e4m3x2(div(x0), div(x1));
    dst[c] = static_cast<uint8_t>(w);
    if (c + 1 < c1) dst[c + 1] = static_cast<uint8_t>(w >> 8);
  }
}

// One thread per (row, group) of a column-major X (element (r, c) at c*ldx + r):
// consecutive threads read consecutive rows, so every load of the warp is coalesced.
__global__ void __launch_bounds__(256) quant_1x128_cols_kernel(const float* __restrict__ X, long long rows,
                                                               long long cols, long long ldx,
                                                               uint8_t* __restrict__ Q, float* __restrict__ S) {
  const long long kbn = (cols + 127) / 128;
  const long long r = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long kb = blockIdx.y;
  if (r >= rows || kb >= kbn) return;
  const long long c0 = kb * 128;
  const long long c1 = (c0 + 128 < cols) ? c0 + 128 : cols;
  float amax = 0.0f;
  for (long long c = c0; c < c1; ++c) amax = fmaxf(amax, fabsf(X[c * ldx + r]));
  const float s = group_scale(amax);
  uint8_t* dst = Q + r * cols;
  if (markstein_ok(s)) quant_col_group(markstein_div(s), X, ldx, r, c0, c1, dst);
  else quant_col_group(ExactDiv{s}, X, ldx, r, c0, c1, dst);
  S[kb * rows + r] = s;
}

// One CTA per 128x128 block of the weight X[K, N] (element (k, n) at k*rs + n*cs).
// Phase 1 loads the block with 16-byte loads (16 per thread, all issued before use)
// and stages it transposed in shared memory as [n][k]; phase 2 has each thread encode
// 64 consecutive k of one n and write them as 16-byte rows of Q[n][k]. The shared tile
// is XOR-swizzled (column k of row n stored at k ^ g(n), g(n) = ((n >> 2) ^ ((n & 3) << 3)) & 31)
// so both the transposing stores of phase 1 and the row reads of phase 2 are free of
// bank conflicts.
__device__ __forceinline__ int qswz(int n) { return ((n >> 2) ^ ((n & 3) << 3)) & 31; }

// Phase 2 of quant_128x128_kernel: codes of k in [kh, kh + 64) of one staged row,
// written as four 16-byte chunks (bytewise for the last K-block when K % 16 != 0
// or the block is ragged; kvalid = the number of valid k from kh on).
template <class Div>
__device__ __forceinline__ void encode_half_row(const Div& div, const float* row, int g, int kh, uint8_t* dst,
                                                bool vec, int kvalid) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int kk = kh + u * 16 + h * 4;
      const float x[4] = {row[(kk + 0) ^ g], row[(kk + 1) ^ g], row[(kk + 2) ^ g], row[(kk + 3) ^ g]};
      w[h] = pack4(div, x);
    }
    if (vec) {
      *reinterpret_cast<uint4*>(dst + u * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (u * 16 + j < kvalid) dst[u * 16 + j] = static_cast<uint8_t>(w[j >> 2] >> (8 * (j & 3)));
    }
  }
}

__global__ void __launch_bounds__(256) quant_128x128_kernel(const float* __restrict__ X, long long K, long long N,
                                                            long long rs, long long cs, uint8_t* __restrict__ Q,
                                                            float* __restrict__ S) {
  extern __shared__ float tile[];  // [128 n][128 k], swizzled
  __shared__ float warp_amax[8];
  const long long kb = blockIdx.y, nb = blockIdx.x;
  const long long k0 = kb * 128, n0 = nb * 128;
  const long long nbn = (N + 127) / 128;
  const int t = threadIdx.x;
  float amax = 0.0f;
  if (cs == 1) {
    // N contiguous: float4 = 4 consecutive n of one k. idx -> (kk = idx / 32, n4 = idx % 32).
    const bool vec = (rs & 3) == 0 && n0 + 128 <= N;
    float4 r4[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int idx = i * 256 + t, kk = idx >> 5, n4 = idx & 31;
      const long long k = k0 + kk, n = n0 + 4 * n4;
      if (k < K && vec) {
        r4[i] = __ldcs(reinterpret_cast<const float4*>(X + k * rs + n));
      } else {
        float e[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) e[q] = (k < K && n + q < N) ? X[k * rs + n + q] : 0.0f;
        r4[i] = make_float4(e[0], e[1], e[2], e[3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int idx = i * 256 + t, kk = idx >> 5, n4 = idx & 31;
      const float e[4] = {r4[i].x, r4[i].y, r4[i].z, r4[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int n = 4 * n4 + q;
        amax = fmaxf(amax, fabsf(e[q]));
        tile[n * 128 + (kk ^ qswz(n))] = e[q];
      }
    }
  } else {
    // K contiguous (rs == 1) or general strides: float4 = 4 consecutive k of one n when
    // possible. idx -> (n = idx / 32, k4 = idx % 32).
    const bool vec = rs == 1 && (cs & 3) == 0 && k0 + 128 <= K;
    float4 r4[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int idx = i * 256 + t, nn = idx >> 5, k4 = idx & 31;
      const long long n = n0 + nn, k = k0 + 4 * k4;
      if (n < N && vec) {
        r4[i] = __ldcs(reinterpret_cast<const float4*>(X + n * cs + k));
      } else {
        float e[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) e[q] = (n < N && k + q < K) ? X[(k + q) * rs + n * cs] : 0.0f;
        r4[i] = make_float4(e[0], e[1], e[2], e[3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int idx = i * 256 + t, nn = idx >> 5, k4 = idx & 31;
      const float e[4] = {r4[i].x, r4[i].y, r4[i].z, r4[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        amax = fmaxf(amax, fabsf(e[q]));
        tile[nn * 128 + ((4 * k4 + q) ^ qswz(nn))] = e[q];
      }
    }
  }
  amax = warp_max(amax);
  if ((t & 31) == 0) warp_amax[t >> 5] = amax;
  __syncthreads();
  float m = warp_amax[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, warp_amax[w]);
  const float sc = group_scale(m);
  if (t == 0) S[kb * nbn + nb] = sc;

  // Phase 2: warp w, lane l -> row n = 32*(w & 3) + l, k in [64*(w >> 2), +64).
  const int nn = 32 * ((t >> 5) & 3) + (t & 31);
  const int kh = 64 * (t >> 7);
  const long long n = n0 + nn;
  if (n >= N) return;
  const float* row = tile + nn * 128;
  uint8_t* dst = Q + n * K + k0 + kh;
  const bool vec = (k0 + kh + 64 <= K) && ((K & 15) == 0);
  const int kvalid = static_cast<int>(K - k0 - kh);
  if (markstein_ok(sc)) encode_half_row(markstein_div(sc), row, qswz(nn), kh, dst, vec, kvalid);
  else encode_half_row(ExactDiv{sc}, row, qswz(nn), kh, dst, vec, kvalid);
}

__global__ void fill_epilogue_kernel(int M, int N, const void* bias, int bias_dtype, int act, void* C,
                                     int c_dtype, long long ldc) {
  const long long total = static_cast<long long>(M) * N;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / N, c = i - r * N;
    const float b = bias != nullptr ? load_bias(bias, bias_dtype, static_cast<int>(c)) : 0.0f;
    store_one(C, c_dtype, r * ldc + c, act_apply_precise(b, act));
  }
}

// Waits on an mbarrier that nothing arrives on; the bounded wait gives up after
// `limit_cycles` SM cycles, records kErrTimeout and the kernel returns normally.
__global__ void wait_selftest_kernel(unsigned long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_cycles);
  __syncthreads();
}

}  // namespace

cudaError_t launch_quant_1x128(const float* X, long long rows, long long cols, long long rs,
                               long long cs, uint8_t* Q, float* S, cudaStream_t stream) {
  const long long kbn = (cols + 127) / 128;
  if (cs == 1) {
    const long long groups = rows * kbn;
    const long long blocks = (groups + 8 * kGroupsPerWarp - 1) / (8 * kGroupsPerWarp);
    quant_1x128_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(X, rows, cols, rs, Q, S);
  } else {
    dim3 grid(static_cast<unsigned>((rows + 255) / 256), static_cast<unsigned>(kbn));
    quant_1x128_cols_kernel<<<grid, 256, 0, stream>>>(X, rows, cols, cs, Q, S);
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_128x128(const float* X, long long K, long long N, long long rs, long long cs,
                                 uint8_t* Q, float* S, cudaStream_t stream) {
  const int smem = 128 * 128 * static_cast<int>(sizeof(float));
  cudaError_t e = cudaFuncSetAttribute(quant_128x128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((N + 127) / 128), static_cast<unsigned>((K + 127) / 128));
  quant_128x128_kernel<<<grid, 256, smem, stream>>>(X, K, N, rs, cs, Q, S);
  return cudaGetLastError();
}

cudaError_t launch_fill_epilogue(int M, int N, const void* bias, int bias_dtype, int act, void* C,
                                 int c_dtype, long long ldc, cudaStream_t stream) {
  const long long total = static_cast<long long>(M) * N;
  const long long blocks = (total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096;
  fill_epilogue_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(M, N, bias, bias_dtype, act, C,
                                                                          c_dtype, ldc);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns * kCyclesPerNs);
  return cudaGetLastError();
}

unsigned take_error_word_misc() { return take_error_word(); }

}  // namespace smg
