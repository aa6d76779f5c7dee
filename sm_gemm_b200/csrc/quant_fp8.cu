// FP32 -> FP8 E4M3 group quantiser (1x128 row groups for activations, 128x128 blocks
// for weights), the memory-bound producer of the operands of the block-scaled GEMM.
//
// Per group, following the DeepGEMM kernel-library walkthrough (zwxr.cn),
// section 2.4: amax = max|x| over the group's elements, scale s = amax / 448 (FP32,
// correctly rounded division; 1.0 for an all-zero group), code = E4M3(x / s) with a
// correctly rounded division and the hardware's round-to-nearest-even, saturating
// conversion (cvt.rn.satfinite.e4m3x2.f32). The result is bit-exact with a plain
// sequential implementation: the max is order-independent and every other step is
// a single correctly rounded operation (MarksteinDiv below gives the correctly
// rounded quotient at a few instructions per element).
//
// Both row-major group shapes are fed by TMA: a persistent CTA streams fp32 tiles
// through a shared-memory ring (one producer thread, eight encoding warps), so HBM
// sees a few hundred KB in flight per SM while the warps encode. Column-major 1x128
// input (rows contiguous) uses a plain per-thread kernel.
//
// Plus two small kernels: the K == 0 epilogue fill, and the bounded-wait self-test.
#include <cuda_fp8.h>

#include "epilogue.cuh"
#include "fp8_codec.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace smg {

namespace {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
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

// 16 codes of one lane's elements v[j][e] (group columns c0 + 32j + e) into dst (the
// code of column c0); bytewise with bounds when the group is ragged or cols % 4 != 0.
template <class Div>
__device__ __forceinline__ void store_codes16(const Div& div, const float (&v)[4][4], uint8_t* dst, long long c0,
                                              long long cols, bool vec) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w = pack4(div, v[j]);
    if (vec) {
      *reinterpret_cast<uint32_t*>(dst + 32 * j) = w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (c0 + 32 * j + e < cols) dst[32 * j + e] = static_cast<uint8_t>(w >> (8 * e));
    }
  }
}

// Pass 2 of quant_128x128_tma_kernel (see there) for block (kb, nb).
template <bool kNContig, class Div>
__device__ __forceinline__ void encode_block(const Div& div, const float* tile, int ptid, long long kb, long long nb,
                                             long long K, long long N, uint8_t* __restrict__ Q) {
  const long long k0 = kb * 128;
  if (kNContig) {
    const int n = ptid & 127, kh = (ptid >> 7) * 64;
    const long long ng = nb * 128 + n;
    if (ng >= N) return;
    uint8_t* dst = Q + ng * K + k0 + kh;
    const bool vec = (K & 15) == 0 && k0 + kh + 64 <= K;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t w[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int k = kh + 16 * u + 4 * h;
        const float x[4] = {tile[k * 128 + n], tile[(k + 1) * 128 + n], tile[(k + 2) * 128 + n],
                            tile[(k + 3) * 128 + n]};
        w[h] = pack4(div, x);
      }
      if (vec) {
        *reinterpret_cast<uint4*>(dst + 16 * u) = make_uint4(w[0], w[1], w[2], w[3]);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (k0 + kh + 16 * u + j < K) dst[16 * u + j] = static_cast<uint8_t>(w[j >> 2] >> (8 * (j & 3)));
      }
    }
  } else {
    const int warp = ptid >> 5, lane = ptid & 31;
    const long long kg = k0 + 4 * lane;
    const bool vec = (K & 3) == 0 && kg + 4 <= K;
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
      const int n = warp * 16 + i;
      const long long ng = nb * 128 + n;
      if (ng >= N) break;
      const float4 t4 = reinterpret_cast<const float4*>(tile + n * 128)[lane];
      const float x[4] = {t4.x, t4.y, t4.z, t4.w};
      const uint32_t w = pack4(div, x);
      uint8_t* dst = Q + ng * K + kg;
      if (vec) {
        *reinterpret_cast<uint32_t*>(dst) = w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (kg + e < K) dst[e] = static_cast<uint8_t>(w >> (8 * e));
      }
    }
  }
}

// ---------------------------------------------------------------- TMA-fed quantisers
//
// Shared structure: warp 8 is the producer (lane 0 issues one 2-D TMA load per tile into
// the next ring stage, completing on full[stage]); warps 0-7 read the stage, release it
// on empty[stage] (8 arrivals) and encode. All waits are bounded (abort flag + limit).
constexpr int kQConsumers = 8;
constexpr int kQThreads = (kQConsumers + 1) * 32;

struct QRing {
  uint32_t base;      // shared address of stage 0 (1024-byte aligned)
  const uint8_t* gen; // generic address of stage 0
  uint32_t bars;      // full[0..S), empty[0..S)
  volatile int* abort_flag;
};

template <int kStages, int kTileBytes>
__device__ __forceinline__ QRing q_ring_setup(uint8_t* smem_raw) {
  QRing q;
  q.base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  q.gen = smem_raw + (q.base - smem_u32(smem_raw));
  q.bars = q.base + kStages * kTileBytes;
  q.abort_flag = reinterpret_cast<volatile int*>(const_cast<uint8_t*>(q.gen) + kStages * kTileBytes + 16 * kStages);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(q.bars + 8u * i, 1);
      mbar_init(q.bars + 8u * (kStages + i), kQConsumers);
    }
    *q.abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Programmatic dependent launch: the next kernel on the stream may start its own set-up
  // now, and this one touches global memory only once the previous kernel has finished
  // (griddepcontrol.wait returns at once when there is none).
  pdl_launch_dependents();
  pdl_wait();
  return q;
}

// Producer loop: tile i of this CTA is tile blockIdx.x + i * gridDim.x; coords(t, x, y)
// gives its TMA box origin. After an abort it waits (bounded) for the loads in flight.
template <int kStages, int kTileBytes, class Coords>
__device__ __forceinline__ void q_produce(const QRing& q, const CUtensorMap* tm, long long T, Coords coords,
                                          unsigned long long limit) {
  tma_prefetch_desc(tm);
  int stage = 0;
  uint32_t phase = 0;
  long long issued = 0;
  for (long long t = blockIdx.x; t < T; t += gridDim.x) {
    if (!mbar_wait(q.bars + 8u * (kStages + stage), phase ^ 1u, q.abort_flag, limit)) break;
    int x, y;
    coords(t, x, y);
    mbar_arrive_expect_tx(q.bars + 8u * stage, kTileBytes);
    tma_load_2d(q.base + stage * kTileBytes, tm, q.bars + 8u * stage, x, y);
    ++issued;
    if (++stage == kStages) { stage = 0; phase ^= 1u; }
  }
  if (*q.abort_flag) {
    volatile int no_abort = 0;
    for (long long i = 0; i < issued && i < kStages; ++i) {
      if (--stage < 0) { stage = kStages - 1; phase ^= 1u; }
      mbar_wait(q.bars + 8u * stage, phase, &no_abort, limit);
    }
  }
}

// 1x128 groups of a row-major X[rows][cols]: one tile = 32 rows x 128 columns (16 KB, one
// group per row). Warp w encodes rows 4w..4w+3 of the tile, eight lanes per row: lane l
// reads the float4s at columns 32j + 4(l % 8), j < 4 (each quarter-warp reads 128
// contiguous bytes, free of bank conflicts), reduces the row's amax in three shuffle
// steps, releases the stage, then encodes and stores its 16 codes.
constexpr int kQ1Rows = 32;
constexpr int kQ1TileBytes = kQ1Rows * 128 * 4;
constexpr int kQ1Stages = 4;
constexpr int kQ1Smem = 1024 + kQ1Stages * kQ1TileBytes + 16 * kQ1Stages + 16;

__global__ void __launch_bounds__(kQThreads) quant_1x128_tma_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                     long long rows, long long cols,
                                                                     uint8_t* __restrict__ Q, float* __restrict__ S,
                                                                     unsigned long long limit) {
  extern __shared__ uint8_t smem_raw[];
  const QRing q = q_ring_setup<kQ1Stages, kQ1TileBytes>(smem_raw);
  const long long kbn = (cols + 127) / 128;
  const long long T = (rows + kQ1Rows - 1) / kQ1Rows * kbn;
  const int warp = static_cast<int>(warp_id()), lane = static_cast<int>(lane_id());
  if (warp == kQConsumers) {
    if (lane == 0)
      q_produce<kQ1Stages, kQ1TileBytes>(q, &tm_x, T, [&](long long t, int& x, int& y) {
        const long long rt = t / kbn;
        x = static_cast<int>((t - rt * kbn) * 128);
        y = static_cast<int>(rt * kQ1Rows);
      }, limit);
    return;
  }
  const int gi = lane >> 3, sub = lane & 7;
  const int trow = warp * 4 + gi;
  const bool vec_st = (cols & 3) == 0;
  // (row tile, group) of this CTA's current tile, advanced by gridDim.x tiles per step.
  long long rt = blockIdx.x / kbn, kb = blockIdx.x - (blockIdx.x / kbn) * kbn;
  const long long step_rt = gridDim.x / kbn, step_kb = gridDim.x - step_rt * kbn;
  int stage = 0;
  uint32_t phase = 0;
  bool dead = false;
  for (long long t = blockIdx.x; t < T; t += gridDim.x) {
    if (!dead) dead = !mbar_wait(q.bars + 8u * stage, phase, q.abort_flag, limit);
    dead = __any_sync(0xffffffffu, dead);
    float v[4][4];
    if (!dead) {
      const float* src = reinterpret_cast<const float*>(q.gen + stage * kQ1TileBytes) + trow * 128 + 4 * sub;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 t4 = *reinterpret_cast<const float4*>(src + 32 * j);
        v[j][0] = t4.x; v[j][1] = t4.y; v[j][2] = t4.z; v[j][3] = t4.w;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(q.bars + 8u * (kQ1Stages + stage));
    if (!dead) {
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(v[j][e]));
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const long long r = rt * kQ1Rows + trow;
      if (r < rows) {
        const float sc = group_scale(amax);
        const long long c0 = kb * 128 + 4 * sub;
        uint8_t* dst = Q + r * cols + c0;
        const bool vec = vec_st && kb * 128 + 128 <= cols;
        if (markstein_ok(sc)) store_codes16(markstein_div(sc), v, dst, c0, cols, vec);
        else store_codes16(ExactDiv{sc}, v, dst, c0, cols, vec);
        if (sub == 0) S[kb * rows + r] = sc;
      }
    }
    kb += step_kb;
    rt += step_rt;
    if (kb >= kbn) {
      kb -= kbn;
      ++rt;
    }
    if (++stage == kQ1Stages) { stage = 0; phase ^= 1u; }
  }
}

// 128x128 blocks of the weight X[K, N]; codes are written transposed, Q[n][k]. One tile
// = one block (64 KB), three stages, one CTA per SM. kNContig: X row-major (n
// contiguous), the stage holds T[k][n]; otherwise X column-major (k contiguous) and the
// stage holds T[n][k]. Pass 1: every consumer thread takes the amax of 64 elements (16
// float4 reads), the block's amax is reduced through shared memory (one named barrier).
// Pass 2 reads the stage again in the order the codes are stored:
//  - T[k][n]: thread (n = i % 128, kh = i / 128) walks 64 k of column n (a warp reads 32
//    consecutive n of one k row: no bank conflicts) and stores 4 x 16 codes;
//  - T[n][k]: warp w walks rows n = 16w..16w+15, lane l encodes k = 4l..4l+3 of each
//    (a warp reads one 512-byte row) and stores 4 codes.
constexpr int kQ2TileBytes = 128 * 128 * 4;
constexpr int kQ2Stages = 3;
constexpr int kQ2Smem = 1024 + kQ2Stages * kQ2TileBytes + 16 * kQ2Stages + 16 + 2 * kQConsumers * 4;

template <bool kNContig>
__global__ void __launch_bounds__(kQThreads, 1) quant_128x128_tma_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                          long long K, long long N,
                                                                          uint8_t* __restrict__ Q,
                                                                          float* __restrict__ S,
                                                                          unsigned long long limit) {
  extern __shared__ uint8_t smem_raw[];
  const QRing q = q_ring_setup<kQ2Stages, kQ2TileBytes>(smem_raw);
  float* red = reinterpret_cast<float*>(const_cast<uint8_t*>(q.gen) + kQ2Stages * kQ2TileBytes + 16 * kQ2Stages + 16);
  const long long kbn = (K + 127) / 128, nbn = (N + 127) / 128;
  const long long T = kbn * nbn;
  const int warp = static_cast<int>(warp_id()), lane = static_cast<int>(lane_id());
  if (warp == kQConsumers) {
    if (lane == 0)
      q_produce<kQ2Stages, kQ2TileBytes>(q, &tm_x, T, [&](long long t, int& x, int& y) {
        const long long kb = t / nbn, nb = t - kb * nbn;
        x = static_cast<int>((kNContig ? nb : kb) * 128);
        y = static_cast<int>((kNContig ? kb : nb) * 128);
      }, limit);
    return;
  }
  const int ptid = static_cast<int>(threadIdx.x);
  int stage = 0;
  uint32_t phase = 0;
  bool dead = false;
  uint32_t it = 0;
  for (long long t = blockIdx.x; t < T; t += gridDim.x, ++it) {
    if (!dead) dead = !mbar_wait(q.bars + 8u * stage, phase, q.abort_flag, limit);
    dead = __any_sync(0xffffffffu, dead);
    const float* tile = reinterpret_cast<const float*>(q.gen + stage * kQ2TileBytes);
    float amax = 0.0f;
    if (!dead) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float4 t4 = reinterpret_cast<const float4*>(tile)[i * 256 + ptid];
        amax = fmaxf(fmaxf(amax, fmaxf(fabsf(t4.x), fabsf(t4.y))), fmaxf(fabsf(t4.z), fabsf(t4.w)));
      }
    }
    amax = warp_max(amax);
    float* rb = red + (it & 1) * kQConsumers;
    if (lane == 0) rb[warp] = amax;
    named_barrier_sync(1, kQConsumers * 32);
    float m = rb[0];
#pragma unroll
    for (int w = 1; w < kQConsumers; ++w) m = fmaxf(m, rb[w]);
    const long long kb = t / nbn, nb = t - kb * nbn;
    const float sc = group_scale(m);
    if (!dead) {
      if (ptid == 0) S[kb * nbn + nb] = sc;
      if (markstein_ok(sc)) encode_block<kNContig>(markstein_div(sc), tile, ptid, kb, nb, K, N, Q);
      else encode_block<kNContig>(ExactDiv{sc}, tile, ptid, kb, nb, K, N, Q);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(q.bars + 8u * (kQ2Stages + stage));
    if (++stage == kQ2Stages) { stage = 0; phase ^= 1u; }
  }
}

__global__ void fill_epilogue_kernel(int M, int N, const void* bias, int bias_dtype, int act, void* C,
                                     int c_dtype, long long ldc) {
  const long long total = static_cast<long long>(M) * N;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / N, c = i - r * N;
    // act(bias) in double, rounded once to the output type.
    const double b = bias != nullptr ? static_cast<double>(load_bias(bias, bias_dtype, static_cast<int>(c))) : 0.0;
    const double y = act_apply_f64(b, act);
    const long long off = r * ldc + c;
    if (c_dtype == 0) static_cast<float*>(C)[off] = __double2float_rn(y);
    else if (c_dtype == 1) static_cast<__nv_bfloat16*>(C)[off] = __double2bfloat16(y);
    else static_cast<__half*>(C)[off] = __double2half(y);
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

namespace {
// Launch configuration with programmatic dependent launch (the quantisers call
// griddepcontrol.wait before touching global memory, so they may start early).
cudaLaunchConfig_t pdl_config(unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                              cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  add_pdl_attr(cfg, attr);
  return cfg;
}
}  // namespace

cudaError_t launch_quant_1x128_tma(const CUtensorMap& tm_x, long long rows, long long cols, uint8_t* Q, float* S,
                                   int sms, unsigned long long limit, cudaStream_t stream) {
  const cudaError_t attr = smem_opt_in<quant_1x128_tma_kernel>(kQ1Smem);
  if (attr != cudaSuccess) return attr;
  static int per_sm = 0;
  if (per_sm == 0 && cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_1x128_tma_kernel, kQThreads,
                                                                    kQ1Smem) != cudaSuccess) {
    cudaGetLastError();
    per_sm = 1;
  }
  const long long tiles = (rows + kQ1Rows - 1) / kQ1Rows * ((cols + 127) / 128);
  const long long cap = static_cast<long long>(per_sm > 0 ? per_sm : 1) * sms;
  const long long blocks = tiles < cap ? tiles : cap;
  cudaLaunchAttribute la[1];
  const cudaLaunchConfig_t cfg = pdl_config(static_cast<unsigned>(blocks), kQThreads, kQ1Smem, stream, la);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, quant_1x128_tma_kernel, tm_x, rows, cols, Q, S, limit);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_quant_1x128_cols(const float* X, long long rows, long long cols, long long ldx, uint8_t* Q,
                                    float* S, cudaStream_t stream) {
  const long long kbn = (cols + 127) / 128;
  dim3 grid(static_cast<unsigned>((rows + 255) / 256), static_cast<unsigned>(kbn));
  quant_1x128_cols_kernel<<<grid, 256, 0, stream>>>(X, rows, cols, ldx, Q, S);
  return cudaGetLastError();
}

cudaError_t launch_quant_128x128_tma(const CUtensorMap& tm_x, bool n_contig, long long K, long long N, uint8_t* Q,
                                     float* S, int sms, unsigned long long limit, cudaStream_t stream) {
  const long long tiles = ((K + 127) / 128) * ((N + 127) / 128);
  const unsigned blocks = static_cast<unsigned>(tiles < sms ? tiles : sms);
  cudaLaunchAttribute la[1];
  const cudaLaunchConfig_t cfg = pdl_config(blocks, kQThreads, kQ2Smem, stream, la);
  cudaError_t e;
  if (n_contig) {
    const cudaError_t attr = smem_opt_in<quant_128x128_tma_kernel<true>>(kQ2Smem);
    if (attr != cudaSuccess) return attr;
    e = cudaLaunchKernelEx(&cfg, quant_128x128_tma_kernel<true>, tm_x, K, N, Q, S, limit);
  } else {
    const cudaError_t attr = smem_opt_in<quant_128x128_tma_kernel<false>>(kQ2Smem);
    if (attr != cudaSuccess) return attr;
    e = cudaLaunchKernelEx(&cfg, quant_128x128_tma_kernel<false>, tm_x, K, N, Q, S, limit);
  }
  if (e != cudaSuccess) return e;
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
