// Row log-softmax of the LM-head logits, the second, light pass of the GEMM + bias +
// LogSoftmax fusion of "为什么我们要死磕GEMM" (kwkr.cn), section 7.2 (scheme B):
// out[m, n] = logit[m, n] - lse[m], lse[m] = log sum_n exp(logit[m, n]).
//
// The swap-AB GEMM epilogue already reduced every 128-column tile of a row to a pair
// (max, sum of exp(logit - max)); this pass merges a row's pairs with the online rule
//   (m1, s1) + (m2, s2) = (M, s1 e^(m1 - M) + s2 e^(m2 - M)),  M = max(m1, m2)
// (a pair with s = 0 is the identity), so the logits are read once more, only to
// subtract lse. Without partials (logits from the large-tile kernels) the same merge
// runs over the row's logits themselves. Reductions use a fixed order: results are
// deterministic run to run.
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace smg {

namespace {

struct MaxSum {
  float m, s;
};

// One exponential per merge: the pair with the larger max keeps its sum as it is.
__device__ __forceinline__ MaxSum merge(MaxSum a, MaxSum b) {
  if (a.s == 0.0f) return b;
  if (b.s == 0.0f) return a;
  if (a.m >= b.m) return {a.m, a.s + b.s * expf(b.m - a.m)};
  return {b.m, a.s * expf(a.m - b.m) + b.s};
}

__device__ __forceinline__ MaxSum warp_merge(MaxSum v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    MaxSum u{__shfl_xor_sync(0xffffffffu, v.m, o), __shfl_xor_sync(0xffffffffu, v.s, o)};
    v = merge(v, u);
  }
  return v;
}

// Block-wide merge (256 threads) in a fixed order: a butterfly within each warp, then
// one over the warps' results in warp 0. The result is returned to thread 0.
__device__ __forceinline__ MaxSum block_merge(MaxSum v, MaxSum* sh) {
  v = warp_merge(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sh[w] = v;
  __syncthreads();
  if (w == 0) {
    v = lane < static_cast<int>(blockDim.x >> 5) ? sh[lane] : MaxSum{-INFINITY, 0.0f};
    v = warp_merge(v);
  }
  return v;
}

// One CTA per row: lse[m] from the row's tile partials part[t * M + m], t < n_tiles.
__global__ void __launch_bounds__(256) lse_from_partials_kernel(const float2* __restrict__ part, int n_tiles, int M,
                                                                float* __restrict__ lse) {
  __shared__ MaxSum sh[8];
  const int m = blockIdx.x;
  MaxSum v{-INFINITY, 0.0f};
  for (int t = threadIdx.x; t < n_tiles; t += blockDim.x) {
    const float2 q = part[static_cast<size_t>(t) * M + m];
    v = merge(v, MaxSum{q.x, q.y});
  }
  v = block_merge(v, sh);
  if (threadIdx.x == 0) lse[m] = v.s > 0.0f ? v.m + logf(v.s) : -INFINITY;
}

// One CTA per row: lse[m] straight from the logits (online max and sum per thread).
__global__ void __launch_bounds__(256) lse_from_logits_kernel(const float* __restrict__ C, long long ldc, int N,
                                                              float* __restrict__ lse) {
  __shared__ MaxSum sh[8];
  const float* row = C + static_cast<long long>(blockIdx.x) * ldc;
  MaxSum v{-INFINITY, 0.0f};
  for (int n = threadIdx.x; n < N; n += blockDim.x) v = merge(v, MaxSum{row[n], 1.0f});
  v = block_merge(v, sh);
  if (threadIdx.x == 0) lse[blockIdx.x] = v.s > 0.0f ? v.m + logf(v.s) : -INFINITY;
}

// C[m, n] -= lse[m] over the whole matrix (grid-stride; float4 when rows are 16-byte
// aligned and N is a multiple of 4).
__global__ void __launch_bounds__(256) subtract_lse_kernel(float* __restrict__ C, long long ldc, int M, int N,
                                                           const float* __restrict__ lse) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if ((N & 3) == 0 && (ldc & 3) == 0) {
    const int n4 = N >> 2;
    const long long total = static_cast<long long>(M) * n4;
    for (long long i = tid; i < total; i += stride) {
      const long long m = i / n4, c = i - m * n4;
      float4* p = reinterpret_cast<float4*>(C + m * ldc) + c;
      const float l = lse[m];
      float4 x = *p;
      x.x -= l; x.y -= l; x.z -= l; x.w -= l;
      *p = x;
    }
  } else {
    const long long total = static_cast<long long>(M) * N;
    for (long long i = tid; i < total; i += stride) {
      const long long m = i / N, n = i - m * N;
      C[m * ldc + n] -= lse[m];
    }
  }
}

// One warp per (128-column tile t, row m) of an FP32 logit matrix: the tile's max logit and
// sum of exp(logit - max), written to part[t * M + m] as on the swap-AB GEMM's epilogue
// (columns past N contribute nothing; a tile with none gives the identity (-inf, 0)).
__global__ void __launch_bounds__(256) lse_tile_partials_kernel(const float* __restrict__ C, long long ldc, int M,
                                                                int N, int n_tiles, float2* __restrict__ part) {
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<long long>(M) * n_tiles) return;
  const int t = static_cast<int>(w / M), m = static_cast<int>(w - static_cast<long long>(t) * M);
  const float* row = C + static_cast<long long>(m) * ldc;
  MaxSum v{-INFINITY, 0.0f};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int n = t * 128 + 32 * j + lane;
    if (n < N) v = merge(v, MaxSum{row[n], 1.0f});
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    MaxSum u{__shfl_xor_sync(0xffffffffu, v.m, o), __shfl_xor_sync(0xffffffffu, v.s, o)};
    v = merge(v, u);
  }
  if (lane == 0) part[static_cast<long long>(t) * M + m] = v.s > 0.0f ? make_float2(v.m, v.s) : make_float2(-INFINITY, 0.0f);
}

__device__ __forceinline__ void st_cluster_f2(uint32_t addr, float a, float b) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ float2 ld_cluster_f2(uint32_t addr) {
  float2 r;
  asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(r.x), "=f"(r.y) : "r"(addr) : "memory");
  return r;
}

// Merge and subtract in one launch: CTA (x, m) subtracts row m's lse from columns
// [x chunk, (x + 1) chunk) of the row. The lse comes from the row's partials: with CS = 1
// every CTA merges all of them; with clusters of CS CTAs along x, CTA rank r merges the
// r-th of CS equal shares, writes its result to CTA 0's shared memory, and after a cluster
// barrier every CTA merges the CS results in rank order (the partials, read with a stride
// of M pairs, then cross from L2 once per cluster instead of once per CTA). Either way
// every CTA of a row takes the same steps in the same order, so all get the same lse bit
// for bit (CTA 0 stores it). Each thread issues the loads of its first four float4 of the
// chunk before the merge, so their latency overlaps it, and loads its partials four at a
// time.
template <int CS>
__global__ void __launch_bounds__(256) lse_merge_subtract_kernel(const float2* __restrict__ part, int n_parts,
                                                                 int M, float* __restrict__ C, long long ldc, int N,
                                                                 int chunk, float* __restrict__ lse) {
  __shared__ MaxSum sh[8];
  __shared__ float2 shares[CS];  // read in CTA 0 only (cluster ranks' merged shares)
  __shared__ float l_sh;
  pdl_launch_dependents();
  pdl_wait();
  const int m = blockIdx.y;
  const int bd = static_cast<int>(blockDim.x);
  float* row = C + static_cast<long long>(m) * ldc;
  const int c0 = blockIdx.x * chunk;
  const int c1 = c0 + chunk < N ? c0 + chunk : N;
  const bool vec = (ldc & 3) == 0 && (N & 3) == 0;
  float4* r4 = reinterpret_cast<float4*>(row);
  const int q0 = (c0 >> 2) + static_cast<int>(threadIdx.x), q1 = c1 >> 2;
  float4 x[4];
  if (vec) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (q0 + u * bd < q1) x[u] = r4[q0 + u * bd];
  }
  const int rank = CS > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int per = (n_parts + CS - 1) / CS;
  const int p0 = rank * per, p1 = p0 + per < n_parts ? p0 + per : n_parts;
  // Partials p0 + threadIdx.x, + blockDim.x, ... merged in that order (identity pairs
  // past p1 change nothing).
  MaxSum v{-INFINITY, 0.0f};
  for (int t0 = p0 + static_cast<int>(threadIdx.x); t0 < p1; t0 += 4 * bd) {
    float2 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = t0 + u * bd;
      q[u] = t < p1 ? part[static_cast<size_t>(t) * M + m] : make_float2(-INFINITY, 0.0f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) v = merge(v, MaxSum{q[u].x, q[u].y});
  }
  v = block_merge(v, sh);
  if constexpr (CS > 1) {
    if (threadIdx.x == 0) st_cluster_f2(mapa_shared(smem_u32(&shares[rank]), 0), v.m, v.s);
    cluster_sync();
    if (threadIdx.x == 0) {
      v = MaxSum{-INFINITY, 0.0f};
#pragma unroll
      for (int i = 0; i < CS; ++i) {
        const float2 q = ld_cluster_f2(mapa_shared(smem_u32(&shares[i]), 0));
        v = merge(v, MaxSum{q.x, q.y});
      }
    }
  }
  if (threadIdx.x == 0) {
    const float l = v.s > 0.0f ? v.m + logf(v.s) : -INFINITY;
    l_sh = l;
    if (blockIdx.x == 0) lse[m] = l;
  }
  __syncthreads();
  const float l = l_sh;
  if (vec) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int q = q0 + u * bd;
      if (q < q1) {
        x[u].x -= l; x[u].y -= l; x[u].z -= l; x[u].w -= l;
        r4[q] = x[u];
      }
    }
    for (int q = q0 + 4 * bd; q < q1; q += bd) {
      float4 y = r4[q];
      y.x -= l; y.y -= l; y.z -= l; y.w -= l;
      r4[q] = y;
    }
  } else {
    for (int n = c0 + static_cast<int>(threadIdx.x); n < c1; n += bd) row[n] -= l;
  }
  // CTA 0's shares stay in place until every CTA of the cluster has read them.
  if constexpr (CS > 1) cluster_sync();
}

}  // namespace

cudaError_t launch_lse_tile_partials(const float* C, long long ldc, int M, int N, float2* part, cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  const int n_tiles = (N + 127) / 128;
  const long long warps = static_cast<long long>(M) * n_tiles;
  lse_tile_partials_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, stream>>>(C, ldc, M, N, n_tiles, part);
  return cudaGetLastError();
}

cudaError_t launch_log_softmax_rows(float* C, long long ldc, int M, int N, const float2* part, int n_tiles,
                                    float* lse, int sms, cudaStream_t stream) {
  if (M <= 0 || (part == nullptr && N <= 0)) return cudaSuccess;
  if (part != nullptr && N > 0 && M <= 65535) {
    // One launch: about four CTAs per SM over the rows' column chunks (multiples of 1024).
    // With at least kCs chunks per row, the chunks of a row run in clusters of kCs CTAs
    // that share the merge (the grid's x rounded up to whole clusters; the extra CTAs
    // merge and subtract nothing).
    constexpr int kCs = 8;
    const long long ctas_per_row = (4LL * (sms > 0 ? sms : 1) + M - 1) / M;
    long long chunk = (static_cast<long long>(N) + ctas_per_row - 1) / ctas_per_row;
    chunk = (chunk + 1023) / 1024 * 1024;
    unsigned gx = static_cast<unsigned>((N + chunk - 1) / chunk);
    const bool clustered = gx >= static_cast<unsigned>(kCs);
    if (clustered) gx = (gx + kCs - 1) / kCs * kCs;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(gx, static_cast<unsigned>(M), 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    if (clustered) {
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = kCs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
    }
    add_pdl_attr(cfg, attr);
    const cudaError_t e =
        clustered ? cudaLaunchKernelEx(&cfg, lse_merge_subtract_kernel<kCs>, part, n_tiles, M, C, ldc, N,
                                       static_cast<int>(chunk), lse)
                  : cudaLaunchKernelEx(&cfg, lse_merge_subtract_kernel<1>, part, n_tiles, M, C, ldc, N,
                                       static_cast<int>(chunk), lse);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if (part != nullptr) lse_from_partials_kernel<<<M, 256, 0, stream>>>(part, n_tiles, M, lse);
  else lse_from_logits_kernel<<<M, 256, 0, stream>>>(C, ldc, N, lse);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || N <= 0) return e;
  const long long work = static_cast<long long>(M) * N / 4;
  const long long want = (work + 255) / 256;
  const long long cap = 4LL * (sms > 0 ? sms : 1);
  subtract_lse_kernel<<<static_cast<unsigned>(want < cap ? (want > 0 ? want : 1) : cap), 256, 0, stream>>>(C, ldc, M,
                                                                                                         N, lse);
  return cudaGetLastError();
}

}  // namespace smg
