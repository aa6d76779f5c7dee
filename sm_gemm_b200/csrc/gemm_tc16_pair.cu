// Large-tile 16-bit GEMM on CTA pairs (tcgen05.mma.cta_group::2): one 256 x 256 output
// tile per pair of SMs, FP32 accumulators in both SMs' TMEM, fused epilogue.
//
// Against the one-SM 128 x 256 kernel (gemm_tc16.cu) each SM now stages only its own
// 128 rows of A and its own 128 columns of B per K-block (32 KB instead of 48 KB for the
// same 128 x 256 share of the output), which halves the B traffic from L2 per FLOP and
// leaves room for 6 pipeline stages. The pipeline is still the copy-ahead-of-the-math
// scheme of the DeepGEMM kernel-library walkthrough (zwxr.cn), section 2.3; the fused
// epilogue is its section 5.1.
//
// Roles (256 threads per CTA, both CTAs of the cluster):
//  warp 0   TMA producer: loads this CTA's A rows and B columns; the byte count of
//           both CTAs' copies completes on the rank-0 CTA's "full" barrier.
//  warp 1   MMA issuer (rank 0 only): 4 x K=16 MMAs of 256 x 256 per stage; commits
//           free the stage in both CTAs and signal both CTAs' accumulators.
//  Both run their loops on the whole warp, so descriptors and coordinates stay in
//  warp-uniform registers, and one elected lane issues.
//  warp 2   TMEM allocator (cta_group::2, 512 columns = two 256-column accumulators).
//  warps 4-11 epilogue: each CTA drains its own 128 rows; warp w reads TMEM lanes
//           32*(w%4).. and the 128 columns 128*((w-4)/4).. of the tile, so two warps on
//           each SM sub-partition share the work and the epilogue of the CTA's last
//           tile (which nothing overlaps) takes half as long as with one. They release
//           the accumulator to the rank-0 MMA issuer with a cluster-scope arrive.
// Stream-K partial tiles are kept per (cluster, slot, rank) and reduced per rank.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstring>

#include "epilogue.cuh"
#include "kernels.h"
#include "operands.cuh"
#include "sm100.cuh"

namespace smg {

namespace {
constexpr int kEpiWarp0 = 4;
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 32 * kEpiWarp0 + kEpiThreads;
constexpr int kEpiCols = 128;  // tile columns per epilogue warp
constexpr int kTileN = 256;  // columns of the pair tile (128 per CTA for B, all 256 in each TMEM)
constexpr int kTcols = 512;
}  // namespace

// Output modes of the epilogue (separate instantiations, so each keeps its own code and
// registers): kOutDirect - 16/32-bit C written from registers with 16-byte stores;
// kOutFp8 - E4M3 codes + 1x128 scales (c_dtype E4M3); kOutTma - 16/32-bit C staged in
// shared memory (one swizzled 32 x 32 box per epilogue warp and chunk) and written by a
// TMA tile store through tm_c, the registers -> shared -> global write-back of the
// Tensor-Core page ("Chunk处理完毕").
constexpr int kOutDirect = 0, kOutFp8 = 1, kOutTma = 2;
constexpr int kStageWarpBytes = 4096;  // TMA-store staging per epilogue warp (2 x bf16/f16 box or 1 x f32 box)

// Bias, activation and cast of one 32 x 32 chunk (lane = row, v = its 32 columns), written
// to this warp's staging buffer in the layout of a TMA box {32 columns, 32 rows} with the
// map's swizzle (16-bit C: 64-byte rows, 64-byte swizzle; FP32 C: 128-byte rows, 128-byte
// swizzle: the 16-byte chunk j of row r sits at j ^ ((r >> 1) & 3), resp. j ^ (r & 7),
// so the 32 lanes' stores hit different banks), then one lane stores the box. 16-bit
// chunks alternate between two 2 KB halves of the buffer, FP32 chunks use all 4 KB; a
// half is rewritten only once the store that read it has finished reading.
__device__ __forceinline__ void stage_and_store32(const EpiArgs& e, const CUtensorMap* tm_c, uint32_t buf, int c,
                                                  uint32_t lane, int row0, int col0, float (&v)[32]) {
  if (e.bias != nullptr || e.act != 0) epi_bias_act32(e, col0, v);
  const bool f32 = e.c_dtype == 0;
  const uint32_t dst = f32 ? buf : buf + (c & 1) * 2048;
  if (lane == 0) {
    if (f32) bulk_wait_group_read<0>();
    else bulk_wait_group_read<1>();
  }
  __syncwarp();
  const uint32_t r = lane;
  if (f32) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t a = dst + r * 128 + 16 * (j ^ (r & 7));
      asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v[4 * j]), "f"(v[4 * j + 1]),
                   "f"(v[4 * j + 2]), "f"(v[4 * j + 3])
                   : "memory");
    }
  } else {
    const bool bf = e.c_dtype == 1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t w[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float x0 = v[8 * j + 2 * h], x1 = v[8 * j + 2 * h + 1];
        if (bf) {
          __nv_bfloat162 t = __floats2bfloat162_rn(x0, x1);
          w[h] = *reinterpret_cast<uint32_t*>(&t);
        } else {
          __half2 t = __floats2half2_rn(x0, x1);
          w[h] = *reinterpret_cast<uint32_t*>(&t);
        }
      }
      const uint32_t a = dst + r * 64 + 16 * (j ^ ((r >> 1) & 3));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                   : "memory");
    }
  }
  fence_proxy_async_shared();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tm_c, dst, col0, row0);
    bulk_commit_group();
  }
}

template <int BK, int STAGES, int OUT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc16_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_c, const Tc16Params p) {
  constexpr bool FP8OUT = OUT == kOutFp8;
  constexpr int A_BYTES = 128 * BK * 2;
  constexpr int B_BYTES = 128 * BK * 2;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr int KSTEPS = BK / 16;
  constexpr int STAGING = OUT == kOutTma ? kEpiWarps * kStageWarpBytes : 0;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem_base - smem_u32(smem_raw));
  const uint32_t staging = smem_base + STAGES * STAGE_BYTES;  // 1024-byte aligned
  const uint32_t bar_base = smem_base + STAGES * STAGE_BYTES + STAGING;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 4);
  uint8_t* misc = smem_gen + STAGES * STAGE_BYTES + STAGING + 8 * (2 * STAGES + 5);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* reduce_flag = reinterpret_cast<volatile int*>(misc + 8);

  const uint32_t warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kEpiWarps);  // every epilogue warp of both CTAs
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (OUT == kOutTma) tma_prefetch_desc(&tm_c);
  }
  if (warp == 2) {
    tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), kTcols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or copy targets them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();
  const TileSched& s = p.s;
  const uint64_t limit = p.wait_limit_cycles;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // The whole warp runs the loop (its addresses stay warp-uniform); one elected lane
    // issues the copies.
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    WorkIter it;
    it.init(s, cluster);
    Seg seg;
    bool ok = true;
    while (ok && it.next(s, seg)) {
      int mt, nt;
      tile_coords(s, seg.tile, mt, nt);
      const int a_row = mt * 256 + static_cast<int>(rank) * 128;
      const int b_row = nt * kTileN + static_cast<int>(rank) * 128;
      for (int kb = seg.kb0; kb < seg.kb1; ++kb) {
        const bool w = mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, limit);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint32_t leader_full = mapa_shared(full_bar(stage), 0);
        if (elect_one()) {
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          load_operand_pair<128, BK>(sa, &tm_a, leader_full, p.a_mn_major, a_row, kb * BK);
          load_operand_pair<128, BK>(sa + A_BYTES, &tm_b, leader_full, p.b_mn_major, b_row, kb * BK);
        }
        __syncwarp();
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok && rank == 0 && lane == 0) {
      // Wait (bounded, independent of the abort flag) for copies still in flight.
      int st = stage;
      uint32_t ph = phase;
      volatile int no_abort = 0;
      for (long long i = 0; i < issued && i < STAGES; ++i) {
        if (--st < 0) { st = STAGES - 1; ph ^= 1u; }
        mbar_wait(full_bar(st), ph, &no_abort, limit);
      }
    }
  } else if (warp == 1 && rank == 0) {
    // ---------------------------------------------------------------- MMA issuer
    // Warp-wide loop, one elected lane issues (always the same lane, so its commits
    // cover every MMA it issued).
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    WorkIter it;
    it.init(s, cluster);
    Seg seg;
    bool ok = true;
    while (ok && it.next(s, seg)) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, limit))) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * kTileN;
      for (int kb = seg.kb0; kb < seg.kb1; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(full_bar(stage), phase, abort_flag, limit))) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint32_t sb = sa + A_BYTES;
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < KSTEPS; ++k) {
            umma_f16_pair(d_tmem, operand_desc<128, BK>(sa, p.a_mn_major, k),
                          operand_desc<128, BK>(sb, p.b_mn_major, k), p.idesc, (kb > seg.kb0 || k > 0) ? 1u : 0u);
          }
          umma_commit_pair(empty_bar(stage), 0x3);
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (elect_one()) umma_commit_pair(tfull_bar(acc), 0x3);
      __syncwarp();
      ++local;
    }
    if (elect_one()) umma_commit_pair(drain_bar, 0x1);
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(drain_bar, 0, &no_abort, limit);
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int cq = (warp - kEpiWarp0) >> 2;  // which 128-column half of the tile
    const int r_local = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const int epi_tid = threadIdx.x - kEpiWarp0 * 32;
    const int c_base = cq * kEpiCols;        // first tile column of this warp
    constexpr int SLOT = 128 * kTileN;
    // TMEM chunk c (32 columns) of this warp's accumulator columns, as floats; and back.
    auto tmem_chunk = [&](uint32_t tacc, int c, float (&v)[32]) {
      uint32_t r[32];
      tmem_ld_32x32b_x32_sync(tacc + c * 32, r);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
    };
    auto tmem_keep = [&](uint32_t tacc, int c, const float (&v)[32]) {
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(v[j]);
      tmem_st_32x32b_x32(tacc + c * 32, r);
    };
    // This warp is done with accumulator buffer b (its TMEM reads and writes included).
    auto release_acc = [&](int b) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(b), 0));
    };
    int local = 0;
    WorkIter it;
    it.init(s, cluster);
    Seg seg;
    bool dead = false;
    while (it.next(s, seg)) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!dead) dead = !mbar_wait(tfull_bar(acc), acc_phase, abort_flag, limit);
      dead = __any_sync(0xffffffffu, dead);
      int mt, nt;
      tile_coords(s, seg.tile, mt, nt);
      const int row = mt * 256 + static_cast<int>(rank) * 128 + r_local;
      const uint32_t tacc = tmem_base + lane_addr + acc * kTileN + c_base;
      const int col0 = nt * kTileN + c_base;
      const bool whole = (seg.kb0 == 0 && seg.kb1 == s.kb_total);
      float* my_slot = p.slots + ((static_cast<size_t>(cluster) * 2 + seg.slot) * 2 + rank) * SLOT;
      if (!dead) {
        tc_fence_after();
        if constexpr (FP8OUT) {
          if (whole) {
            // This warp's 128 columns are one 1x128 group of each row: two passes over
            // TMEM, the activated values written back in place between them.
            epi_group_fp8_2pass(p.e, row, col0, [&](int c, float (&v)[32]) { tmem_chunk(tacc, c, v); },
                                [&](int c, const float (&v)[32]) { tmem_keep(tacc, c, v); },
                                [&](int c, float (&v)[32]) {
                                  if (c == 0) tmem_st_wait();  // pass 1's stores have landed
                                  tmem_chunk(tacc, c, v);
                                });
          } else {
#pragma unroll 1
            for (int c = 0; c < kEpiCols / 32; ++c) {
              float v[32];
              tmem_chunk(tacc, c, v);
              slot_store<32>(my_slot, r_local, c_base + c * 32, v);
            }
          }
        } else {
#pragma unroll 1
          for (int c = 0; c < kEpiCols / 32; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tacc + c * 32, r);
            tmem_ld_wait();
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            if (whole) {
              if constexpr (OUT == kOutTma) {
                stage_and_store32(p.e, &tm_c, staging + (warp - kEpiWarp0) * kStageWarpBytes, c, lane,
                                  mt * 256 + static_cast<int>(rank) * 128 + q * 32, col0 + c * 32, v);
              } else {
                epi_row32(p.e, row, col0 + c * 32, v);
              }
            } else {
              slot_store<32>(my_slot, r_local, c_base + c * 32, v);
            }
          }
        }
        // A stream-K piece with FP8 output keeps its accumulator buffer through the fix-up
        // below (see there); every other tile releases it now.
        if (whole || !FP8OUT) release_acc(acc);
      }

      if (!whole) {
        // Stream-K tile: the last contributor to arrive sums the partials in K order and
        // runs the epilogue. The fix-up's L2 traffic is slow while the other SMs stream
        // operands, so a 16/32-bit output frees the accumulator first (the next tile's
        // MMAs proceed meanwhile) and reads every partial from the slots. The FP8-output
        // epilogue needs the finished values twice (group amax, then the codes): its
        // pieces keep the buffer, and the reducer adds its own partial from TMEM and
        // keeps pass 1's activated values there, instead of summing the slots twice.
        const long long t_sk = seg.tile - s.dp_tiles;
        __threadfence();
        named_barrier_sync(1, kEpiThreads);
        if (epi_tid == 0) {
          const int c_lo = sk_owner(s, t_sk * s.kb_total);
          const int c_hi = sk_owner(s, (t_sk + 1) * s.kb_total - 1);
          int n = 0;
          for (int c = c_lo; c <= c_hi; ++c) n += sk_bound(s, c) < sk_bound(s, c + 1);
          const bool any_dead = *abort_flag != 0;
          const int old = any_dead ? -1 : counter_arrive(p.counters + t_sk * 2 + rank, p.gen, n);
          *reduce_flag = (!any_dead && old == n - 1);
        }
        named_barrier_sync(1, kEpiThreads);
        if (*reduce_flag) {
          __threadfence();
          if constexpr (FP8OUT) {
            // Pass 1 sums the partials in K order (this CTA's own from TMEM) and keeps
            // the activated values in TMEM for pass 2.
            auto reduce32 = [&](int c, float (&v)[32]) {
              sk_tile_sum<32>(
                  s, t_sk, cluster,
                  [&](int cc) {
                    return p.slots + ((static_cast<size_t>(cc) * 2 + sk_slot_of(s, cc, t_sk)) * 2 + rank) * SLOT;
                  },
                  [&](float* acc_v) {
                    float o[32];
                    tmem_chunk(tacc, c, o);
#pragma unroll
                    for (int j = 0; j < 32; ++j) acc_v[j] += o[j];
                  },
                  r_local, c_base + c * 32, v);
            };
            epi_group_fp8_2pass(p.e, row, col0, reduce32, [&](int c, const float (&v)[32]) { tmem_keep(tacc, c, v); },
                                [&](int c, float (&v)[32]) {
                                  if (c == 0) tmem_st_wait();
                                  tmem_chunk(tacc, c, v);
                                });
          } else {
            const int c_lo = sk_owner(s, t_sk * s.kb_total);
            const int c_hi = sk_owner(s, (t_sk + 1) * s.kb_total - 1);
#pragma unroll 1
            for (int c = 0; c < kEpiCols / 32; ++c) {
              float v[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = 0.0f;
              // Sum of every contributor's partial (CTA order = K order).
#pragma unroll 1
              for (int cc = c_lo; cc <= c_hi; ++cc) {
                if (!(sk_bound(s, cc) < sk_bound(s, cc + 1))) continue;
                const float* src = p.slots + ((static_cast<size_t>(cc) * 2 + sk_slot_of(s, cc, t_sk)) * 2 + rank) * SLOT;
                slot_accumulate<32>(src, r_local, c_base + c * 32, v);
              }
              epi_row32(p.e, row, col0 + c * 32, v);
            }
          }
        }
        if (FP8OUT && !dead) release_acc(acc);
        named_barrier_sync(1, kEpiThreads);
      }
      ++local;
    }
    if (OUT == kOutTma && lane == 0) bulk_wait_group<0>();  // this warp's tile stores have landed
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer stays resident until the rank-0 MMA issuer has drained
  tc_fence_after();
  if (warp == 2) tmem_dealloc_pair(tmem_base, kTcols);
}

namespace {
constexpr int kPairBK = 64, kPairStages = 6;
template <int OUT>
constexpr int pair_smem() {
  return 1024 + kPairStages * (2 * 128 * kPairBK * 2) + (OUT == kOutTma ? kEpiWarps * kStageWarpBytes : 0) +
         8 * (2 * kPairStages + 5) + 16;
}
static_assert(pair_smem<kOutTma>() <= 232448, "shared memory budget");

template <int OUT>
cudaError_t prepare_pair_kernel() {
  return smem_opt_in<gemm_tc16_pair_kernel<kPairBK, kPairStages, OUT>>(pair_smem<OUT>());
}

template <int OUT>
cudaLaunchConfig_t pair_config(int clusters, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = pair_smem<OUT>();
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}
}  // namespace

namespace {
template <int OUT>
int max_clusters_of() {
  if (prepare_pair_kernel<OUT>() != cudaSuccess) return 0;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pair_config<OUT>(1, nullptr, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tc16_pair_kernel<kPairBK, kPairStages, OUT>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n;
}
}  // namespace

int tc16_pair_max_clusters() {
  static int cached = -1;
  if (cached >= 0) return cached;
  const int a = max_clusters_of<kOutDirect>(), b = max_clusters_of<kOutFp8>(), c = max_clusters_of<kOutTma>();
  cached = a < b ? (a < c ? a : c) : (b < c ? b : c);
  return cached;
}

cudaError_t launch_gemm_tc16_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap* tm_c,
                                  const Tc16Params& p, int clusters, cudaStream_t stream) {
  const int out = p.e.c_dtype == kE4M3 ? kOutFp8 : (tm_c != nullptr ? kOutTma : kOutDirect);
  cudaError_t e = out == kOutFp8 ? prepare_pair_kernel<kOutFp8>()
                                 : (out == kOutTma ? prepare_pair_kernel<kOutTma>() : prepare_pair_kernel<kOutDirect>());
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  CUtensorMap none;
  std::memset(&none, 0, sizeof(none));
  const CUtensorMap& mc = tm_c != nullptr ? *tm_c : none;
  if (out == kOutFp8) {
    cudaLaunchConfig_t cfg = pair_config<kOutFp8>(clusters, stream, attr);
    add_pdl_attr(cfg, attr);
    e = cudaLaunchKernelEx(&cfg, gemm_tc16_pair_kernel<kPairBK, kPairStages, kOutFp8>, tm_a, tm_b, mc, p);
  } else if (out == kOutTma) {
    cudaLaunchConfig_t cfg = pair_config<kOutTma>(clusters, stream, attr);
    add_pdl_attr(cfg, attr);
    e = cudaLaunchKernelEx(&cfg, gemm_tc16_pair_kernel<kPairBK, kPairStages, kOutTma>, tm_a, tm_b, mc, p);
  } else {
    cudaLaunchConfig_t cfg = pair_config<kOutDirect>(clusters, stream, attr);
    add_pdl_attr(cfg, attr);
    e = cudaLaunchKernelEx(&cfg, gemm_tc16_pair_kernel<kPairBK, kPairStages, kOutDirect>, tm_a, tm_b, mc, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

int tc16_pair_bk() { return kPairBK; }

unsigned take_error_word_pair() { return take_error_word(); }

}  // namespace smg
