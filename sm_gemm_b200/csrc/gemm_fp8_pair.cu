// Block-scaled FP8 (E4M3) GEMM on CTA pairs (tcgen05.mma.cta_group::2): a 256 x TN
// output tile per pair of SMs (TN = 256 or 128), with per-K-block scale promotion into
// FP32 registers.
//
// Same method as gemm_fp8.cu (the DeepGEMM kernel-library walkthrough, zwxr.cn,
// section 2.4: one FP32 scale per 1x128 activation group and per 128x128 weight block,
// FP32 accumulation, rescale per group): for each 128-wide K-block kb the pair's
// tensor cores write the FP32 partial P_kb of the 256 x TN tile into one of the TMEM
// buffers (each SM holds its 128 rows x TN columns), and 8 promotion warps per SM
// fold it into registers, acc += (sa[kb, m] * sb[kb, n / 128]) * P_kb.
//
// TMEM holds 512 / TN partial buffers, and the MMA of K-block kb can only start once
// the promotion of kb - 512/TN has freed its buffer. With TN = 256 (two buffers) the
// K loop is bound by that round trip (MMA latency + promotion latency over two
// K-blocks) rather than by the tensor cores; TN = 128 has four buffers and twice the
// slack, at the price of re-reading A once per 128 instead of 256 output columns.
//
// Roles (384 threads per CTA = 3 warpgroups):
//  warp 0     TMEM allocator (whole warp), then lane 0 is the TMA producer.
//  warp 1     MMA issuer (rank-0 CTA only).
//  warp 2     scale loader: stages each K-block's 128 row scales and the block scales of
//             this CTA in a shared-memory ring with asynchronous copies, so promotion
//             warps never hold a global load in flight when they release a TMEM buffer
//             (an mbarrier arrive has release semantics and would wait for it).
//  warps 4-11 promotion + epilogue: warp w reads TMEM lanes 32*(w%4).. (tile rows) and
//             the TN/2 columns (TN/2)*((w-4)/4).. of the tile; TN/2 FP32 accumulators
//             per thread.
// Warpgroup 0 gives up registers (setmaxnreg 40) so the two promotion warpgroups can
// hold the accumulators (setmaxnreg 232; 384 x 168 registers at launch).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace smg {

namespace {
constexpr int kThreads = 384;
constexpr int kLoaderWarp = 2;
constexpr int kPromoWarp0 = 4;
constexpr int kPromoWarps = 8;
constexpr int kPromoThreads = kPromoWarps * 32;
constexpr int BKB = 128;                 // K-block in bytes = elements = one scale group
constexpr int A_BYTES = 128 * BKB;       // this CTA's 128 rows of A
constexpr int TCOLS = 512;               // all of TMEM: 512 / TN partial buffers
constexpr int kRing = 8;                 // scale ring slots
constexpr int kSlotFloats = 132;         // 128 row scales + up to 2 block scales, padded to 16 B
// setmaxnreg split: 128 x 40 + 256 x 232 = 64512 registers, all of the 384 x 168 the
// block launches with (prepare() checks the compiled count before any launch).
constexpr int kRoleRegs = 40, kPromoRegs = 232;
static_assert(128 * kRoleRegs + kPromoThreads * kPromoRegs <= kThreads * 168, "register split");

// Per-tile-width constants: this CTA's B rows (TN / 2), stage size, pipeline depth and
// the number of TMEM partial buffers.
template <int TN>
struct PairCfg {
  static constexpr int kBRows = TN / 2;
  static constexpr int B_BYTES = kBRows * BKB;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = TN == 256 ? 6 : 8;
  static constexpr int NBUF = TCOLS / TN;
  static constexpr int CPW = TN / 2;                  // columns per promotion warp
  static constexpr int kBars = 2 * STAGES + 2 * NBUF + 2 * kRing + 1;
  static constexpr int kSmem = 1024 + STAGES * STAGE_BYTES + kRing * kSlotFloats * 4 + 8 * kBars + 16;
  static_assert(kSmem <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int i) {
  return sdesc_sw128(base + i * 32, 16, 1024);
}
}  // namespace

template <int TN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_fp8_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                         const Fp8Params p) {
  using Cfg = PairCfg<TN>;
  constexpr int STAGES = Cfg::STAGES, STAGE_BYTES = Cfg::STAGE_BYTES, NBUF = Cfg::NBUF, CPW = Cfg::CPW;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem_base - smem_u32(smem_raw));
  float* ring = reinterpret_cast<float*>(smem_gen + STAGES * STAGE_BYTES);
  const uint32_t bar_base = smem_base + STAGES * STAGE_BYTES + kRing * kSlotFloats * 4;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto pfull_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
  auto pempty_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + NBUF + b); };
  auto sfull_bar = [&](int r) { return bar_base + 8u * (2 * STAGES + 2 * NBUF + r); };
  auto sempty_bar = [&](int r) { return bar_base + 8u * (2 * STAGES + 2 * NBUF + kRing + r); };
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 2 * NBUF + 2 * kRing);
  uint8_t* misc = smem_gen + STAGES * STAGE_BYTES + kRing * kSlotFloats * 4 + 8 * Cfg::kBars;
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
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(pfull_bar(b), 1);
      mbar_init(pempty_bar(b), 2 * kPromoWarps);
    }
    for (int r = 0; r < kRing; ++r) {
      mbar_init(sfull_bar(r), 32);
      mbar_init(sempty_bar(r), kPromoWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), TCOLS);
    tmem_relinquish_pair();
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();
  const TileSched& s = p.s;
  const uint64_t limit = p.wait_limit_cycles;
  if (warp < kPromoWarp0) {
    // Warpgroup 0: producer, MMA issuer, scale loader (few registers each).
    regs_dec<kRoleRegs>();
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
      const int b_row = nt * TN + static_cast<int>(rank) * Cfg::kBRows;
      for (int kb = seg.kb0; kb < seg.kb1; ++kb) {
        const bool w = mbar_wait_inl(empty_bar(stage), phase ^ 1u, abort_flag, limit);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        const uint32_t sa_s = smem_base + stage * STAGE_BYTES;
        const uint32_t leader_full = mapa_shared(full_bar(stage), 0);
        if (elect_one()) {
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          tma_load_2d_pair(sa_s, &tm_a, leader_full, kb * BKB, a_row);
          tma_load_2d_pair(sa_s + A_BYTES, &tm_b, leader_full, kb * BKB, b_row);
        }
        __syncwarp();
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok && rank == 0 && lane == 0) {
      int st = stage;
      uint32_t ph = phase;
      volatile int no_abort = 0;
      for (long long i = 0; i < issued && i < STAGES; ++i) {
        if (--st < 0) { st = STAGES - 1; ph ^= 1u; }
        mbar_wait_inl(full_bar(st), ph, &no_abort, limit);
      }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // -------------------------------------------------------------- MMA issuer
      // Warp-wide loop, one elected lane issues (always the same lane, so its commits
      // cover every MMA it issued).
      int stage = 0;
      uint32_t phase = 0;
      long long kcount = 0;
      WorkIter it;
      it.init(s, cluster);
      Seg seg;
      bool ok = true;
      while (ok && it.next(s, seg)) {
        for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++kcount) {
          const int buf = static_cast<int>(kcount % NBUF);
          const uint32_t bphase = static_cast<uint32_t>((kcount / NBUF) & 1);
          bool w = mbar_wait_inl(pempty_bar(buf), bphase ^ 1u, abort_flag, limit);
          w = w && mbar_wait_inl(full_bar(stage), phase, abort_flag, limit);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa_s = smem_base + stage * STAGE_BYTES;
          const uint32_t d_tmem = tmem_base + buf * TN;
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < BKB / 32; ++k)
              umma_f8_pair(d_tmem, kmajor_desc(sa_s, k), kmajor_desc(sa_s + A_BYTES, k), p.idesc, k > 0 ? 1u : 0u);
            umma_commit_pair(empty_bar(stage), 0x3);
            umma_commit_pair(pfull_bar(buf), 0x3);
          }
          __syncwarp();
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (elect_one()) umma_commit_pair(drain_bar, 0x1);
      __syncwarp();
      volatile int no_abort = 0;
      mbar_wait_inl(drain_bar, 0, &no_abort, limit);
    }
  } else if (warp == kLoaderWarp) {
    // ---------------------------------------------------------------- scale loader
    // Slot layout: [0, 128) row scales sa[kb, m0 + r]; [128 + h] block scale of the tile's
    // h-th 128-column block, sb[kb, (TN / 128) * nt + h]. The copies are asynchronous (cp.async,
    // zero fill past the matrix edge) and complete on the slot's full barrier, so the
    // loader keeps up to kRing K-blocks of scales in flight instead of one.
    const int M = p.e.M;
    uint32_t kc = 0;
    WorkIter it;
    it.init(s, cluster);
    Seg seg;
    bool dead = false;
    const bool vec = (M & 3) == 0 && (reinterpret_cast<uintptr_t>(p.sa) & 15u) == 0;
    const uint32_t ring_u32 = smem_u32(ring);
    while (it.next(s, seg)) {
      int mt, nt;
      tile_coords(s, seg.tile, mt, nt);
      const int m0 = mt * 256 + static_cast<int>(rank) * 128 + 4 * static_cast<int>(lane);
      for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++kc) {
        const int slot = static_cast<int>(kc % kRing);
        const uint32_t ph = (kc / kRing) & 1;
        if (!dead) dead = !mbar_wait_inl(sempty_bar(slot), ph ^ 1u, abort_flag, limit);
        dead = __any_sync(0xffffffffu, dead);
        if (dead) {
          mbar_arrive(sfull_bar(slot));
          continue;
        }
        const float* src = p.sa + static_cast<long long>(kb) * M + m0;
        const uint32_t dst = ring_u32 + static_cast<uint32_t>(slot * kSlotFloats * 4);
        if (vec) {
          cp_async_16(dst + 16 * lane, m0 < M ? src : p.sa, m0 < M ? 16u : 0u);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            cp_async_4(dst + 16 * lane + 4 * e, m0 + e < M ? src + e : p.sa, m0 + e < M ? 4u : 0u);
        }
        if (lane < TN / 128) {
          const int nb = (TN / 128) * nt + static_cast<int>(lane);
          const float* sbp = p.sb + static_cast<long long>(kb) * p.nb_count + nb;
          cp_async_4(dst + 4 * (128 + lane), nb < p.nb_count ? sbp : p.sb, nb < p.nb_count ? 4u : 0u);
        }
        cp_async_mbar_arrive(sfull_bar(slot));
      }
    }
    cp_async_wait_all();
  }
  } else {
    // Warpgroups 1-2: promotion + epilogue (CPW accumulators per thread).
    regs_inc<kPromoRegs>();
    // ---------------------------------------------------------------- promotion + epilogue
    const int q = warp & 3;
    const int cg = (warp - kPromoWarp0) >> 2;  // 0..1: column half of the tile
    const int r_local = q * 32 + lane;
    const int c_local0 = cg * CPW;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const int ptid = threadIdx.x - kPromoWarp0 * 32;
    constexpr int SLOT = 128 * TN;
    uint32_t kcount = 0;
    WorkIter it;
    it.init(s, cluster);
    Seg seg;
    bool dead = false;
    while (it.next(s, seg)) {
      int mt, nt;
      tile_coords(s, seg.tile, mt, nt);
      const int row = mt * 256 + static_cast<int>(rank) * 128 + r_local;
      float acc[CPW];
#pragma unroll
      for (int j = 0; j < CPW; ++j) acc[j] = 0.0f;
      for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++kcount) {
        const int buf = static_cast<int>(kcount % NBUF);
        const uint32_t bphase = (kcount / NBUF) & 1;
        const int slot = static_cast<int>(kcount % kRing);
        const uint32_t sph = (kcount / kRing) & 1;
        if (!dead) dead = !mbar_wait_inl(sfull_bar(slot), sph, abort_flag, limit);
        if (!dead) dead = !mbar_wait_inl(pfull_bar(buf), bphase, abort_flag, limit);
        dead = __any_sync(0xffffffffu, dead);
        if (dead) continue;
        const float* sl = ring + slot * kSlotFloats;
        const float sc = sl[r_local] * sl[128 + c_local0 / 128];
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_addr + buf * TN + c_local0;
        // 32-column TMEM loads, each followed by its packed FMAs.
#pragma unroll
        for (int h = 0; h < CPW / 32; ++h) {
          uint32_t r[32];
          tmem_ld_32x32b_x32_sync(taddr + h * 32, r);
          fma_scaled32(acc + 32 * h, sc, r);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_cluster_relaxed(mapa_shared(pempty_bar(buf), 0));
          mbar_arrive(sempty_bar(slot));
        }
      }

      const bool whole = (seg.kb0 == 0 && seg.kb1 == s.kb_total);
      const int col0 = nt * TN + c_local0;
      if (whole) {
        if (!dead) {
#pragma unroll
          for (int h = 0; h < CPW / 32; ++h)
            epi_row32<false>(p.e, row, col0 + 32 * h, *reinterpret_cast<float(*)[32]>(acc + 32 * h));
        }
      } else {
        float* my_slot = p.slots + ((static_cast<size_t>(cluster) * 2 + seg.slot) * 2 + rank) * SLOT;
        if (!dead) slot_store<CPW>(my_slot, r_local, c_local0, acc);
        const long long t_sk = seg.tile - s.dp_tiles;
        __threadfence();
        named_barrier_sync(1, kPromoThreads);
        if (ptid == 0) {
          const int c_lo = sk_owner(s, t_sk * s.kb_total);
          const int c_hi = sk_owner(s, (t_sk + 1) * s.kb_total - 1);
          int n = 0;
          for (int c = c_lo; c <= c_hi; ++c) n += sk_bound(s, c) < sk_bound(s, c + 1);
          const bool any_dead = *abort_flag != 0;
          const int old = any_dead ? -1 : counter_arrive(p.counters + t_sk * 2 + rank, p.gen, n);
          *reduce_flag = (!any_dead && old == n - 1);
        }
        named_barrier_sync(1, kPromoThreads);
        if (*reduce_flag) {
          __threadfence();
          const int c_lo = sk_owner(s, t_sk * s.kb_total);
          const int c_hi = sk_owner(s, (t_sk + 1) * s.kb_total - 1);
#pragma unroll 1
          for (int h = 0; h < CPW / 32; ++h) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.0f;
#pragma unroll 1
            for (int cc = c_lo; cc <= c_hi; ++cc) {
              if (!(sk_bound(s, cc) < sk_bound(s, cc + 1))) continue;
              const float* src = p.slots + ((static_cast<size_t>(cc) * 2 + sk_slot_of(s, cc, t_sk)) * 2 + rank) * SLOT;
              slot_accumulate<32>(src, r_local, c_local0 + 32 * h, v);
            }
            epi_row32<false>(p.e, row, col0 + 32 * h, v);
          }
        }
        named_barrier_sync(1, kPromoThreads);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 0) tmem_dealloc_pair(tmem_base, TCOLS);
}

namespace {
// Checks that the registers the kernel launches with cover the setmaxnreg split
// (otherwise the promotion warps' increase would never be granted); a build that breaks
// the split fails here instead of launching.
template <int TN>
cudaError_t prepare_once() {
  cudaFuncAttributes attr{};
  const cudaError_t e = cudaFuncGetAttributes(&attr, gemm_fp8_pair_kernel<TN>);
  if (e != cudaSuccess) return e;
  if (attr.numRegs * kThreads < 128 * kRoleRegs + kPromoThreads * kPromoRegs) return cudaErrorInvalidConfiguration;
  return cudaSuccess;
}

template <int TN>
cudaError_t prepare() {
  static cudaError_t st = prepare_once<TN>();
  if (st != cudaSuccess) return st;
  return smem_opt_in<gemm_fp8_pair_kernel<TN>>(PairCfg<TN>::kSmem);
}

template <int TN>
cudaLaunchConfig_t pair_config(int clusters, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = PairCfg<TN>::kSmem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int TN>
int max_clusters() {
  static int cached = -1;
  if (cached >= 0) return cached;
  if (prepare<TN>() != cudaSuccess) return 0;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pair_config<TN>(1, nullptr, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_fp8_pair_kernel<TN>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cached = n;
  return n;
}

template <int TN>
cudaError_t launch(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const Fp8Params& p, int clusters,
                   cudaStream_t stream) {
  cudaError_t e = prepare<TN>();
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_config<TN>(clusters, stream, attr);
  add_pdl_attr(cfg, attr);
  e = cudaLaunchKernelEx(&cfg, gemm_fp8_pair_kernel<TN>, tm_a, tm_b, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}
}  // namespace

int fp8_pair_max_clusters(int tn) { return tn == 128 ? max_clusters<128>() : max_clusters<256>(); }

cudaError_t launch_gemm_fp8_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const Fp8Params& p,
                                 int clusters, int tn, cudaStream_t stream) {
  return tn == 128 ? launch<128>(tm_a, tm_b, p, clusters, stream) : launch<256>(tm_a, tm_b, p, clusters, stream);
}

unsigned take_error_word_fp8_pair() { return take_error_word(); }

}  // namespace smg
