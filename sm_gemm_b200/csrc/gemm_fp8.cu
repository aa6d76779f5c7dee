// Block-scaled FP8 (E4M3) GEMM with per-K-block scale promotion into FP32, one SM per
// 128 x 128 output tile.
//
// The DeepGEMM kernel-library walkthrough (zwxr.cn), section 2.4 quantises with one
// FP32 scale per 1x128 group of the activations and per 128x128 block of the
// weights, and accumulates the low-precision products in FP32 before rescaling. Here
// each 128-wide K-block kb of a tile is multiplied on the tensor core into an FP32 TMEM
// partial P_kb (kind::f8f6f4, four K=32 steps), and promotion warps fold it into a
// register accumulator: acc += (sa[kb,m] * sb[kb,nb]) * P_kb. The scales are arbitrary
// FP32 values (amax/448), not powers of two, so the hardware block-scaled MMA (UE8M0 /
// UE4M3 scale factors) cannot apply them exactly; the promotion is done in software.
// Two TMEM partial buffers let the MMA of kb+1 run while kb is promoted.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2 TMEM
// allocator, warp 3 scale loader, warps 4..11 promotion + epilogue: warp w reads TMEM
// lanes 32*(w%4).. (tile rows) and columns 64*((w-4)/4).. (64 of the 128 columns).
//
// The scale loader stages each K-block's 128 row scales and its block scale in an
// 8-slot shared-memory ring with asynchronous copies. Promotion warps then never have
// a global load in flight when they release a TMEM buffer (an mbarrier arrive has
// release semantics and would wait for such loads), and read their scales from
// shared memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace smg {

namespace {
constexpr int kThreads = 384;
constexpr int kLoaderWarp = 3;
constexpr int kPromoWarp0 = 4;
constexpr int kPromoWarps = 8;
constexpr int kPromoThreads = kPromoWarps * 32;
constexpr int BM = kFp8BM, BN = kFp8BN, BKB = kFp8BK;  // BK in bytes = elements
constexpr int A_BYTES = BM * BKB;                       // 16 KB
constexpr int B_BYTES = BN * BKB;                       // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int STAGES = 6;
constexpr int TCOLS = 256;       // two 128-column FP32 partial buffers
constexpr int kRing = 8;         // scale ring slots
constexpr int kSlotFloats = 132; // 128 row scales + block scale, padded to 16 bytes

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int i) {
  // K-major tile of 128 rows x 128 bytes, 128-byte swizzle; K step i = 32 bytes.
  return sdesc_sw128(base + i * 32, 16, 1024);
}
}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const Fp8Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem_base - smem_u32(smem_raw));
  float* ring = reinterpret_cast<float*>(smem_gen + STAGES * STAGE_BYTES);
  const uint32_t bar_base = smem_base + STAGES * STAGE_BYTES + kRing * kSlotFloats * 4;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto pfull_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
  auto pempty_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + 2 + b); };
  auto sfull_bar = [&](int r) { return bar_base + 8u * (2 * STAGES + 4 + r); };
  auto sempty_bar = [&](int r) { return bar_base + 8u * (2 * STAGES + 4 + kRing + r); };
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 4 + 2 * kRing);
  uint8_t* misc = smem_gen + STAGES * STAGE_BYTES + kRing * kSlotFloats * 4 + 8 * (2 * STAGES + 5 + 2 * kRing);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* reduce_flag = reinterpret_cast<volatile int*>(misc + 8);

  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(pfull_bar(b), 1);
      mbar_init(pempty_bar(b), kPromoWarps);
    }
    for (int r = 0; r < kRing; ++r) {
      mbar_init(sfull_bar(r), 32);
      mbar_init(sempty_bar(r), kPromoWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();
  const TileSched& s = p.s;
  const uint64_t limit = p.wait_limit_cycles;
  const int M = p.e.M;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    WorkIter it;
    it.init(s, blockIdx.x);
    Seg seg;
    bool ok = true;
    while (ok && it.next(s, seg)) {
      int mt, nt;
      tile_coords(s, seg.tile, mt, nt);
      for (int kb = seg.kb0; kb < seg.kb1; ++kb) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, limit)) { ok = false; break; }
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
        tma_load_2d(sa, &tm_a, full_bar(stage), kb * BKB, mt * BM);
        tma_load_2d(sa + A_BYTES, &tm_b, full_bar(stage), kb * BKB, nt * BN);
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok) {
      int st = stage;
      uint32_t ph = phase;
      volatile int no_abort = 0;
      for (long long i = 0; i < issued && i < STAGES; ++i) {
        if (--st < 0) { st = STAGES - 1; ph ^= 1u; }
        mbar_wait(full_bar(st), ph, &no_abort, limit);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t kcount = 0;  // K-blocks issued by this CTA: selects the partial buffer
    WorkIter it;
    it.init(s, blockIdx.x);
    Seg seg;
    bool ok = true;
    while (ok && it.next(s, seg)) {
      for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++kcount) {
        const int buf = static_cast<int>(kcount & 1);
        const uint32_t bphase = (kcount >> 1) & 1;
        if (!mbar_wait(pempty_bar(buf), bphase ^ 1u, abort_flag, limit)) { ok = false; break; }
        if (!mbar_wait(full_bar(stage), phase, abort_flag, limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint32_t d_tmem = tmem_base + buf * BN;
#pragma unroll
        for (int k = 0; k < BKB / 32; ++k)
          umma_f8(d_tmem, kmajor_desc(sa, k), kmajor_desc(sa + A_BYTES, k), p.idesc, k > 0 ? 1u : 0u);
        umma_commit(empty_bar(stage));
        umma_commit(pfull_bar(buf));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    umma_commit(drain_bar);
    volatile int no_abort = 0;
    mbar_wait(drain_bar, 0, &no_abort, limit);
  } else if (warp == kLoaderWarp) {
    // ---------------------------------------------------------------- scale loader
    // Slot layout: [0, 128) row scales sa[kb, m0 + r]; [128] block scale sb[kb, nt].
    // Asynchronous copies (cp.async, zero fill past the matrix edge) complete on the
    // slot's full barrier, so up to kRing K-blocks of scales are in flight at once.
    uint32_t kc = 0;
    WorkIter it;
    it.init(s, blockIdx.x);
    Seg seg;
    bool dead = false;
    const bool vec = (M & 3) == 0 && (reinterpret_cast<uintptr_t>(p.sa) & 15u) == 0;
    const uint32_t ring_u32 = smem_u32(ring);
    while (it.next(s, seg)) {
      int mt, nt;
      tile_coords(s, seg.tile, mt, nt);
      const int m0 = mt * BM + 4 * static_cast<int>(lane);
      for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++kc) {
        const int slot = static_cast<int>(kc % kRing);
        const uint32_t ph = (kc / kRing) & 1;
        if (!dead) dead = !mbar_wait(sempty_bar(slot), ph ^ 1u, abort_flag, limit);
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
        if (lane == 0) cp_async_4(dst + 4 * 128, p.sb + static_cast<long long>(kb) * p.nb_count + nt, 4u);
        cp_async_mbar_arrive(sfull_bar(slot));
      }
    }
    cp_async_wait_all();
  } else if (warp >= kPromoWarp0) {
    // ---------------------------------------------------------------- promotion + epilogue
    const int q = warp & 3;
    const int half = (warp - kPromoWarp0) >> 2;
    const int r_local = q * 32 + lane;
    const int c_local0 = half * 64;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const int ptid = threadIdx.x - kPromoWarp0 * 32;
    uint32_t kcount = 0;
    WorkIter it;
    it.init(s, blockIdx.x);
    Seg seg;
    // `dead` is warp-uniform. After an abandoned wait the loop keeps walking the
    // (deterministic) segment list without touching TMEM or memory, so every named
    // barrier below is still reached by all promotion threads.
    bool dead = false;
    while (it.next(s, seg)) {
      int mt, nt;
      tile_coords(s, seg.tile, mt, nt);
      const int row = mt * BM + r_local;
      float acc[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.0f;
      for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++kcount) {
        const int buf = static_cast<int>(kcount & 1);
        const uint32_t bphase = (kcount >> 1) & 1;
        const int slot = static_cast<int>(kcount % kRing);
        const uint32_t sph = (kcount / kRing) & 1;
        if (!dead) dead = !mbar_wait(sfull_bar(slot), sph, abort_flag, limit);
        if (!dead) dead = !mbar_wait(pfull_bar(buf), bphase, abort_flag, limit);
        dead = __any_sync(0xffffffffu, dead);
        if (dead) continue;
        const float* sl = ring + slot * kSlotFloats;
        const float sc = sl[r_local] * sl[128];
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_addr + buf * BN + c_local0;
        // Both 32-column loads are issued before one wait: one TMEM round trip per K-block.
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(taddr, r0);
        tmem_ld_32x32b_x32(taddr + 32, r1);
        tmem_ld_wait();
        fma_scaled32(acc, sc, r0);
        fma_scaled32(acc + 32, sc, r1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(pempty_bar(buf));
          mbar_arrive(sempty_bar(slot));
        }
      }

      const bool whole = (seg.kb0 == 0 && seg.kb1 == s.kb_total);
      const int col0 = nt * BN + c_local0;
      if (whole) {
        if (!dead) {
          epi_row32<false>(p.e, row, col0, *reinterpret_cast<float(*)[32]>(acc));
          epi_row32<false>(p.e, row, col0 + 32, *reinterpret_cast<float(*)[32]>(acc + 32));
        }
      } else {
        // Stream-K partial: store, then the last contributor reduces in CTA order.
        float* my_slot = p.slots + (static_cast<size_t>(blockIdx.x) * 2 + seg.slot) * (BM * BN);
        if (!dead) slot_store<64>(my_slot, r_local, c_local0, acc);
        const long long t_sk = seg.tile - s.dp_tiles;
        __threadfence();
        named_barrier_sync(1, kPromoThreads);
        if (ptid == 0) {
          const int c_lo = sk_owner(s, t_sk * s.kb_total);
          const int c_hi = sk_owner(s, (t_sk + 1) * s.kb_total - 1);
          int n = 0;
          for (int c = c_lo; c <= c_hi; ++c) n += sk_bound(s, c) < sk_bound(s, c + 1);
          const bool any_dead = *abort_flag != 0;
          const int old = any_dead ? -1 : counter_arrive(p.counters + t_sk, p.gen, n);
          *reduce_flag = (!any_dead && old == n - 1);
        }
        named_barrier_sync(1, kPromoThreads);
        if (*reduce_flag) {
          __threadfence();
          const int c_lo = sk_owner(s, t_sk * s.kb_total);
          const int c_hi = sk_owner(s, (t_sk + 1) * s.kb_total - 1);
#pragma unroll
          for (int j = 0; j < 64; ++j) acc[j] = 0.0f;
#pragma unroll 1
          for (int cc = c_lo; cc <= c_hi; ++cc) {
            if (!(sk_bound(s, cc) < sk_bound(s, cc + 1))) continue;
            const float* src = p.slots + (static_cast<size_t>(cc) * 2 + sk_slot_of(s, cc, t_sk)) * (BM * BN);
            slot_accumulate<64>(src, r_local, c_local0, acc);
          }
          epi_row32<false>(p.e, row, col0, *reinterpret_cast<float(*)[32]>(acc));
          epi_row32<false>(p.e, row, col0 + 32, *reinterpret_cast<float(*)[32]>(acc + 32));
        }
        named_barrier_sync(1, kPromoThreads);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem_base, TCOLS);
}

cudaError_t launch_gemm_fp8(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const Fp8Params& p,
                            int grid, cudaStream_t stream) {
  constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + kRing * kSlotFloats * 4 + 8 * (2 * STAGES + 5 + 2 * kRing) + 16;
  static_assert(SMEM <= 232448, "shared memory budget");
  const cudaError_t attr = smem_opt_in<gemm_fp8_kernel>(SMEM);
  if (attr != cudaSuccess) return attr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute la[1];
  add_pdl_attr(cfg, la);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_fp8_kernel, tm_a, tm_b, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

unsigned take_error_word_fp8() { return take_error_word(); }

}  // namespace smg
