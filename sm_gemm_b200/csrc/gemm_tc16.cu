// Persistent warp-specialised tcgen05 GEMM for 16-bit inputs (bf16 / f16), FP32
// accumulation in TMEM, fused bias + activation + cast epilogue.
//
// One kernel template serves both paths of gemm_bf16:
//  - large tiles: MMA tile 128 x 256 (MMA "A" = A rows, MMA "B" = B columns), BK = 64;
//  - skinny M (the thin-and-tall LM-head / decode shape of "为什么我们要死磕GEMM",
//    kwkr.cn, sections 2.2 and 7.2): swap-AB, the weight supplies the 128 MMA rows
//    and the few tokens are the MMA N (16..64), so the tensor core streams the
//    weight once; the epilogue writes the transposed accumulator. For the LM head
//    fused with its log-softmax (same page, section 7.2) the epilogue also reduces
//    each 128-column tile of every token row to (max, sum of exp) partials.
//
// Warp roles (256 threads): warp 0 = TMA producer, warp 1 = MMA issuer, warp 2 =
// TMEM allocator, warp 3 idle, warps 4..7 = epilogue (warp w reads TMEM lanes
// 32*(w%4) .. +31). Shared memory holds an S-stage ring of operand tiles with
// full/empty mbarriers; TMEM holds two accumulators so the epilogue of one tile
// overlaps the MMAs of the next (DeepGEMM kernel-library walkthrough, zwxr.cn,
// section 2.3: keep the copy running ahead of the math). The fused epilogue is that
// page's section 5.1; the FP32 accumulator its section 2.4.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "operands.cuh"
#include "sm100.cuh"

namespace smg {

namespace {

constexpr int kEpiWarp0 = 4;
constexpr int kThreads = 256;

// Log-softmax partials of one epilogue chunk (swap-AB layout: thread = output column n,
// v[j] = accumulator of token tok0 + j). For each token, the 128 columns' max logit
// (bias included) and sum of exp(logit - max) are reduced across the 4 epilogue warps
// (shuffles, then `red`: 8 x CH floats of shared memory) and written to
// part[vt * M + token]. Every epilogue thread calls it (named barrier 2, 128 threads);
// dead threads and columns past N contribute nothing.
template <int CH>
__device__ __forceinline__ void lse_partial(const Tc16Params& p, int n, int tok0, int vt, const float* v, bool dead,
                                            float* red, int epi_tid) {
  const bool valid = !dead && n < p.e.N;
  const float b = (valid && p.e.bias != nullptr) ? load_bias(p.e.bias, p.e.bias_dtype, n) : 0.0f;
  const int w = epi_tid >> 5, ln = epi_tid & 31;
  float x[CH];
#pragma unroll
  for (int j = 0; j < CH; ++j) {
    x[j] = valid ? v[j] + b : -INFINITY;
    float m = x[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (ln == 0) red[w * CH + j] = m;
  }
  named_barrier_sync(2, 128);
#pragma unroll
  for (int j = 0; j < CH; ++j) {
    const float mx = fmaxf(fmaxf(red[j], red[CH + j]), fmaxf(red[2 * CH + j], red[3 * CH + j]));
    float e = valid ? expf(x[j] - mx) : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
    if (ln == 0) red[4 * CH + w * CH + j] = e;
  }
  named_barrier_sync(2, 128);
  if (epi_tid < CH && tok0 + epi_tid < p.e.M) {
    const int j = epi_tid;
    const float mx = fmaxf(fmaxf(red[j], red[CH + j]), fmaxf(red[2 * CH + j], red[3 * CH + j]));
    const float sum = ((red[4 * CH + j] + red[5 * CH + j]) + red[6 * CH + j]) + red[7 * CH + j];
    p.lse_part[static_cast<size_t>(vt) * p.e.M + tok0 + j] = make_float2(mx, sum);
  }
  named_barrier_sync(2, 128);
}

}  // namespace

template <int MMA_N, int BK, int STAGES, bool SWAP>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc16_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const Tc16Params p) {
  constexpr int A_BYTES = 128 * BK * 2;
  constexpr int B_BYTES = MMA_N * BK * 2;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr int KSTEPS = BK / 16;
  constexpr int TCOLS = TmemCols<MMA_N>::v;
  constexpr int CH = MMA_N < 32 ? MMA_N : 32;  // epilogue chunk (TMEM columns per load)

  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem_base - smem_u32(smem_raw));
  const uint32_t bar_base = smem_base + STAGES * STAGE_BYTES;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 4);
  uint8_t* misc = smem_gen + STAGES * STAGE_BYTES + 8 * (2 * STAGES + 5);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* reduce_flag = reinterpret_cast<volatile int*>(misc + 8);
  float* lse_red = reinterpret_cast<float*>(misc + 16);  // 8 x CH floats (log-softmax partials)

  const uint32_t warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 4);
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
        load_operand<128, BK>(sa, &tm_a, full_bar(stage), p.a_mn_major, mt * 128, kb * BK);
        load_operand<MMA_N, BK>(sa + A_BYTES, &tm_b, full_bar(stage), p.b_mn_major, nt * MMA_N, kb * BK);
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok) {
      // Wait (bounded, independent of the abort flag) for copies still in flight.
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
    int local = 0;
    WorkIter it;
    it.init(s, blockIdx.x);
    Seg seg;
    bool ok = true;
    while (ok && it.next(s, seg)) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, limit)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * MMA_N;
      for (int kb = seg.kb0; kb < seg.kb1; ++kb) {
        if (!mbar_wait(full_bar(stage), phase, abort_flag, limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint32_t sb = sa + A_BYTES;
#pragma unroll
        for (int k = 0; k < KSTEPS; ++k) {
          umma_f16(d_tmem, operand_desc<128, BK>(sa, p.a_mn_major, k),
                   operand_desc<MMA_N, BK>(sb, p.b_mn_major, k), p.idesc,
                   (kb > seg.kb0 || k > 0) ? 1u : 0u);
        }
        umma_commit(empty_bar(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      umma_commit(tfull_bar(acc));
      ++local;
    }
    // Drain: every MMA issued above completes before TMEM is released.
    umma_commit(drain_bar);
    volatile int no_abort = 0;
    mbar_wait(drain_bar, 0, &no_abort, limit);
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int r_local = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const int epi_tid = threadIdx.x - kEpiWarp0 * 32;
    int local = 0;
    WorkIter it;
    it.init(s, blockIdx.x);
    Seg seg;
    // `dead` is warp-uniform; after an abandoned wait the loop keeps walking the
    // segment list without touching TMEM or memory so that all 128 epilogue threads
    // still reach every named barrier.
    bool dead = false;
    while (it.next(s, seg)) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!dead) dead = !mbar_wait(tfull_bar(acc), acc_phase, abort_flag, limit);
      dead = __any_sync(0xffffffffu, dead);
      int mt, nt;
      tile_coords(s, seg.tile, mt, nt);
      const uint32_t tacc = tmem_base + lane_addr + acc * MMA_N;
      const bool whole = (seg.kb0 == 0 && seg.kb1 == s.kb_total);
      float* my_slot = p.slots + (static_cast<size_t>(blockIdx.x) * 2 + seg.slot) * (128 * MMA_N);
      // Log-softmax partials (swap-AB only): every epilogue warp, dead or not, takes part
      // in their named barriers, so the chunk loop then runs on all warps.
      const bool lse_on = SWAP && p.lse_part != nullptr;
      if (!dead || (lse_on && whole)) {
        if (!dead) tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < MMA_N / CH; ++c) {
          float v[32];
          if (!dead) {
            uint32_t r[32];
            if constexpr (CH == 32) {
              tmem_ld_32x32b_x32(tacc + c * 32, r);
            } else {
              uint32_t r16[16];
              tmem_ld_32x32b_x16(tacc + c * 16, r16);
#pragma unroll
              for (int j = 0; j < 16; ++j) r[j] = r16[j];
            }
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.0f;
          }
          if (whole) {
            if constexpr (SWAP) {
              if (lse_on) lse_partial<CH>(p, mt * 128 + r_local, nt * MMA_N + c * CH, mt, v, dead, lse_red, epi_tid);
              if (!dead) epi_col<CH>(p.e, mt * 128 + r_local, nt * MMA_N + c * CH, v);
            } else {
              if (!dead) epi_row32(p.e, mt * 128 + r_local, nt * MMA_N + c * CH, v);
            }
          } else if (!dead) {
            slot_store<CH>(my_slot, r_local, c * CH, v);
          }
        }
        if (!dead) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty_bar(acc));
        }
      }

      if (!whole) {
        // Stream-K fix-up: the last contributor of the tile sums every contributor's
        // partial in CTA order (= K order) and runs the epilogue.
        const long long t_sk = seg.tile - s.dp_tiles;
        __threadfence();
        named_barrier_sync(1, 128);
        if (epi_tid == 0) {
          const int c_lo = sk_owner(s, t_sk * s.kb_total);
          const int c_hi = sk_owner(s, (t_sk + 1) * s.kb_total - 1);
          int n = 0;
          for (int c = c_lo; c <= c_hi; ++c) n += sk_bound(s, c) < sk_bound(s, c + 1);
          const bool any_dead = *abort_flag != 0;
          const int old = any_dead ? -1 : counter_arrive(p.counters + t_sk, p.gen, n);
          *reduce_flag = (!any_dead && old == n - 1);
        }
        named_barrier_sync(1, 128);
        if (*reduce_flag) {
          __threadfence();
          const int c_lo = sk_owner(s, t_sk * s.kb_total);
          const int c_hi = sk_owner(s, (t_sk + 1) * s.kb_total - 1);
#pragma unroll 1
          for (int c = 0; c < MMA_N / CH; ++c) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.0f;
#pragma unroll 1
            for (int cc = c_lo; cc <= c_hi; ++cc) {
              if (!(sk_bound(s, cc) < sk_bound(s, cc + 1))) continue;
              const float* src = p.slots + (static_cast<size_t>(cc) * 2 + sk_slot_of(s, cc, t_sk)) * (128 * MMA_N);
              slot_accumulate<CH>(src, r_local, c * CH, v);
            }
            if constexpr (SWAP) {
              if (lse_on) lse_partial<CH>(p, mt * 128 + r_local, nt * MMA_N + c * CH, mt, v, false, lse_red, epi_tid);
              epi_col<CH>(p.e, mt * 128 + r_local, nt * MMA_N + c * CH, v);
            } else {
              epi_row32(p.e, mt * 128 + r_local, nt * MMA_N + c * CH, v);
            }
          }
        }
        named_barrier_sync(1, 128);
      }
      ++local;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem_base, TCOLS);
}

// ------------------------------------------------------------------ host launchers

template <int MMA_N, int BK, int STAGES, bool SWAP>
static cudaError_t launch_tc16(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const Tc16Params& p,
                               int grid, cudaStream_t stream) {
  constexpr int STAGE_BYTES = 128 * BK * 2 + MMA_N * BK * 2;
  constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 8 * (2 * STAGES + 5) + 16 + 8 * 32 * 4;
  static_assert(SMEM <= 232448, "shared memory budget");
  auto kern = gemm_tc16_kernel<MMA_N, BK, STAGES, SWAP>;
  cudaError_t e = smem_opt_in<gemm_tc16_kernel<MMA_N, BK, STAGES, SWAP>>(SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  add_pdl_attr(cfg, attr);
  e = cudaLaunchKernelEx(&cfg, kern, tm_a, tm_b, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc16(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const Tc16Params& p,
                             Tc16Variant v, int grid, cudaStream_t stream) {
  switch (v) {
    case Tc16Variant::kLarge: return launch_tc16<256, 64, 4, false>(tm_a, tm_b, p, grid, stream);
    case Tc16Variant::kSkinny16: return launch_tc16<16, 128, 6, true>(tm_a, tm_b, p, grid, stream);
    case Tc16Variant::kSkinny32: return launch_tc16<32, 128, 5, true>(tm_a, tm_b, p, grid, stream);
    case Tc16Variant::kSkinny64: return launch_tc16<64, 128, 4, true>(tm_a, tm_b, p, grid, stream);
  }
  return cudaErrorInvalidValue;
}

int tc16_mma_n(Tc16Variant v) {
  switch (v) {
    case Tc16Variant::kLarge: return 256;
    case Tc16Variant::kSkinny16: return 16;
    case Tc16Variant::kSkinny32: return 32;
    case Tc16Variant::kSkinny64: return 64;
  }
  return 0;
}

int tc16_bk(Tc16Variant v) { return v == Tc16Variant::kLarge ? 64 : 128; }

unsigned take_error_word_tc16() { return take_error_word(); }

}  // namespace smg
