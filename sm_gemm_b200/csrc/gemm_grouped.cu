// Grouped 16-bit GEMM: G independent problems C_g = act(A_g B_g + bias_g) in one
// persistent launch on CTA pairs (256 x 256 tiles, tcgen05.mma.cta_group::2).
//
// This is the batching remedy of "为什么我们要死磕GEMM" (kwkr.cn), section 5.3: many small
// GEMMs issued one by one each pay a launch and a ragged last wave, while one launch
// over all of their tiles keeps every SM busy until the last tile. Tiles are numbered
// group by group (grouped raster inside a group); cluster c takes tiles c, c + P, c + 2P,
// ... over the whole list, so consecutive tiles of one group run side by side.
//
// Per-group data (GroupDesc: both TMA descriptors, sizes, output and bias pointers) comes
// with the launch as a kernel parameter for up to kInlineGroups groups, else from a device
// table that the host writes into the caller's workspace before the launch. Every role
// finds a tile's group by binary search over the groups' first-tile indices. With the
// device table the producer issues fence.proxy.tensormap acquire on a group's
// descriptors before its first copy from them, since the table may have been rewritten
// since an earlier launch.
//
// Roles as in gemm_tc16_pair.cu: warp 0 TMA producer and warp 1 MMA issuer (warp-wide
// loops, one elected lane issues; MMA on the rank-0 CTA only), warp 2 TMEM allocator,
// warps 4-11 epilogue (each CTA drains its own 128 rows of the two TMEM accumulators;
// warp w takes lanes 32*(w%4).. and the 128 columns 128*((w-4)/4).. of the tile, or the
// 64 columns 64*((w-4)/4).. of a transposed tile).
// When the tiles leave a ragged last wave (R = T mod P tiles for P clusters), those R
// tiles are split along K into S pieces (R S <= P) that run side by side; each piece's
// partial goes to a workspace slot and the last piece to finish sums them in order.
//
// A group whose last row of tiles holds at most 128 rows (M mod 256 in 1..128) would
// leave half of each of those 256-row tiles empty. Those tiles run transposed instead:
// the pair computes the 256 x 128 tile of C^T = B^T A^T, with 256 columns of B as the
// MMA's M (128 per CTA, the same load as B's half of a normal tile) and the up to 128
// remaining rows of A as its N (64 per CTA), and the epilogue writes each TMEM lane (one
// column of C) down the rows. Half the tensor-core work of the padded tile; the MMA then
// reads shared memory faster than at N = 256 per unit of work, but still needs fewer
// cycles per tile than the half-empty one.
#include <cuda_bf16.h>
#include <cstring>
#include <type_traits>
#include <cuda_fp16.h>

#include "epilogue.cuh"
#include "grouped.h"
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
constexpr int kTileN = 256;
constexpr int kTcols = 512;

__device__ __forceinline__ void tensormap_acquire(const CUtensorMap* map) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(reinterpret_cast<uint64_t>(map))
               : "memory");
}

// Group of tile t (the last group whose first tile is <= t; empty groups share their
// successor's first tile and are skipped) and the tile's (mt, nt) inside it.
__device__ __forceinline__ int locate(const GroupedParams& p, long long t, int& mt, int& nt) {
  int lo = 0, hi = p.G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.groups[mid].tile0 <= t) lo = mid;
    else hi = mid - 1;
  }
  const GroupDesc& d = p.groups[lo];
  TileSched ts{};
  ts.m_tiles = d.m_tiles;
  ts.n_tiles = d.n_tiles;
  ts.group_m = p.group_m < d.m_tiles ? p.group_m : d.m_tiles;
  tile_coords(ts, static_cast<int>(t - d.tile0), mt, nt);
  return lo;
}
}  // namespace

// One unit of work: tile `tile` of group `g` over K-blocks [kb0, kb1); unit >= 0 marks a
// piece of a split tail tile (its partial goes to workspace slot `unit`).
struct GItem {
  long long tile;
  int g, mt, nt, kb0, kb1, unit;
  bool tr;  // transposed remainder tile (C^T = B^T A^T, <= 128 rows of A)
};

// Work of cluster c: its piece of the split tail (if any) first, so the tail's fix-up
// overlaps later tiles, then the data-parallel tiles c, c + P, ... below T - R.
struct GIter {
  int c, P;
  long long next_dp;
  bool unit_pending;

  __device__ __forceinline__ void init(const GroupedParams& p, const GroupedSplit& sp, int cluster,
                                       int nclusters) {
    c = cluster;
    P = nclusters;
    next_dp = cluster;
    unit_pending = sp.split_tiles > 0 && cluster < sp.split_tiles * sp.splits;
    (void)p;
  }
  __device__ __forceinline__ bool next(const GroupedParams& p, const GroupedSplit& sp, GItem& it) {
    if (unit_pending) {
      unit_pending = false;
      it.tile = p.total_tiles - sp.split_tiles + c / sp.splits;
      it.g = locate(p, it.tile, it.mt, it.nt);
      const int kbn = p.groups[it.g].kb_total, piece = c % sp.splits;
      it.kb0 = static_cast<int>(static_cast<long long>(piece) * kbn / sp.splits);
      it.kb1 = static_cast<int>(static_cast<long long>(piece + 1) * kbn / sp.splits);
      it.unit = c;
      it.tr = p.groups[it.g].rem_t != 0 && it.mt == p.groups[it.g].m_tiles - 1;
      return true;
    }
    if (next_dp < p.total_tiles - sp.split_tiles) {
      it.tile = next_dp;
      it.g = locate(p, it.tile, it.mt, it.nt);
      it.kb0 = 0;
      it.kb1 = p.groups[it.g].kb_total;
      it.unit = -1;
      it.tr = p.groups[it.g].rem_t != 0 && it.mt == p.groups[it.g].m_tiles - 1;
      next_dp += P;
      return true;
    }
    return false;
  }
};

struct NoInlineTable {};

template <int BK, int STAGES, bool INLINE>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_grouped_kernel(const __grid_constant__ GroupedParams p_in, const __grid_constant__ GroupedSplit sp,
                        const __grid_constant__ std::conditional_t<INLINE, GroupTableInline, NoInlineTable> inl) {
  GroupedParams p = p_in;
  if constexpr (INLINE) p.groups = inl.d;
  constexpr int A_BYTES = 128 * BK * 2;
  constexpr int B_BYTES = 128 * BK * 2;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr int KSTEPS = BK / 16;
  constexpr int SLOT = 128 * kTileN;  // floats of one CTA's partial tile

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

  const uint32_t warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;

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
  if (warp == 2) {
    tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), kTcols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();
  const uint64_t limit = p.wait_limit_cycles;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    int last_g = -1;
    bool ok = true;
    GIter wi;
    wi.init(p, sp, cluster, nclusters);
    GItem it;
    while (ok && wi.next(p, sp, it)) {
      const GroupDesc* d = p.groups + it.g;
      if (!INLINE && it.g != last_g && elect_one()) {
        tensormap_acquire(&d->tm_a);
        tensormap_acquire(&d->tm_b);
      }
      last_g = it.g;
      // Normal tile: 128 rows of A and 128 columns of B per CTA. Transposed tile: the
      // same 128 columns of B in the A slot and 64 rows of A in the B slot.
      const int a_row = it.mt * 256 + static_cast<int>(rank) * (it.tr ? 64 : 128);
      const int b_row = it.nt * kTileN + static_cast<int>(rank) * 128;
      const uint32_t tx_bytes = it.tr ? 2 * (A_BYTES + B_BYTES / 2) : 2 * STAGE_BYTES;
      for (int kb = it.kb0; kb < it.kb1; ++kb) {
        const bool w = mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, limit);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint32_t leader_full = mapa_shared(full_bar(stage), 0);
        if (elect_one()) {
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), tx_bytes);
          if (!it.tr) {
            load_operand_pair_r64<128, BK>(sa, &d->tm_a, leader_full, p.a_mn_major, a_row, kb * BK);
            load_operand_pair<128, BK>(sa + A_BYTES, &d->tm_b, leader_full, p.b_mn_major, b_row, kb * BK);
          } else {
            load_operand_pair<128, BK>(sa, &d->tm_b, leader_full, p.b_mn_major, b_row, kb * BK);
            load_operand_pair_r64<64, BK>(sa + A_BYTES, &d->tm_a, leader_full, p.a_mn_major, a_row, kb * BK);
          }
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
        mbar_wait(full_bar(st), ph, &no_abort, limit);
      }
    }
  } else if (warp == 1 && rank == 0) {
    // ---------------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    bool ok = true;
    GIter wi;
    wi.init(p, sp, cluster, nclusters);
    GItem it;
    while (ok && wi.next(p, sp, it)) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, limit))) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * kTileN;
      // Transposed tile: B's columns are the MMA's A operand and A's rows its B operand
      // (64 rows per CTA; for BK = 64 the slice descriptors of a 64- and a 128-row tile
      // coincide, so only the major-ness flags and the instruction descriptor change).
      static_assert(BK == 64, "64-row operand tiles share the 128-row slice descriptors");
      const int amn = it.tr ? p.b_mn_major : p.a_mn_major;
      const int bmn = it.tr ? p.a_mn_major : p.b_mn_major;
      const uint32_t idesc = it.tr ? p.idesc_t : p.idesc;
      for (int kb = it.kb0; kb < it.kb1; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(full_bar(stage), phase, abort_flag, limit))) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint32_t sb = sa + A_BYTES;
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < KSTEPS; ++k) {
            umma_f16_pair(d_tmem, operand_desc<128, BK>(sa, amn, k), operand_desc<128, BK>(sb, bmn, k), idesc,
                          (kb > it.kb0 || k > 0) ? 1u : 0u);
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
    const int r_local = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const int epi_tid = threadIdx.x - kEpiWarp0 * 32;
    const int cg = (warp - kEpiWarp0) >> 2;  // which half of the tile's columns
    int local = 0;
    bool dead = false;
    GIter wi;
    wi.init(p, sp, cluster, nclusters);
    GItem it;
    while (wi.next(p, sp, it)) {
      const GroupDesc* d = p.groups + it.g;
      const EpiArgs e{d->M, d->N, d->bias, p.bias_dtype, p.act, d->C, p.c_dtype, d->ldc};
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!dead) dead = !mbar_wait(tfull_bar(acc), acc_phase, abort_flag, limit);
      dead = __any_sync(0xffffffffu, dead);
      // Normal tile: this thread owns row `fixed` of C from column `run0` on (128 tile
      // columns per warp); transposed tile: column `fixed` of C (its TMEM lane) from row
      // `run0` down (64 tile columns, i.e. rows of C, per warp).
      const int cols = it.tr ? kEpiCols / 2 : kEpiCols;
      const int c_base = cg * cols;
      const int fixed = (it.tr ? it.nt * kTileN : it.mt * 256) + static_cast<int>(rank) * 128 + r_local;
      const int run0 = (it.tr ? it.mt * 256 : it.nt * kTileN) + c_base;
      auto emit = [&](int c, float(&v)[32]) {
        if (it.tr) epi_col<32>(e, fixed, run0 + c * 32, v);
        else epi_row32(e, fixed, run0 + c * 32, v);
      };
      const uint32_t tacc = tmem_base + lane_addr + acc * kTileN + c_base;
      const bool split = it.unit >= 0;
      float* my_slot = split ? sp.slots + (static_cast<size_t>(it.unit) * 2 + rank) * SLOT : nullptr;
      if (!dead) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < cols / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tacc + c * 32, r);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          if (split) slot_store<32>(my_slot, r_local, c_base + c * 32, v);
          else emit(c, v);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
      }
      if (split) {
        // The last of the tile's S pieces (per rank) sums them in piece order (= K order)
        // and runs the epilogue: deterministic, and no CTA waits for another.
        const long long r_tail = it.tile - (p.total_tiles - sp.split_tiles);
        __threadfence();
        named_barrier_sync(1, kEpiThreads);
        if (epi_tid == 0) {
          const bool any_dead = *abort_flag != 0;
          const int old = any_dead ? -1 : counter_arrive(sp.counters + r_tail * 2 + rank, sp.gen, sp.splits);
          *reduce_flag = (!any_dead && old == sp.splits - 1);
        }
        named_barrier_sync(1, kEpiThreads);
        if (*reduce_flag) {
          __threadfence();
#pragma unroll 1
          for (int c = 0; c < cols / 32; ++c) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.0f;
#pragma unroll 1
            for (int pc = 0; pc < sp.splits; ++pc) {
              const float* src = sp.slots + ((r_tail * sp.splits + pc) * 2 + rank) * static_cast<size_t>(SLOT);
              slot_accumulate<32>(src, r_local, c_base + c * 32, v);
            }
            emit(c, v);
          }
        }
        named_barrier_sync(1, kEpiThreads);
      }
      ++local;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 2) tmem_dealloc_pair(tmem_base, kTcols);
}

namespace {
constexpr int kBK = 64, kStages = 6;
constexpr int kSmem = 1024 + kStages * (2 * 128 * kBK * 2) + 8 * (2 * kStages + 5) + 16;  // + misc words
static_assert(kSmem <= 232448, "shared memory budget");

cudaError_t prepare() {
  const cudaError_t e = smem_opt_in<gemm_grouped_kernel<kBK, kStages, false>>(kSmem);
  if (e != cudaSuccess) return e;
  return smem_opt_in<gemm_grouped_kernel<kBK, kStages, true>>(kSmem);
}

cudaLaunchConfig_t config(int clusters, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}
}  // namespace

int grouped_max_clusters() {
  static int cached = -1;
  if (cached >= 0) return cached;
  if (prepare() != cudaSuccess) return 0;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = config(1, nullptr, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_grouped_kernel<kBK, kStages, false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cached = n;
  return n;
}

int grouped_bk() { return kBK; }

cudaError_t launch_gemm_grouped_split(const GroupedParams& p, const GroupedSplit& sp, const GroupTableInline* inl,
                                      int clusters, cudaStream_t stream) {
  cudaError_t e = prepare();
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = config(clusters, stream, attr);
  add_pdl_attr(cfg, attr);
  if (inl != nullptr) e = cudaLaunchKernelEx(&cfg, gemm_grouped_kernel<kBK, kStages, true>, p, sp, *inl);
  else e = cudaLaunchKernelEx(&cfg, gemm_grouped_kernel<kBK, kStages, false>, p, sp, NoInlineTable{});
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

namespace {
// More than kInlineGroups records reach the workspace through kernels whose parameters
// carry up to kUploadGroups records each (within the 32 KB a launch's parameters may
// hold): the table travels by value with the launch, so a call captured in a CUDA graph
// replays it, where a copy from the caller's pageable host memory would be read again at
// every replay from memory freed after the call.
constexpr int kUploadGroups = 96;
struct GroupTableChunk {
  GroupDesc d[kUploadGroups];
};
static_assert(sizeof(GroupTableChunk) <= 32000, "kernel parameter budget");

__global__ void __launch_bounds__(256) upload_group_table_kernel(const __grid_constant__ GroupTableChunk c, int count,
                                                                 GroupDesc* __restrict__ dst) {
  const uint4* src = reinterpret_cast<const uint4*>(&c);
  uint4* out = reinterpret_cast<uint4*>(dst);
  const int words = count * static_cast<int>(sizeof(GroupDesc) / sizeof(uint4));
  for (int i = static_cast<int>(threadIdx.x); i < words; i += static_cast<int>(blockDim.x)) out[i] = src[i];
}
}  // namespace

cudaError_t launch_upload_group_table(const GroupDesc* table, int G, GroupDesc* dst, cudaStream_t stream) {
  static_assert(sizeof(GroupDesc) % sizeof(uint4) == 0, "records are whole 16-byte words");
  for (int first = 0; first < G; first += kUploadGroups) {
    const int count = G - first < kUploadGroups ? G - first : kUploadGroups;
    GroupTableChunk c;
    std::memcpy(c.d, table + first, static_cast<size_t>(count) * sizeof(GroupDesc));
    upload_group_table_kernel<<<1, 256, 0, stream>>>(c, count, dst + first);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_gemm_grouped(const GroupedParams& p, int clusters, cudaStream_t stream) {
  return launch_gemm_grouped_split(p, GroupedSplit{0, 0, nullptr, nullptr, 0}, nullptr, clusters, stream);
}

unsigned take_error_word_grouped() { return take_error_word(); }

}  // namespace smg
