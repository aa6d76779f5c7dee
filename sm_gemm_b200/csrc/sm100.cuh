// Blackwell (sm_100a) building blocks shared by the GEMM kernels: mbarriers with a
// bounded wait, TMA tile loads, tcgen05 (TMEM allocation, MMA, commit, loads), the
// UMMA shared-memory and instruction descriptors, and the persistent tile scheduler
// (grouped rasterisation, data-parallel tiles followed by a stream-K range).
//
// The pipeline is the "copy the next tile while the current one is multiplied"
// scheme of the DeepGEMM kernel-library walkthrough (zwxr.cn), section 2.3, built
// from TMA + an S-stage mbarrier ring instead of thread copies and a 2-buffer swap.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <cstdlib>

namespace smg {

// ------------------------------------------------------------------ error word

// Bit set in the device error word when a bounded wait gives up. The host reads and
// clears it in smgemm_check(). Each translation unit has its own word (internal
// linkage, no relocatable device code needed) and exports a take_error_word_* hook.
constexpr unsigned kErrTimeout = 1u;

namespace {
__device__ unsigned int g_error_word = 0;

// Returns and clears this translation unit's device error word (current device).
inline unsigned take_error_word() {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v)) != cudaSuccess) return 0;
  if (v != 0) {
    const unsigned z = 0;
    cudaMemcpyToSymbol(g_error_word, &z, sizeof(z));
  }
  return v;
}
}  // namespace

// ------------------------------------------------------------------ small helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31; }
__device__ __forceinline__ uint32_t warp_id() { return threadIdx.x >> 5; }

// One lane of the (fully active) warp: elect.sync picks the lowest active lane, so
// the same lane is elected every time.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(pred));
  return pred != 0;
}

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Asynchronous global -> shared copies (cp.async) of 4 or 16 bytes; bytes of the
// destination past src_bytes are zero-filled (src_bytes = 0 reads nothing).
// cp_async_mbar_arrive makes the mbarrier count one arrival once every earlier
// cp.async of this thread has landed (the .noinc form: the arrival is one of the
// barrier's expected count), so the copying thread never waits for its loads.
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Slow path of mbar_wait: spin on try_wait, checking the CTA abort flag and the SM cycle
// counter (clock64, cheap) every 64 polls; give up after `limit_cycles` cycles.
static __device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            uint64_t limit_cycles) {
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (static_cast<uint64_t>(clock64() - t0) > limit_cycles) {
      *abort_flag = 1;
      atomicOr(&g_error_word, kErrTimeout);
      return false;
    }
  }
}

// The same bounded wait with the slow path inlined, for kernels that re-partition
// registers with setmaxnreg (ptxas cannot allocate a setmaxnreg region that calls a
// non-inlined function).
__device__ __forceinline__ bool mbar_wait_inl(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                              uint64_t limit_cycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (static_cast<uint64_t>(clock64() - t0) > limit_cycles) {
      *abort_flag = 1;
      atomicOr(&g_error_word, kErrTimeout);
      return false;
    }
  }
}

// Wait until the phase with the given parity of barrier `bar` has completed, for at
// most `limit_cycles` SM cycles. On expiry: record kErrTimeout in the device error
// word, raise the CTA-wide abort flag and return false. Every later wait of the CTA
// returns false soon after when the abort flag is up, so a stalled pipeline drains in
// about one limit instead of one per wait. The common case (phase already complete,
// or completing during the first poll) stays inline and never reads a timer.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_cycles) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, abort_flag, limit_cycles);
}

// Per-warpgroup register reallocation (all warps of the warpgroup execute it).
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------------------------ programmatic dependent launch

// Kernels launched with programmatic stream serialisation may begin while the previous
// kernel on the stream is still finishing. Each kernel lets its successor start setting up
// (launch_dependents) and, before touching global memory, waits until the previous
// kernel has completed and its writes are visible (wait: immediate when there is none).
// Only set-up (barrier init, TMEM allocation, descriptor prefetch) precedes the wait.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Host side: the launch attribute, unless SMGEMM_PDL=0 (pdl_enabled() reads the switch
// snapshot the library takes when a call enters it; defined with the C ABI).
bool pdl_enabled();
// Opts `Kernel` into `bytes` of dynamic shared memory, once per device: the attribute
// belongs to the function on the device that is current when it is set, and persists, so
// later calls on that device skip the runtime call (a per-call cost for small GEMMs).
template <auto Kernel>
inline cudaError_t smem_opt_in(int bytes) {
  constexpr int kMaxDev = 64;
  static std::atomic<int> set_to[kMaxDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool track = dev >= 0 && dev < kMaxDev;
  if (track && set_to[dev].load(std::memory_order_acquire) == bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && track) set_to[dev].store(bytes, std::memory_order_release);
  return e;
}

inline void add_pdl_attr(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attrs) {
  if (!pdl_enabled()) return;
  attrs[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs += 1;
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk tensor copy global -> shared; completion is counted in bytes on `bar`.
// c0 is the innermost (contiguous) coordinate. No multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// 2-D tiled bulk tensor copy shared -> global of this CTA's tile at smem `src`
// (coordinates c0 innermost; rows or columns outside the tensor are not written),
// tracked by the issuing thread's bulk async-group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read shared memory / are pending.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Orders this thread's generic-proxy shared-memory writes before later async-proxy
// (TMA) reads of them.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05 / TMEM

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], 16-bit inputs (bf16 or f16), FP32 accumulate.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// D[tmem] (+)= A * B with 8-bit float inputs (E4M3 here), FP32 accumulate.
__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets lane (base + t),
// columns col .. col+31 of `taddr`.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}


// The same 32-column load followed, in one asm statement, by its wait: the registers
// are defined only once the data has landed, so no use of them can be scheduled
// ahead of the wait.
__device__ __forceinline__ void tmem_ld_32x32b_x32_sync(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from registers to TMEM (the layout of
// tmem_ld_32x32b_x32), and the wait for this thread's earlier TMEM stores.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// acc[j] += s * x[j] (x holds FP32 bit patterns) for j < 32, as 16 packed FP32x2 FMAs
// (fma.rn.f32x2, sm_100): each half is an ordinary correctly rounded fused
// multiply-add, so results equal fmaf's, at half the issued instructions.
__device__ __forceinline__ void fma_scaled32(float* acc, float s, const uint32_t (&x)[32]) {
  const float2 s2 = make_float2(s, s);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float2 a = __ffma2_rn(s2, make_float2(__uint_as_float(x[2 * j]), __uint_as_float(x[2 * j + 1])),
                                make_float2(acc[2 * j], acc[2 * j + 1]));
    acc[2 * j] = a.x;
    acc[2 * j + 1] = a.y;
  }
}

// ------------------------------------------------------------------ CTA pairs (cta_group::2)
//
// Two CTAs of a cluster (ranks 0 and 1, on the two SMs of one TPC) share one MMA: the
// rank-0 CTA issues tcgen05.mma.cta_group::2 over both CTAs' shared-memory operand
// tiles and the result lands in both CTAs' TMEM (rows 0..127 in rank 0, 128..255 in
// rank 1). No load here uses TMA multicast: each CTA loads only its own tiles.

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier of any CTA of the cluster (address from mapa_shared).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Arrive with relaxed semantics on an mbarrier of any CTA of the cluster. For releasing
// a TMEM buffer after tcgen05.wait::ld has returned: the loads are complete, so no
// memory ordering is needed, and a cluster-scope release would stall the thread for
// about 1.5k cycles per arrive.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA tile load into this CTA's shared memory whose byte count completes on an
// mbarrier of either CTA of the pair (here: always the rank-0 CTA's).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_f8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Arrive once on the barrier at offset `bar` in every CTA of `cta_mask` when all
// tcgen05.mma issued so far by this thread (over the pair) have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          bar),
      "h"(cta_mask)
      : "memory");
}

// ------------------------------------------------------------------ UMMA descriptors

// Shared-memory matrix descriptor (sm_100 format): start address, leading and stride
// byte offsets (all >> 4), descriptor version 1, base offset 0, 128-byte swizzle.
//  - K-major tiles (rows of 128 B along K, 8-row swizzle atoms of 1 KB): SBO = 1024,
//    LBO unused (16).
//  - MN-major tiles (rows of 128 B along M/N, one row per k): SBO = 1024 (8 k-rows),
//    LBO = byte distance between consecutive 64-element M/N atoms.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor for kind::f16 / kind::f8f6f4 with FP32 accumulation.
// fmt: kind::f16 -> 0 = F16, 1 = BF16; kind::f8f6f4 -> 0 = E4M3.
__host__ __device__ constexpr uint32_t idesc_f32acc(uint32_t a_fmt, uint32_t b_fmt, uint32_t a_mn,
                                                    uint32_t b_mn, uint32_t M, uint32_t N) {
  return (1u << 4) | (a_fmt << 7) | (b_fmt << 10) | (a_mn << 15) | (b_mn << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

// ------------------------------------------------------------------ tile scheduler

// Work of one launch: an (m_tiles x n_tiles) grid of output tiles, each needing
// kb_total K-blocks. Tiles [0, dp_tiles) (in rasterised order) go round-robin to the
// CTAs with their full K range; the remaining tiles form a flat space of
// sk_iters = (tiles - dp_tiles) * kb_total K-block iterations cut into num_ctas
// contiguous ranges (stream-K). A tile whose K range is cut is summed in fixed CTA
// order by whichever contributor finishes last, so results are deterministic.
// Partial tiles are stored as float4 units [col/4][row] (the TMEM lane is the row), so
// the 32 lanes of a warp write and read 512 contiguous bytes per instruction.
struct TileSched {
  int m_tiles, n_tiles, kb_total;
  int dp_tiles;
  int num_ctas;
  int group_m;
  long long sk_iters;
  int sk_ctas;  // CTAs 0 .. sk_ctas-1 share the stream-K range (<= num_ctas)
};

struct Seg {
  int tile;      // rasterised tile index
  int kb0, kb1;  // K-block range [kb0, kb1)
  int slot;      // 0 / 1: which workspace slot a partial result of this CTA goes to
};

__host__ __device__ inline long long sk_bound(const TileSched& s, int c) {
  return c >= s.sk_ctas ? s.sk_iters : (s.sk_iters * c) / s.sk_ctas;
}

// CTA owning stream-K iteration i.
__host__ __device__ inline int sk_owner(const TileSched& s, long long i) {
  int c = static_cast<int>((i * s.sk_ctas) / (s.sk_iters > 0 ? s.sk_iters : 1));
  if (c >= s.sk_ctas) c = s.sk_ctas - 1;
  while (c + 1 < s.sk_ctas && sk_bound(s, c + 1) <= i) ++c;
  while (c > 0 && sk_bound(s, c) > i) --c;
  return c;
}

// Rasterised tile index -> (m tile, n tile): groups of group_m tile-rows, walked down
// the rows of a group first, then across the columns, so CTAs running together share
// B columns and a small band of A rows in L2.
__host__ __device__ inline void tile_coords(const TileSched& s, int t, int& mt, int& nt) {
  const int per_group = s.group_m * s.n_tiles;
  const int g = t / per_group;
  const int first_m = g * s.group_m;
  int gm = s.m_tiles - first_m;
  if (gm > s.group_m) gm = s.group_m;
  const int r = t - g * per_group;
  mt = first_m + r % gm;
  nt = r / gm;
}

struct WorkIter {
  int dp_next;
  long long sk_begin, sk_pos, sk_end;

  __host__ __device__ void init(const TileSched& s, int cta) {
    dp_next = cta;
    sk_begin = sk_pos = sk_bound(s, cta);
    sk_end = sk_bound(s, cta + 1);
  }
  // Stream-K range first, then the data-parallel tiles: the fix-up of a split tile
  // (done by its last contributor's epilogue warps) then overlaps the MMAs of that
  // CTA's remaining tiles instead of landing in the kernel's tail. (Measured on the
  // 4096^3 and FFN shapes: with the pieces last instead, the fix-ups, all in the tail
  // at once, cost 5-13 us more per call.)
  __host__ __device__ bool next(const TileSched& s, Seg& out) {
    if (sk_pos < sk_end) {
      const long long t = sk_pos / s.kb_total;
      const int kb0 = static_cast<int>(sk_pos - t * s.kb_total);
      long long rem = sk_end - sk_pos;
      int kb1 = s.kb_total;
      if (rem < kb1 - kb0) kb1 = kb0 + static_cast<int>(rem);
      out.tile = s.dp_tiles + static_cast<int>(t);
      out.kb0 = kb0;
      out.kb1 = kb1;
      out.slot = (sk_pos == sk_begin) ? 0 : 1;
      sk_pos += kb1 - kb0;
      return true;
    }
    if (dp_next < s.dp_tiles) {
      out.tile = dp_next;
      out.kb0 = 0;
      out.kb1 = s.kb_total;
      out.slot = 0;
      dp_next += s.num_ctas;
      return true;
    }
    return false;
  }
};

// Arrival of one of the n contributors to a split tile on the tile's counter. A counter
// word holds the call's generation (upper 48 bits, a number the host draws afresh for
// every call, never 0) and the number of this call's arrivals (lower 16 bits); a word of
// another generation - left by an earlier call, or whatever a fresh workspace holds -
// counts as zero arrivals. So the workspace needs no zeroing before a call (the chance
// that a stale word carries the current generation is 2^-48). The last arrival resets the
// word to zero: a call replayed from a CUDA graph carries the generation it was captured
// with, and must find the counters of its previous run back at zero arrivals. Returns the
// number of earlier arrivals of this call, or -1 if the compare-and-swap kept failing (it
// cannot fail more often than there are contributors; the bound only keeps the loop
// finite).
__device__ __forceinline__ int counter_arrive(unsigned long long* c, unsigned long long gen, int n) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(c);
#pragma unroll 1
  for (int i = 0; i < 4096; ++i) {
    const bool same = (cur >> 16) == gen;
    const unsigned long long want = same ? cur + 1ull : ((gen << 16) | 1ull);
    const unsigned long long prev = atomicCAS(c, cur, want);
    if (prev == cur) {
      const int old = same ? static_cast<int>(cur & 0xffffull) : 0;
      if (old == n - 1) atomicExch(c, 0ull);  // every contributor has arrived
      return old;
    }
    cur = prev;
  }
  atomicOr(&g_error_word, kErrTimeout);  // reported by smgemm_check like an abandoned wait
  return -1;
}

// Partial-tile slot access for the TMEM lane `r` (tile row) and N consecutive columns
// starting at col0 (N and col0 multiples of 4): float4 units at [col/4][r], so a
// warp's 32 lanes touch 512 contiguous bytes per instruction.
template <int N>
__device__ __forceinline__ void slot_store(float* slot, int r, int col0, const float* v) {
  float4* s4 = reinterpret_cast<float4*>(slot);
#pragma unroll
  for (int q = 0; q < N / 4; ++q)
    s4[((col0 >> 2) + q) * 128 + r] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

template <int N>
__device__ __forceinline__ void slot_accumulate(const float* slot, int r, int col0, float* v) {
  const float4* s4 = reinterpret_cast<const float4*>(slot);
#pragma unroll
  for (int q = 0; q < N / 4; ++q) {
    const float4 t = __ldcg(s4 + ((col0 >> 2) + q) * 128 + r);
    v[4 * q] += t.x;
    v[4 * q + 1] += t.y;
    v[4 * q + 2] += t.z;
    v[4 * q + 3] += t.w;
  }
}

// v += slot0, then v += slot1 (the same additions, in the same order, as two
// slot_accumulate calls), with both slots' loads issued before the first add: a split
// tile's reduction waits for one L2 round trip per pair of contributors instead of one
// per contributor.
template <int N>
__device__ __forceinline__ void slot_accumulate2(const float* slot0, const float* slot1, int r, int col0, float* v) {
  const float4* a4 = reinterpret_cast<const float4*>(slot0);
  const float4* b4 = reinterpret_cast<const float4*>(slot1);
  float4 a[N / 4], b[N / 4];
#pragma unroll
  for (int q = 0; q < N / 4; ++q) a[q] = __ldcg(a4 + ((col0 >> 2) + q) * 128 + r);
#pragma unroll
  for (int q = 0; q < N / 4; ++q) b[q] = __ldcg(b4 + ((col0 >> 2) + q) * 128 + r);
#pragma unroll
  for (int q = 0; q < N / 4; ++q) {
    v[4 * q] += a[q].x;
    v[4 * q + 1] += a[q].y;
    v[4 * q + 2] += a[q].z;
    v[4 * q + 3] += a[q].w;
  }
#pragma unroll
  for (int q = 0; q < N / 4; ++q) {
    v[4 * q] += b[q].x;
    v[4 * q + 1] += b[q].y;
    v[4 * q + 2] += b[q].z;
    v[4 * q + 3] += b[q].w;
  }
}

// Sum, in contributor (= K) order, of the N columns col0.. of the partials of stream-K
// tile t_sk: slot_of(cc) gives contributor cc's slot, and own(v), when the calling CTA
// `self` is a contributor whose partial is still on chip (TMEM or registers), adds that
// partial in its place instead of reading it back. Slot loads are issued two
// contributors at a time.
template <int N, class SlotOf, class Own>
__device__ __forceinline__ void sk_tile_sum(const TileSched& s, long long t_sk, int self, SlotOf slot_of, Own own,
                                            int r, int col0, float* v) {
#pragma unroll
  for (int j = 0; j < N; ++j) v[j] = 0.0f;
  const int c_lo = sk_owner(s, t_sk * s.kb_total);
  const int c_hi = sk_owner(s, (t_sk + 1) * s.kb_total - 1);
  const float* pend = nullptr;
#pragma unroll 1
  for (int cc = c_lo; cc <= c_hi; ++cc) {
    if (!(sk_bound(s, cc) < sk_bound(s, cc + 1))) continue;
    if (cc == self) {
      if (pend != nullptr) slot_accumulate<N>(pend, r, col0, v);
      pend = nullptr;
      own(v);
      continue;
    }
    const float* src = slot_of(cc);
    if (pend == nullptr) {
      pend = src;
    } else {
      slot_accumulate2<N>(pend, src, r, col0, v);
      pend = nullptr;
    }
  }
  if (pend != nullptr) slot_accumulate<N>(pend, r, col0, v);
}

// The slot a contributor CTA `c` used for stream-K tile `t_sk` (index among the
// stream-K tiles): 0 if the tile holds the start of c's range, else 1.
__host__ __device__ inline int sk_slot_of(const TileSched& s, int c, long long t_sk) {
  const long long begin = sk_bound(s, c);
  return (begin / s.kb_total == t_sk) ? 0 : 1;
}

}  // namespace smg
