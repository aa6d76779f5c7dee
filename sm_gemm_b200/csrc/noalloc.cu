// gemm_bf16_noalloc: gemm_bf16 for callers that cannot allocate device memory.
//
// Some callers of a GEMM library own no device allocator: an inference-engine plugin
// or custom-op host that is handed only its input and output buffers, or a
// latency-critical decode loop where a cudaMalloc (which can synchronise the whole
// device) is not acceptable. gemm_bf16 needs caller-provided scratch for the partial
// tiles of its stream-K schedule; this entry point instead uses a fixed scratch array
// that lives in the library's own device image (a file-scope __device__ array), so
// the caller passes inputs and outputs only. The method's sources have no counterpart
// for this; it is a property of the library, not of the GEMM.
//
// Limits and behaviour:
//  - The scratch is kNoAllocScratchBytes (16 MiB) per GPU. Every GPU that loads this
//    library holds that array until the process exits.
//  - A call whose schedule needs more scratch than that is rejected with
//    SMGEMM_ERR_WORKSPACE before anything is enqueued.
//  - All calls share the one array, and it keeps the previous call's contents; nothing
//    in it needs clearing (the split tiles' arrival counters carry a per-call
//    generation, so words left by an earlier call never count). Calls that can overlap
//    on the GPU (different streams, different host threads) race on the array and must
//    not be issued concurrently.
//  - The first call on each device resolves the array's device address
//    (cudaGetSymbolAddress, with that device current). Under CUDA's default lazy
//    module loading that first call is also what loads the library's device code on
//    the device and reserves the array, which can take milliseconds and synchronise,
//    so make it during warm-up, outside any latency-critical loop and before any
//    stream capture.
//  - The address is cached per device together with the identity of the CUDA context
//    it was taken in; after cudaDeviceReset (a new primary context, the old address
//    invalid) the next call takes the address again, as a first call does.
//  - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/smgemm.h"

namespace {

constexpr size_t kNoAllocScratchBytes = SMGEMM_NOALLOC_SCRATCH_BYTES;
static_assert(kNoAllocScratchBytes == (16u << 20), "header and library disagree on the scratch size");

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

// Unique id of the calling thread's current CUDA context (0 if it cannot be told),
// through the driver's cuCtxGetCurrent / cuCtxGetId reached via the runtime's
// entry-point query, so the library still loads without a driver.
typedef CUresult (*PFN_ctxGetCurrent)(CUcontext*);
typedef CUresult (*PFN_ctxGetId)(CUcontext, unsigned long long*);

unsigned long long current_context_id() {
  static PFN_ctxGetCurrent get_current = nullptr;
  static PFN_ctxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_ctxGetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_ctxGetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device (host code must not use
// the symbol's name as an address: it is only a host-side stand-in for the array).
// Taken again whenever the current context is not the one the cached address came from.
smgemm_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SMGEMM_ERR_CUDA;
  }
  std::lock_guard<std::mutex> g(g_mu);
  const unsigned long long ctx = g_scratch_addr[dev] != nullptr ? current_context_id() : 0;
  if (g_scratch_addr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SMGEMM_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();  // the symbol query has made the context current
  }
  *out = g_scratch_addr[dev];
  return SMGEMM_OK;
}

}  // namespace

extern "C" smgemm_status gemm_bf16_noalloc(int64_t M, int64_t N, int64_t K, const void* A, smgemm_dtype ab_dtype,
                                           smgemm_layout layout_a, int64_t lda, const void* B,
                                           smgemm_layout layout_b, int64_t ldb, const void* bias,
                                           smgemm_dtype bias_dtype, smgemm_act act, void* C, smgemm_dtype c_dtype,
                                           int64_t ldc, smgemm_stream_t stream) {
  // gemm_bf16 checks the exact scratch need of its schedule against the size passed
  // and returns SMGEMM_ERR_WORKSPACE before enqueueing anything when it does not fit.
  void* scratch = nullptr;
  if (M > 0 && N > 0) {
    const smgemm_status st = scratch_address(&scratch);
    if (st != SMGEMM_OK) return st;
  }
  return gemm_bf16(M, N, K, A, ab_dtype, layout_a, lda, B, layout_b, ldb, bias, bias_dtype, act, C, c_dtype, ldc,
                   scratch, scratch != nullptr ? kNoAllocScratchBytes : 0, stream);
}
