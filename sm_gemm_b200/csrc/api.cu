// C-ABI of the GEMM library: argument validation, TMA descriptor encoding, schedule
// planning (tile grid, data-parallel / stream-K split, workspace) and dispatch to the
// sm_100a kernels. Declared in include/smgemm.h.
//
// The library links the CUDA runtime statically and reaches the one driver function it
// needs (cuTensorMapEncodeTiled) through the runtime's entry-point query, so the shared
// object loads on machines without a GPU driver; every entry point that needs the GPU
// fails with SMGEMM_ERR_CUDA there.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include <unistd.h>  // environ

#include <nvtx3/nvToolsExt.h>

#include "../../include/smgemm.h"
#include "grouped.h"
#include "kernels.h"

using namespace smg;

namespace {

// ------------------------------------------------------------------ environment switches

// The SMGEMM_* switches (tuning and test overrides), read in one pass over the
// environment when a call enters the library, instead of a separate scan of the whole
// environment for each of the dozen switches a GEMM call consults.
enum Knob {
  kKnobGrid, kKnobSched, kKnobSplitK, kKnobForceConfig, kKnobPair, kKnobForceLarge, kKnobGroupM, kKnobFp8Tn,
  kKnobLog, kKnobWaitLimitNs, kKnobEpiStore, kKnobGroupedSplit, kKnobPdl, kKnobGroupedTranspose, kKnobGroupedOrder,
  kNumKnobs
};
const char* const kKnobNames[kNumKnobs] = {
    "SMGEMM_GRID", "SMGEMM_SCHED", "SMGEMM_SPLITK", "SMGEMM_FORCE_CONFIG", "SMGEMM_PAIR", "SMGEMM_FORCE_LARGE",
    "SMGEMM_GROUP_M", "SMGEMM_FP8_TN", "SMGEMM_LOG", "SMGEMM_WAIT_LIMIT_NS", "SMGEMM_EPI_STORE",
    "SMGEMM_SCHED_GROUPED_SPLIT", "SMGEMM_PDL", "SMGEMM_GROUPED_TRANSPOSE", "SMGEMM_GROUPED_ORDER"};
thread_local const char* g_knobs[kNumKnobs] = {};

void refresh_knobs() {
  const char* k[kNumKnobs] = {};
  for (char** e = environ; e != nullptr && *e != nullptr; ++e) {
    const char* s = *e;
    if (std::strncmp(s, "SMGEMM_", 7) != 0) continue;
    const char* eq = std::strchr(s, '=');
    if (eq == nullptr) continue;
    const size_t n = static_cast<size_t>(eq - s);
    for (int i = 0; i < kNumKnobs; ++i) {
      if (std::strlen(kKnobNames[i]) == n && std::memcmp(kKnobNames[i], s, n) == 0) {
        k[i] = eq + 1;
        break;
      }
    }
  }
  for (int i = 0; i < kNumKnobs; ++i) g_knobs[i] = k[i];
}

const char* knob(Knob i) { return g_knobs[i]; }

// Every entry point that plans or launches work opens one: an NVTX range named after the
// entry point, so a profiler's timeline shows which library call enqueued which kernels
// (the profiling practice of "为什么我们要死磕GEMM" (kwkr.cn), section 7.1; without an
// attached tool a range costs one predictable branch, NVTX's header-only API), and a
// fresh snapshot of the SMGEMM_* switches for the call.
struct CallScope {
  explicit CallScope(const char* name) {
    nvtxRangePushA(name);
    refresh_knobs();
  }
  ~CallScope() { nvtxRangePop(); }
};

}  // namespace

namespace smg {
// Launch attribute switch of the kernel launchers (declared in sm100.cuh): programmatic
// dependent launch unless SMGEMM_PDL=0 when the current call entered the library.
bool pdl_enabled() {
  const char* v = knob(kKnobPdl);
  return !(v != nullptr && v[0] == '0');
}
}  // namespace smg

namespace {

// ------------------------------------------------------------------ driver entry point

typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                    CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

PFN_encodeTiled encode_fn() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  });
  return fn;
}

// ------------------------------------------------------------------ device info

struct DevInfo {
  bool ok = false;
  int sms = 0;
};

smgemm_status current_device(DevInfo& out) {
  static std::mutex mu;
  static DevInfo cache[64];
  static bool filled[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return SMGEMM_ERR_CUDA;
  }
  std::lock_guard<std::mutex> g(mu);
  if (!filled[dev]) {
    cudaDeviceProp prop;
    DevInfo d;
    if (cudaGetDeviceProperties(&prop, dev) == cudaSuccess) {
      d.ok = (prop.major == 10 && prop.minor == 0);
      d.sms = prop.multiProcessorCount;
    } else {
      cudaGetLastError();
    }
    cache[dev] = d;
    filled[dev] = true;
  }
  out = cache[dev];
  return out.ok ? SMGEMM_OK : SMGEMM_ERR_CUDA;
}

// ------------------------------------------------------------------ config / logging

thread_local char g_last_config[256] = "none";

// The plan of the last GEMM call on this thread, formatted into g_last_config only when
// asked for (smgemm_last_config, SMGEMM_LOG): formatting it on every call cost ~0.5 us of
// host time per call, a tenth of a small GEMM's.
struct PendingConfig {
  bool pending = false;
  const char* path = "";
  int mma_n = 0, m_tiles = 0, n_tiles = 0, kb_total = 0, grid = 0, dp_tiles = 0, sk_ctas = 0;
  long long sk_iters = 0;
  size_t ws = 0;
};
thread_local PendingConfig g_pending;

void format_pending_config() {
  if (!g_pending.pending) return;
  const PendingConfig& c = g_pending;
  std::snprintf(g_last_config, sizeof(g_last_config),
                "path=%s tile=128x%d tiles=%dx%d kb=%d grid=%d dp_tiles=%d sk_iters=%lld sk_ctas=%d ws=%zu", c.path,
                c.mma_n, c.m_tiles, c.n_tiles, c.kb_total, c.grid, c.dp_tiles, c.sk_iters, c.sk_ctas, c.ws);
  g_pending.pending = false;
}

// The buffer for a configuration string written directly (replaces a pending plan).
char* config_text() {
  g_pending.pending = false;
  return g_last_config;
}

long long env_ll(Knob name, long long dflt) {
  const char* v = knob(name);
  if (v == nullptr || *v == 0) return dflt;
  return std::atoll(v);
}

enum class SchedMode { kAuto, kDP, kSK };

SchedMode sched_mode() {
  const char* v = knob(kKnobSched);
  if (v == nullptr) return SchedMode::kAuto;
  if (std::strcmp(v, "dp") == 0) return SchedMode::kDP;
  if (std::strcmp(v, "sk") == 0) return SchedMode::kSK;
  return SchedMode::kAuto;
}

// SMGEMM_FORCE_CONFIG picks the kernel family instead of the heuristics, for tuning and
// tests: "pair" (256 x 256 tiles on CTA pairs), "single" (one-SM large tiles), "large"
// (no swap-AB path for small M; pair or single as usual), "pair128" (FP8: 256 x 128
// pair tiles). Unknown or empty values leave the heuristics in charge. The older
// switches SMGEMM_PAIR=0, SMGEMM_FORCE_LARGE=1 and SMGEMM_FP8_TN=128 mean "single",
// "large" and "pair128".
bool force_config_is(const char* want) {
  const char* v = knob(kKnobForceConfig);
  return v != nullptr && std::strcmp(v, want) == 0;
}

// Tile-grid plan over T output tiles and P persistent CTAs (or CTA pairs).
//  - auto: whole waves of tiles run data-parallel; the R = T mod P tiles of a ragged
//    last wave are split along K into s = min(P / R, KB / 8) equal pieces that run
//    side by side (one piece per CTA), so the last wave takes 1/s of a tile instead of
//    a whole one. Pieces of tiles that share operands start at the same K offsets, so
//    L2 reuse is kept (a free-running stream-K range would scatter the CTAs that share
//    a B column block across K and re-stream it from HBM). The pages' concern this
//    addresses: small or ragged shapes leave SMs idle ("为什么我们要死磕GEMM",
//    kwkr.cn, section 3.3).
//  - SMGEMM_SCHED=dp: data-parallel only; SMGEMM_SCHED=sk: every tile in one stream-K
//    range over all CTAs (kept for tests).
struct Plan {
  TileSched s;
  int grid = 0;
  size_t counter_bytes = 0;
  size_t slot_bytes = 0;  // all slots
  size_t ws_bytes() const { return counter_bytes + slot_bytes; }
};

// Schedule choices measured per shape by an offline sweep (sm_gemm_b200/tune.py, the
// tuning-to-a-static-table practice of the DeepGEMM kernel-library walkthrough (zwxr.cn),
// section 5.2). A listed shape takes its group_m and split-K choice from the table;
// SMGEMM_GROUP_M and SMGEMM_SPLITK still override both.
struct TunedConfig {
  int kind;
  long long M, N, K;
  int layout_a, group_m, splitk;
};
constexpr TunedConfig kTuned[] = {
#include "tuned_configs.inc"
    {-1, 0, 0, 0, 0, 0, 0}};

const TunedConfig* find_tuned(int kind, int64_t M, int64_t N, int64_t K, int layout_a) {
  for (const TunedConfig& t : kTuned)
    if (t.kind == kind && t.M == M && t.N == N && t.K == K && t.layout_a == layout_a) return &t;
  return nullptr;
}

Plan make_plan(int m_tiles, int n_tiles, int kb_total, int sms, int group_m, size_t slot_floats,
               int counters_per_tile = 1, long long splitk_default = 0) {
  Plan pl;
  const long long T = static_cast<long long>(m_tiles) * n_tiles;
  long long max_ctas = env_ll(kKnobGrid, sms);
  if (max_ctas < 1) max_ctas = 1;
  if (max_ctas > sms) max_ctas = sms;
  SchedMode mode = sched_mode();
  constexpr int kMinItersPerPiece = 8;
  // SMGEMM_SPLITK=s: 1 = every tile whole (data-parallel only); s >= 2 = every tile's K
  // range cut into about s pieces (one stream-K range over min(P, s T) CTAs).
  const long long splitk = env_ll(kKnobSplitK, splitk_default);
  if (splitk == 1) mode = SchedMode::kDP;

  long long dp = T, sk_iters = 0, sk_ctas = 0, grid = std::min<long long>(T, max_ctas);
  if (splitk >= 2) {
    dp = 0;
    sk_iters = T * kb_total;
    grid = sk_ctas = std::min<long long>(std::min<long long>(max_ctas, T * splitk), sk_iters);
  } else if (mode == SchedMode::kSK) {
    dp = 0;
    sk_iters = T * kb_total;
    grid = sk_ctas = std::min<long long>(max_ctas, sk_iters);
  } else if (mode == SchedMode::kAuto) {
    const long long waves = T / max_ctas, R = T % max_ctas;
    long long split = R > 0 ? std::min<long long>(max_ctas / R, kb_total / kMinItersPerPiece) : 1;
    if (split >= 2) {
      dp = waves * max_ctas;
      sk_iters = R * kb_total;
      sk_ctas = R * split;
      grid = waves > 0 ? max_ctas : sk_ctas;
    }
  }
  pl.s.m_tiles = m_tiles;
  pl.s.n_tiles = n_tiles;
  pl.s.kb_total = kb_total;
  pl.s.dp_tiles = static_cast<int>(dp);
  pl.s.num_ctas = static_cast<int>(grid);
  pl.s.group_m = std::max(1, std::min(group_m, m_tiles));
  pl.s.sk_iters = sk_iters;
  pl.s.sk_ctas = static_cast<int>(sk_iters > 0 ? sk_ctas : grid);
  pl.grid = static_cast<int>(grid);
  if (sk_iters > 0) {
    pl.counter_bytes =
        ((static_cast<size_t>(T - dp) * counters_per_tile * sizeof(unsigned long long)) + 255) / 256 * 256;
    pl.slot_bytes = static_cast<size_t>(sk_ctas) * 2 * slot_floats * sizeof(float);
  }
  return pl;
}

// ------------------------------------------------------------------ TMA maps

// A tensor map is a pure function of its arguments (it holds the global address, not a
// handle to the allocation), so encoded maps are kept per host thread, keyed by every
// argument, and a call on the same operand as a recent call reuses its map instead of
// encoding it again (the shape -> descriptor cache of the DeepGEMM kernel-library
// walkthrough (zwxr.cn), section 4.3). A stale entry for memory freed and reallocated at
// the same address is still exactly the map an encode would produce.
struct MapKey {
  const void* base;
  uint64_t inner, outer, stride;
  uint32_t box_inner, box_outer;
  int dt, swizzle;
  bool operator==(const MapKey& o) const {
    return base == o.base && inner == o.inner && outer == o.outer && stride == o.stride &&
           box_inner == o.box_inner && box_outer == o.box_outer && dt == o.dt && swizzle == o.swizzle;
  }
};

struct MapCache {
  static constexpr int kEntries = 32;
  MapKey key[kEntries];
  CUtensorMap map[kEntries];
  bool used[kEntries] = {};
  int next = 0;
};

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
               uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  thread_local MapCache cache;
  const MapKey k{base, inner, outer, row_stride_bytes, box_inner, box_outer, static_cast<int>(dt),
                 static_cast<int>(swizzle)};
  for (int i = 0; i < MapCache::kEntries; ++i) {
    if (cache.used[i] && cache.key[i] == k) {
      *map = cache.map[i];
      return true;
    }
  }
  PFN_encodeTiled fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const int slot = cache.next;
  cache.next = (cache.next + 1) % MapCache::kEntries;
  cache.key[slot] = k;
  cache.map[slot] = *map;
  cache.used[slot] = true;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(int dt) { return dt == kF32 ? 4 : (dt == kE4M3 ? 1 : 2); }

bool valid_out_dtype(int dt) { return dt == kF32 || dt == kBF16 || dt == kF16; }
bool valid_bias_dtype(int dt) { return dt == kF32 || dt == kBF16 || dt == kF16; }
bool valid_act(int a) { return a == kActNone || a == kActGeluTanh || a == kActSilu; }
bool valid_layout(int l) { return l == SMGEMM_ROW_MAJOR || l == SMGEMM_COL_MAJOR; }

smgemm_status check_output(int64_t M, int64_t N, const void* C, int c_dtype, int64_t ldc, const void* bias,
                           int bias_dtype, int act) {
  if (!valid_out_dtype(c_dtype) || !valid_act(act)) return SMGEMM_ERR_INVALID_ARG;
  if (bias != nullptr && !valid_bias_dtype(bias_dtype)) return SMGEMM_ERR_INVALID_ARG;
  if (C == nullptr || ldc < N) return SMGEMM_ERR_INVALID_ARG;
  if (!aligned16(C) || (ldc * elem_size(c_dtype)) % 16 != 0) return SMGEMM_ERR_ALIGNMENT;
  if (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) % elem_size(bias_dtype)) != 0)
    return SMGEMM_ERR_ALIGNMENT;
  (void)M;
  return SMGEMM_OK;
}

bool fits_int(int64_t v) { return v >= 0 && v <= 0x7FFFFFFF; }

smgemm_status launch_status(cudaError_t e) {
  if (e == cudaSuccess) return SMGEMM_OK;
  cudaGetLastError();
  return SMGEMM_ERR_CUDA;
}

// ------------------------------------------------------------------ 16-bit GEMM plan

struct Gemm16Plan {
  Tc16Variant v;
  bool skinny;
  bool pair;  // large tiles on CTA pairs (256 x 256 per cluster)
  Plan pl;
  int mma_n, bk;
};

// Large tiles run on CTA pairs unless SMGEMM_PAIR=0 or the device reports no
// co-resident pair clusters; `sms` is then the SM count and `pair_clusters` the number
// of co-resident clusters of two.
Gemm16Plan plan_gemm16(int64_t M, int64_t N, int64_t K, int layout_a, int sms, int pair_clusters,
                       bool allow_skinny = true) {
  Gemm16Plan g;
  const bool force_single = force_config_is("single") || env_ll(kKnobPair, 1) == 0;
  const bool force_large = env_ll(kKnobForceLarge, 0) != 0 || !allow_skinny || force_config_is("large") ||
                           force_config_is("pair") || force_single;
  g.skinny = (M <= 64 && layout_a == SMGEMM_ROW_MAJOR && !force_large);
  g.pair = !g.skinny && pair_clusters > 0 && !force_single;
  if (g.skinny) g.v = M <= 16 ? Tc16Variant::kSkinny16 : (M <= 32 ? Tc16Variant::kSkinny32 : Tc16Variant::kSkinny64);
  else g.v = Tc16Variant::kLarge;
  g.mma_n = tc16_mma_n(g.v);
  g.bk = g.pair ? tc16_pair_bk() : tc16_bk(g.v);
  const int kb = static_cast<int>((K + g.bk - 1) / g.bk);
  const TunedConfig* t = g.pair ? find_tuned(0, M, N, K, layout_a) : nullptr;
  const int group_m = static_cast<int>(env_ll(kKnobGroupM, t != nullptr ? t->group_m : 8));
  if (g.pair) {
    g.pl = make_plan(static_cast<int>((M + 255) / 256), static_cast<int>((N + 255) / 256), std::max(kb, 1),
                     pair_clusters, group_m, static_cast<size_t>(2) * 128 * 256, 2, t != nullptr ? t->splitk : 0);
    return g;
  }
  int m_tiles, n_tiles;
  if (g.skinny) {
    m_tiles = static_cast<int>((N + 127) / 128);  // MMA rows run over the output columns
    n_tiles = 1;
  } else {
    m_tiles = static_cast<int>((M + 127) / 128);
    n_tiles = static_cast<int>((N + g.mma_n - 1) / g.mma_n);
  }
  g.pl = make_plan(m_tiles, n_tiles, std::max(kb, 1), sms, group_m, static_cast<size_t>(128) * g.mma_n);
  return g;
}

// FP8 tiles run on CTA pairs (256 x tn) unless SMGEMM_PAIR=0 or no pair cluster fits.
struct Fp8Plan {
  bool pair;
  int tn;  // pair tile width: 256 or 128
  Plan pl;
};

int fp8_tile_n() { return (env_ll(kKnobFp8Tn, 256) == 128 || force_config_is("pair128")) ? 128 : 256; }

Fp8Plan plan_fp8(int64_t M, int64_t N, int64_t K, int sms, int tn, int pair_clusters) {
  Fp8Plan f;
  const int kb = static_cast<int>((K + kFp8BK - 1) / kFp8BK);
  f.pair = pair_clusters > 0 && env_ll(kKnobPair, 1) != 0 && !force_config_is("single");
  f.tn = tn;
  const TunedConfig* t = f.pair && tn == 256 ? find_tuned(1, M, N, K, SMGEMM_ROW_MAJOR) : nullptr;
  const int group_m = static_cast<int>(env_ll(kKnobGroupM, t != nullptr ? t->group_m : 8));
  if (f.pair) {
    f.pl = make_plan(static_cast<int>((M + 255) / 256), static_cast<int>((N + tn - 1) / tn), std::max(kb, 1),
                     pair_clusters, group_m, static_cast<size_t>(2) * 128 * tn, 2, t != nullptr ? t->splitk : 0);
  } else {
    f.pl = make_plan(static_cast<int>((M + kFp8BM - 1) / kFp8BM), static_cast<int>((N + kFp8BN - 1) / kFp8BN),
                     std::max(kb, 1), sms, group_m, static_cast<size_t>(kFp8BM) * kFp8BN);
  }
  return f;
}

// Generation of a call's split-tile counters: a fresh 48-bit number per call (never 0),
// starting from a value drawn from the clock, so counters left by earlier calls (or the
// contents of a fresh workspace) never read as this call's arrivals and the workspace
// needs no zeroing - one stream operation less per call.
unsigned long long next_generation() {
  static std::atomic<unsigned long long> counter{[] {
    unsigned long long z = static_cast<unsigned long long>(
                               std::chrono::steady_clock::now().time_since_epoch().count()) +
                           0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;  // splitmix64 finaliser (Steele, Lea, Flood)
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }()};
  unsigned long long g;
  do {
    g = counter.fetch_add(1, std::memory_order_relaxed) & 0xFFFFFFFFFFFFull;
  } while (g == 0);
  return g;
}

smgemm_status prepare_workspace(const Plan& pl, void* ws, size_t ws_bytes, float** slots,
                                unsigned long long** counters, unsigned long long* gen) {
  *slots = nullptr;
  *counters = nullptr;
  *gen = 0;
  if (pl.ws_bytes() == 0) return SMGEMM_OK;
  if (ws == nullptr || ws_bytes < pl.ws_bytes()) return SMGEMM_ERR_WORKSPACE;
  if (!aligned16(ws)) return SMGEMM_ERR_ALIGNMENT;
  *counters = static_cast<unsigned long long*>(ws);
  *slots = reinterpret_cast<float*>(static_cast<char*>(ws) + pl.counter_bytes);
  *gen = next_generation();
  return SMGEMM_OK;
}

void note_config(const char* path, const Plan& pl, int mma_n) {
  g_pending.pending = true;
  g_pending.path = path;  // string literals
  g_pending.mma_n = mma_n;
  g_pending.m_tiles = pl.s.m_tiles;
  g_pending.n_tiles = pl.s.n_tiles;
  g_pending.kb_total = pl.s.kb_total;
  g_pending.grid = pl.grid;
  g_pending.dp_tiles = pl.s.dp_tiles;
  g_pending.sk_iters = pl.s.sk_iters;
  g_pending.sk_ctas = pl.s.sk_ctas;
  g_pending.ws = pl.ws_bytes();
  if (env_ll(kKnobLog, 0)) {
    format_pending_config();
    std::fprintf(stderr, "[smgemm] %s\n", g_last_config);
  }
}

// Limit of the kernels' bounded barrier waits, in SM cycles.
unsigned long long wait_limit() {
  return kCyclesPerNs *
         static_cast<unsigned long long>(env_ll(kKnobWaitLimitNs, static_cast<long long>(kWaitLimitNs)));
}

}  // namespace

extern "C" {

const char* smgemm_status_string(smgemm_status st) {
  switch (st) {
    case SMGEMM_OK: return "ok";
    case SMGEMM_ERR_INVALID_ARG: return "invalid argument";
    case SMGEMM_ERR_UNSUPPORTED: return "unsupported combination";
    case SMGEMM_ERR_ALIGNMENT: return "misaligned pointer or leading dimension (TMA needs 16 bytes)";
    case SMGEMM_ERR_WORKSPACE: return "workspace missing or too small";
    case SMGEMM_ERR_CUDA: return "CUDA error or no sm_100 device";
    case SMGEMM_ERR_TIMEOUT: return "kernel abandoned a barrier wait";
  }
  return "unknown status";
}

const char* smgemm_last_config(void) {
  format_pending_config();
  return g_last_config;
}

size_t smgemm_workspace_size(int64_t M, int64_t N, int64_t K, int kind) {
  refresh_knobs();  // the plan, hence the size, follows the SMGEMM_* switches
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  DevInfo d;
  if (current_device(d) != SMGEMM_OK) return 0;
  if (kind == 1) return plan_fp8(M, N, K, d.sms, fp8_tile_n(), fp8_pair_max_clusters(fp8_tile_n())).pl.ws_bytes();
  // enough for either path (the skinny path is only taken for a row-major A)
  const int pc = tc16_pair_max_clusters();
  return std::max(plan_gemm16(M, N, K, SMGEMM_ROW_MAJOR, d.sms, pc).pl.ws_bytes(),
                  plan_gemm16(M, N, K, SMGEMM_COL_MAJOR, d.sms, pc).pl.ws_bytes());
}

}  // extern "C"

namespace {
// gemm_bf16 with, on the swap-AB path, the log-softmax tile partials written to
// lse_part (nullable; see Tc16Params). *used_partials tells whether they were.
smgemm_status gemm16_impl(int64_t M, int64_t N, int64_t K, const void* A, smgemm_dtype ab_dtype,
                          smgemm_layout layout_a, int64_t lda, const void* B, smgemm_layout layout_b, int64_t ldb,
                          const void* bias, smgemm_dtype bias_dtype, smgemm_act act, void* C, smgemm_dtype c_dtype,
                          int64_t ldc, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                          float2* lse_part, bool* used_partials, float* fp8_scales = nullptr) {
  if (used_partials != nullptr) *used_partials = false;
  const bool fp8_out = fp8_scales != nullptr;  // c_dtype E4M3: codes + 1x128 scales
  if (!fits_int(M) || !fits_int(N) || !fits_int(K)) return SMGEMM_ERR_INVALID_ARG;
  if (ab_dtype != SMGEMM_BF16 && ab_dtype != SMGEMM_F16) return SMGEMM_ERR_UNSUPPORTED;
  if (!valid_layout(layout_a) || !valid_layout(layout_b)) return SMGEMM_ERR_INVALID_ARG;
  if ((fp8_out ? c_dtype != SMGEMM_E4M3 : !valid_out_dtype(c_dtype)) || !valid_act(act)) return SMGEMM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return SMGEMM_OK;
  smgemm_status st = SMGEMM_OK;
  if (fp8_out) {
    if (!valid_act(act) || (bias != nullptr && !valid_bias_dtype(bias_dtype))) return SMGEMM_ERR_INVALID_ARG;
    if (C == nullptr || ldc < N) return SMGEMM_ERR_INVALID_ARG;
    if (!aligned16(C) || ldc % 16 != 0 || (reinterpret_cast<uintptr_t>(fp8_scales) & 3u)) return SMGEMM_ERR_ALIGNMENT;
    if (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) % elem_size(bias_dtype)) != 0)
      return SMGEMM_ERR_ALIGNMENT;
    if (K == 0) return SMGEMM_ERR_UNSUPPORTED;
  } else {
    st = check_output(M, N, C, c_dtype, ldc, bias, bias_dtype, act);
    if (st != SMGEMM_OK) return st;
  }
  if (K > 0) {
    if (A == nullptr || B == nullptr) return SMGEMM_ERR_INVALID_ARG;
    if (lda < (layout_a == SMGEMM_ROW_MAJOR ? K : M) || ldb < (layout_b == SMGEMM_ROW_MAJOR ? N : K))
      return SMGEMM_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || (lda * 2) % 16 != 0 || (ldb * 2) % 16 != 0) return SMGEMM_ERR_ALIGNMENT;
  }
  DevInfo d;
  if (current_device(d) != SMGEMM_OK) return SMGEMM_ERR_CUDA;
  if (K == 0) {
    std::snprintf(config_text(), sizeof(g_last_config), "path=fill");
    return launch_status(launch_fill_epilogue(static_cast<int>(M), static_cast<int>(N), bias, bias_dtype, act, C,
                                              c_dtype, ldc, stream));
  }
  const Gemm16Plan g = plan_gemm16(M, N, K, layout_a, d.sms, tc16_pair_max_clusters(), !fp8_out);
  if (fp8_out && !g.pair) return SMGEMM_ERR_UNSUPPORTED;  // the FP8 epilogue runs on the CTA-pair kernel
  const CUtensorMapDataType dt =
      ab_dtype == SMGEMM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const uint32_t fmt = ab_dtype == SMGEMM_BF16 ? 1u : 0u;
  CUtensorMap tm_a, tm_b;
  Tc16Params p{};
  bool ok;
  if (g.skinny) {
    // MMA "A" = the weight B (128 output columns per tile), MMA "B" = the tokens A.
    const bool w_mn = (layout_b == SMGEMM_ROW_MAJOR);
    if (w_mn) ok = encode_2d(&tm_a, dt, B, N, K, ldb * 2, 64, g.bk);
    else ok = encode_2d(&tm_a, dt, B, K, N, ldb * 2, 64, 128);
    ok = ok && encode_2d(&tm_b, dt, A, K, M, lda * 2, 64, g.mma_n);
    p.a_mn_major = w_mn ? 1 : 0;
    p.b_mn_major = 0;
    p.idesc = idesc_f32acc(fmt, fmt, w_mn ? 1u : 0u, 0u, 128, g.mma_n);
  } else {
    const bool a_mn = (layout_a == SMGEMM_COL_MAJOR);
    const bool b_mn = (layout_b == SMGEMM_ROW_MAJOR);
    // Each CTA loads 128 rows of A; B tiles are 256 columns (one-SM kernel) or 128 (each
    // CTA of a pair).
    const uint32_t b_rows = g.pair ? 128 : 256;
    if (a_mn) ok = encode_2d(&tm_a, dt, A, M, K, lda * 2, 64, g.bk);
    else ok = encode_2d(&tm_a, dt, A, K, M, lda * 2, 64, 128);
    if (b_mn) ok = ok && encode_2d(&tm_b, dt, B, N, K, ldb * 2, 64, g.bk);
    else ok = ok && encode_2d(&tm_b, dt, B, K, N, ldb * 2, 64, b_rows);
    p.a_mn_major = a_mn ? 1 : 0;
    p.b_mn_major = b_mn ? 1 : 0;
    p.idesc = idesc_f32acc(fmt, fmt, a_mn ? 1u : 0u, b_mn ? 1u : 0u, g.pair ? 256 : 128, 256);
  }
  if (!ok) return SMGEMM_ERR_CUDA;
  p.s = g.pl.s;
  p.e = EpiArgs{static_cast<int>(M), static_cast<int>(N), bias, bias_dtype, act, C, c_dtype, ldc, fp8_scales};
  p.wait_limit_cycles = wait_limit();
  p.lse_part = g.skinny ? lse_part : nullptr;
  if (used_partials != nullptr) *used_partials = p.lse_part != nullptr;
  st = prepare_workspace(g.pl, workspace, workspace_bytes, &p.slots, &p.counters, &p.gen);
  if (st != SMGEMM_OK) return st;
  if (g.pair) {
    // C leaves through TMA tile stores (32 x 32 boxes staged in shared memory), measured
    // slightly faster than 16-byte stores from registers (square BF16 4096^3: 97.5 vs
    // 98.7 us); SMGEMM_EPI_STORE=direct selects the register stores. Only when a row of
    // C is a whole number of 16-byte units: a box that ends past N in a partial unit was
    // seen to write the rest of that unit (the columns just right of C) on B200.
    CUtensorMap tm_c;
    const CUtensorMap* pc = nullptr;
    const char* es = knob(kKnobEpiStore);
    if (!fp8_out && (N * elem_size(c_dtype)) % 16 == 0 && !(es != nullptr && std::strcmp(es, "direct") == 0)) {
      const CUtensorMapDataType cdt = c_dtype == SMGEMM_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                      : c_dtype == SMGEMM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                               : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
      if (!encode_2d(&tm_c, cdt, C, N, M, ldc * elem_size(c_dtype), 32, 32,
                     c_dtype == SMGEMM_F32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
        return SMGEMM_ERR_CUDA;
      pc = &tm_c;
    }
    note_config(pc != nullptr ? "pair-tmastore" : "pair", g.pl, 256);
    return launch_status(launch_gemm_tc16_pair(tm_a, tm_b, pc, p, g.pl.grid, stream));
  }
  note_config(g.skinny ? "skinny" : "large", g.pl, g.mma_n);
  return launch_status(launch_gemm_tc16(tm_a, tm_b, p, g.v, g.pl.grid, stream));
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }
}  // namespace

extern "C" {

smgemm_status gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, smgemm_dtype ab_dtype,
                        smgemm_layout layout_a, int64_t lda, const void* B, smgemm_layout layout_b, int64_t ldb,
                        const void* bias, smgemm_dtype bias_dtype, smgemm_act act, void* C, smgemm_dtype c_dtype,
                        int64_t ldc, void* workspace, size_t workspace_bytes, smgemm_stream_t stream) {
  const CallScope scope("smgemm:gemm_bf16");
  return gemm16_impl(M, N, K, A, ab_dtype, layout_a, lda, B, layout_b, ldb, bias, bias_dtype, act, C, c_dtype, ldc,
                     workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr);
}

smgemm_status gemm_bf16_fp8out(int64_t M, int64_t N, int64_t K, const void* A, smgemm_dtype ab_dtype,
                               smgemm_layout layout_a, int64_t lda, const void* B, smgemm_layout layout_b, int64_t ldb,
                               const void* bias, smgemm_dtype bias_dtype, smgemm_act act, uint8_t* Cq, int64_t ldc,
                               float* scales, void* workspace, size_t workspace_bytes, smgemm_stream_t stream) {
  const CallScope scope("smgemm:gemm_bf16_fp8out");
  if (scales == nullptr) return SMGEMM_ERR_INVALID_ARG;
  return gemm16_impl(M, N, K, A, ab_dtype, layout_a, lda, B, layout_b, ldb, bias, bias_dtype, act, Cq, SMGEMM_E4M3,
                     ldc, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, scales);
}

size_t smgemm_logsoftmax_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0) return 0;
  return align256(smgemm_workspace_size(M, N, K, 0)) + align256(static_cast<size_t>(M) * sizeof(float)) +
         align256(static_cast<size_t>((N + 127) / 128) * static_cast<size_t>(M) * sizeof(float2));
}

smgemm_status gemm_bf16_logsoftmax(int64_t M, int64_t N, int64_t K, const void* A, smgemm_dtype ab_dtype,
                                   smgemm_layout layout_a, int64_t lda, const void* B, smgemm_layout layout_b,
                                   int64_t ldb, const void* bias, smgemm_dtype bias_dtype, float* C, int64_t ldc,
                                   void* workspace, size_t workspace_bytes, smgemm_stream_t stream_) {
  const CallScope scope("smgemm:gemm_bf16_logsoftmax");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (M < 0 || N < 0 || K < 0) return SMGEMM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return SMGEMM_OK;
  const size_t need = smgemm_logsoftmax_workspace_size(M, N, K);
  if (need == 0) return SMGEMM_ERR_CUDA;  // no usable device
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return SMGEMM_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t gemm_ws = align256(smgemm_workspace_size(M, N, K, 0));
  float* lse = reinterpret_cast<float*>(ws + gemm_ws);
  float2* part = reinterpret_cast<float2*>(ws + gemm_ws + align256(static_cast<size_t>(M) * sizeof(float)));
  bool used = false;
  smgemm_status st = gemm16_impl(M, N, K, A, ab_dtype, layout_a, lda, B, layout_b, ldb, bias, bias_dtype,
                                 SMGEMM_ACT_NONE, C, SMGEMM_F32, ldc, ws, gemm_ws, stream, part, &used);
  if (st != SMGEMM_OK) return st;
  DevInfo d;
  if (current_device(d) != SMGEMM_OK) return SMGEMM_ERR_CUDA;
  return launch_status(launch_log_softmax_rows(C, ldc, static_cast<int>(M), static_cast<int>(N),
                                               used ? part : nullptr, static_cast<int>((N + 127) / 128), lse, d.sms,
                                               stream));
}

smgemm_status gemm_bf16_lse_partials(int64_t M, int64_t N, int64_t K, const void* A, smgemm_dtype ab_dtype,
                                     smgemm_layout layout_a, int64_t lda, const void* B, smgemm_layout layout_b,
                                     int64_t ldb, const void* bias, smgemm_dtype bias_dtype, float* C, int64_t ldc,
                                     float* part, void* workspace, size_t workspace_bytes, smgemm_stream_t stream_) {
  const CallScope scope("smgemm:gemm_bf16_lse_partials");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (M < 0 || N < 0 || K < 0) return SMGEMM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return SMGEMM_OK;
  if (part == nullptr) return SMGEMM_ERR_INVALID_ARG;
  if (!aligned16(part)) return SMGEMM_ERR_ALIGNMENT;
  bool used = false;
  smgemm_status st = gemm16_impl(M, N, K, A, ab_dtype, layout_a, lda, B, layout_b, ldb, bias, bias_dtype,
                                 SMGEMM_ACT_NONE, C, SMGEMM_F32, ldc, workspace, workspace_bytes, stream,
                                 reinterpret_cast<float2*>(part), &used);
  if (st != SMGEMM_OK || used) return st;
  // Large-tile path (or K = 0): the partials come from the logits just written.
  return launch_status(launch_lse_tile_partials(C, ldc, static_cast<int>(M), static_cast<int>(N),
                                                reinterpret_cast<float2*>(part), stream));
}

smgemm_status logsoftmax_apply_partials(float* C, int64_t ldc, int64_t M, int64_t N, const float* part,
                                        int64_t n_parts, float* lse, smgemm_stream_t stream_) {
  const CallScope scope("smgemm:logsoftmax_apply_partials");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (M < 0 || N < 0 || n_parts < 0 || !fits_int(M) || !fits_int(N) || !fits_int(n_parts))
    return SMGEMM_ERR_INVALID_ARG;
  if (M == 0) return SMGEMM_OK;
  if (part == nullptr || lse == nullptr || n_parts == 0 || (N > 0 && (C == nullptr || ldc < N)))
    return SMGEMM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(part) & 7u) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (N > 0 && !aligned16(C)))
    return SMGEMM_ERR_ALIGNMENT;
  DevInfo d;
  if (current_device(d) != SMGEMM_OK) return SMGEMM_ERR_CUDA;
  return launch_status(launch_log_softmax_rows(C, ldc, static_cast<int>(M), static_cast<int>(N),
                                               reinterpret_cast<const float2*>(part), static_cast<int>(n_parts), lse,
                                               d.sms, stream));
}

// Group table, then (when the device is known) room for splitting a ragged last wave:
// one 2 x 128 x 256-float partial per cluster and two counters per split tile.
size_t grouped_table_bytes(int G) { return (static_cast<size_t>(G) * sizeof(GroupDesc) + 64 + 255) / 256 * 256; }
size_t grouped_split_bytes(int clusters) {
  return static_cast<size_t>(clusters) * 2 * 128 * 256 * sizeof(float) +
         static_cast<size_t>(clusters) * 2 * sizeof(unsigned long long);
}

size_t smgemm_grouped_workspace_size(int G) {
  refresh_knobs();
  if (G <= 0) return 0;
  DevInfo d;
  const int P = current_device(d) == SMGEMM_OK ? grouped_max_clusters() : 0;
  return grouped_table_bytes(G) + (P > 0 ? grouped_split_bytes(P) : 0);
}

smgemm_status gemm_bf16_grouped(int G, const int64_t* M, const int64_t* N, const int64_t* K, const void* const* A,
                                smgemm_dtype ab_dtype, smgemm_layout layout_a, const int64_t* lda,
                                const void* const* B, smgemm_layout layout_b, const int64_t* ldb,
                                const void* const* bias, smgemm_dtype bias_dtype, smgemm_act act, void* const* C,
                                smgemm_dtype c_dtype, const int64_t* ldc, void* workspace, size_t workspace_bytes,
                                smgemm_stream_t stream_) {
  const CallScope scope("smgemm:gemm_bf16_grouped");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (G < 0 || (G > 0 && (M == nullptr || N == nullptr || K == nullptr || A == nullptr || lda == nullptr ||
                          B == nullptr || ldb == nullptr || C == nullptr || ldc == nullptr)))
    return SMGEMM_ERR_INVALID_ARG;
  if (ab_dtype != SMGEMM_BF16 && ab_dtype != SMGEMM_F16) return SMGEMM_ERR_UNSUPPORTED;
  if (!valid_layout(layout_a) || !valid_layout(layout_b)) return SMGEMM_ERR_INVALID_ARG;
  if (!valid_out_dtype(c_dtype) || !valid_act(act)) return SMGEMM_ERR_INVALID_ARG;
  if (G == 0) return SMGEMM_OK;
  // Validate every group before anything is launched.
  for (int g = 0; g < G; ++g) {
    if (!fits_int(M[g]) || !fits_int(N[g]) || !fits_int(K[g])) return SMGEMM_ERR_INVALID_ARG;
    if (M[g] == 0 || N[g] == 0) continue;
    const void* bg = bias != nullptr ? bias[g] : nullptr;
    smgemm_status st = check_output(M[g], N[g], C[g], c_dtype, ldc[g], bg, bias_dtype, act);
    if (st != SMGEMM_OK) return st;
    if (K[g] > 0) {
      if (A[g] == nullptr || B[g] == nullptr) return SMGEMM_ERR_INVALID_ARG;
      if (lda[g] < (layout_a == SMGEMM_ROW_MAJOR ? K[g] : M[g]) || ldb[g] < (layout_b == SMGEMM_ROW_MAJOR ? N[g] : K[g]))
        return SMGEMM_ERR_INVALID_ARG;
      if (!aligned16(A[g]) || !aligned16(B[g]) || (lda[g] * 2) % 16 != 0 || (ldb[g] * 2) % 16 != 0)
        return SMGEMM_ERR_ALIGNMENT;
    }
  }
  if (workspace == nullptr || workspace_bytes < grouped_table_bytes(G)) return SMGEMM_ERR_WORKSPACE;
  // The split-wave partials are read and written as float4 at workspace + table bytes.
  if (!aligned16(workspace)) return SMGEMM_ERR_ALIGNMENT;
  DevInfo d;
  if (current_device(d) != SMGEMM_OK) return SMGEMM_ERR_CUDA;
  const CUtensorMapDataType dt =
      ab_dtype == SMGEMM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const uint32_t fmt = ab_dtype == SMGEMM_BF16 ? 1u : 0u;
  const bool a_mn = (layout_a == SMGEMM_COL_MAJOR);
  const bool b_mn = (layout_b == SMGEMM_ROW_MAJOR);
  const int bk = grouped_bk();
  // Up to kInlineGroups records are passed with the launch (no copy); more go to the
  // workspace (launch_upload_group_table).
  const bool inline_table = G <= kInlineGroups;
  GroupTableInline inl;
  std::vector<GroupDesc> heap;
  if (!inline_table) heap.resize(static_cast<size_t>(G));
  GroupDesc* table = inline_table ? inl.d : heap.data();
  std::vector<int> fills;  // groups with K = 0: filled with act(bias) after the table is enqueued
  long long tiles = 0, t_tiles = 0;
  const bool transpose_rem = env_ll(kKnobGroupedTranspose, 1) != 0;
  // Order of the groups in the table, and so in the tile numbering: by default the
  // groups with the most work (M N K) first, so that the last, ragged wave holds the
  // smallest groups' tiles (measured on mixed expert sizes: 1-1.3% faster than the order
  // given; SMGEMM_GROUPED_ORDER=0 keeps the given order, 2 alternates largest and
  // smallest). Results do not depend on the order: each tile is computed whole or
  // summed in K order.
  std::vector<int> perm(static_cast<size_t>(G));
  for (int g = 0; g < G; ++g) perm[static_cast<size_t>(g)] = g;
  const long long order = env_ll(kKnobGroupedOrder, 1);
  if (order == 1 || order == 2) {
    auto work = [&](int g) {  // in double: the product of three int-sized extents can overflow int64
      return static_cast<double>(M[g]) * static_cast<double>(N[g]) * static_cast<double>(K[g]);
    };
    std::stable_sort(perm.begin(), perm.end(), [&](int x, int y) { return work(x) > work(y); });
    if (order == 2) {  // largest, smallest, second largest, second smallest, ...
      std::vector<int> z;
      z.reserve(perm.size());
      for (size_t lo = 0, hi = perm.size(); lo < hi;) {
        z.push_back(perm[lo++]);
        if (lo < hi) z.push_back(perm[--hi]);
      }
      perm.swap(z);
    }
  }
  for (int i = 0; i < G; ++i) {
    const int g = perm[static_cast<size_t>(i)];
    GroupDesc& e = table[i];
    std::memset(&e, 0, sizeof(e));
    e.tile0 = tiles;
    e.M = static_cast<int>(M[g]);
    e.N = static_cast<int>(N[g]);
    e.ldc = ldc[g];
    e.C = C[g];
    e.bias = bias != nullptr ? bias[g] : nullptr;
    if (M[g] == 0 || N[g] == 0) continue;
    if (K[g] == 0) {  // no products: the output is act(bias) (or act(0))
      fills.push_back(g);
      continue;
    }
    bool ok;
    // A's boxes are 64 rows (K-major): a normal tile loads two per K slice, the B slot
    // of a transposed remainder tile one.
    if (a_mn) ok = encode_2d(&e.tm_a, dt, A[g], M[g], K[g], lda[g] * 2, 64, bk);
    else ok = encode_2d(&e.tm_a, dt, A[g], K[g], M[g], lda[g] * 2, 64, 64);
    if (b_mn) ok = ok && encode_2d(&e.tm_b, dt, B[g], N[g], K[g], ldb[g] * 2, 64, bk);
    else ok = ok && encode_2d(&e.tm_b, dt, B[g], K[g], N[g], ldb[g] * 2, 64, 128);
    if (!ok) return SMGEMM_ERR_CUDA;
    e.m_tiles = static_cast<int>((M[g] + 255) / 256);
    e.n_tiles = static_cast<int>((N[g] + 255) / 256);
    e.kb_total = static_cast<int>((K[g] + bk - 1) / bk);
    e.rem_t = transpose_rem && M[g] - static_cast<int64_t>(e.m_tiles - 1) * 256 <= 128 ? 1 : 0;
    tiles += static_cast<long long>(e.m_tiles) * e.n_tiles;
    if (e.rem_t) t_tiles += e.n_tiles;
  }
  const int clusters_max = tiles > 0 ? grouped_max_clusters() : 0;
  if (tiles > 0 && clusters_max <= 0) return SMGEMM_ERR_CUDA;
  GroupDesc* dev_table = reinterpret_cast<GroupDesc*>((reinterpret_cast<uintptr_t>(workspace) + 63) & ~uintptr_t(63));
  // The table goes with small kernels' parameters (captured by value in a CUDA graph);
  // it is the first thing enqueued, so a failure here leaves every output untouched.
  if (!inline_table && tiles > 0) {
    const smgemm_status st = launch_status(launch_upload_group_table(table, G, dev_table, stream));
    if (st != SMGEMM_OK) return st;
  }
  for (int g : fills) {
    smgemm_status st = launch_status(launch_fill_epilogue(static_cast<int>(M[g]), static_cast<int>(N[g]),
                                                          bias != nullptr ? bias[g] : nullptr, bias_dtype, act, C[g],
                                                          c_dtype, ldc[g], stream));
    if (st != SMGEMM_OK) return st;
  }

  if (tiles == 0) return SMGEMM_OK;
  GroupedParams p{};
  p.groups = dev_table;
  p.G = G;
  p.total_tiles = tiles;
  p.group_m = static_cast<int>(env_ll(kKnobGroupM, 8));
  p.bias_dtype = bias_dtype;
  p.act = act;
  p.c_dtype = c_dtype;
  p.a_mn_major = a_mn ? 1 : 0;
  p.b_mn_major = b_mn ? 1 : 0;
  p.idesc = idesc_f32acc(fmt, fmt, a_mn ? 1u : 0u, b_mn ? 1u : 0u, 256, 256);
  p.idesc_t = idesc_f32acc(fmt, fmt, b_mn ? 1u : 0u, a_mn ? 1u : 0u, 256, 128);
  p.wait_limit_cycles = wait_limit();
  // A ragged last wave (R = tiles mod P tiles for P co-resident clusters; all tiles when
  // there are fewer than P) is split along K into S pieces when every tail tile keeps at
  // least 8 K-blocks per piece and the workspace holds the partials.
  const int P = clusters_max;
  const long long R = tiles % P;
  int S = 0;
  if (R > 0 && env_ll(kKnobGroupedSplit, 1) != 0) {
    int min_kb = 1 << 30;
    long long left = R;
    for (int g = G - 1; g >= 0 && left > 0; --g) {
      const GroupDesc& e = table[static_cast<size_t>(g)];
      const long long t = static_cast<long long>(e.m_tiles) * e.n_tiles;
      if (t == 0) continue;
      min_kb = std::min(min_kb, e.kb_total);
      left -= t;
    }
    S = static_cast<int>(std::min<long long>(P / R, min_kb / 8));
    if (S < 2 || workspace_bytes < grouped_table_bytes(G) + grouped_split_bytes(static_cast<int>(R * S))) S = 0;
  }
  int clusters = static_cast<int>(std::min<long long>(tiles, P));
  GroupedSplit sp{0, 0, nullptr, nullptr, 0};
  if (S >= 2) {
    if (tiles < P) clusters = static_cast<int>(R * S);
    uint8_t* split_base = static_cast<uint8_t*>(workspace) + grouped_table_bytes(G);
    sp.split_tiles = R;
    sp.splits = S;
    sp.slots = reinterpret_cast<float*>(split_base);
    sp.counters = reinterpret_cast<unsigned long long*>(split_base +
                                                        static_cast<size_t>(R * S) * 2 * 128 * 256 * sizeof(float));
    sp.gen = next_generation();
  }
  std::snprintf(config_text(), sizeof(g_last_config),
                "path=grouped groups=%d tiles=%lld transposed_tiles=%lld grid=%d tile=128x256 split_tiles=%lld splits=%d",
                G, tiles, t_tiles, clusters, S >= 2 ? R : 0LL, S >= 2 ? S : 0);
  if (env_ll(kKnobLog, 0)) std::fprintf(stderr, "[smgemm] %s\n", g_last_config);
  return launch_status(launch_gemm_grouped_split(p, sp, inline_table ? &inl : nullptr, clusters, stream));
}

smgemm_status gemm_fp8_blockscaled(int64_t M, int64_t N, int64_t K, const uint8_t* Aq, const float* sa,
                                   const uint8_t* Bq, const float* sb, const void* bias, smgemm_dtype bias_dtype,
                                   smgemm_act act, void* C, smgemm_dtype c_dtype, int64_t ldc, void* workspace,
                                   size_t workspace_bytes, smgemm_stream_t stream_) {
  const CallScope scope("smgemm:gemm_fp8_blockscaled");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!fits_int(M) || !fits_int(N) || !fits_int(K)) return SMGEMM_ERR_INVALID_ARG;
  if (!valid_out_dtype(c_dtype) || !valid_act(act)) return SMGEMM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return SMGEMM_OK;
  smgemm_status st = check_output(M, N, C, c_dtype, ldc, bias, bias_dtype, act);
  if (st != SMGEMM_OK) return st;
  if (K > 0) {
    if (Aq == nullptr || Bq == nullptr || sa == nullptr || sb == nullptr) return SMGEMM_ERR_INVALID_ARG;
    if (!aligned16(Aq) || !aligned16(Bq) || K % 16 != 0) return SMGEMM_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(sa) & 3u) || (reinterpret_cast<uintptr_t>(sb) & 3u)) return SMGEMM_ERR_ALIGNMENT;
  }
  DevInfo d;
  if (current_device(d) != SMGEMM_OK) return SMGEMM_ERR_CUDA;
  if (K == 0) {
    std::snprintf(config_text(), sizeof(g_last_config), "path=fill");
    return launch_status(launch_fill_epilogue(static_cast<int>(M), static_cast<int>(N), bias, bias_dtype, act, C,
                                              c_dtype, ldc, stream));
  }
  const int tn = fp8_tile_n();
  const Fp8Plan f = plan_fp8(M, N, K, d.sms, tn, fp8_pair_max_clusters(tn));
  const Plan& pl = f.pl;
  CUtensorMap tm_a, tm_b;
  bool ok = encode_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, Aq, K, M, K, 128, 128);
  ok = ok && encode_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, Bq, K, N, K, 128, f.pair ? f.tn / 2 : 128);
  if (!ok) return SMGEMM_ERR_CUDA;
  Fp8Params p{};
  p.s = pl.s;
  p.e = EpiArgs{static_cast<int>(M), static_cast<int>(N), bias, bias_dtype, act, C, c_dtype, ldc};
  p.K = static_cast<int>(K);
  p.idesc = f.pair ? idesc_f32acc(0u, 0u, 0u, 0u, 256, f.tn) : idesc_f32acc(0u, 0u, 0u, 0u, 128, 128);
  p.sa = sa;
  p.sb = sb;
  p.nb_count = static_cast<int>((N + 127) / 128);
  p.wait_limit_cycles = wait_limit();
  st = prepare_workspace(pl, workspace, workspace_bytes, &p.slots, &p.counters, &p.gen);
  if (st != SMGEMM_OK) return st;
  if (f.pair) {
    note_config("fp8pair", pl, f.tn);
    return launch_status(launch_gemm_fp8_pair(tm_a, tm_b, p, pl.grid, f.tn, stream));
  }
  note_config("fp8", pl, 128);
  return launch_status(launch_gemm_fp8(tm_a, tm_b, p, pl.grid, stream));
}

smgemm_status quantize_fp8_blockwise(const float* X, int64_t rows, int64_t cols, smgemm_layout layout_x,
                                     int64_t ldx, int group_rows, uint8_t* Q, float* scales,
                                     smgemm_stream_t stream_) {
  const CallScope scope("smgemm:quantize_fp8_blockwise");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (rows < 0 || cols < 0 || !valid_layout(layout_x)) return SMGEMM_ERR_INVALID_ARG;
  if (group_rows != 1 && group_rows != 128) return SMGEMM_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return SMGEMM_OK;
  if (X == nullptr || Q == nullptr || scales == nullptr) return SMGEMM_ERR_INVALID_ARG;
  if (ldx < (layout_x == SMGEMM_ROW_MAJOR ? cols : rows)) return SMGEMM_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Q) || (ldx * 4) % 16 != 0 || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return SMGEMM_ERR_ALIGNMENT;
  DevInfo d;
  if (current_device(d) != SMGEMM_OK) return SMGEMM_ERR_CUDA;
  const bool row_major = layout_x == SMGEMM_ROW_MAJOR;
  if (group_rows == 1 && !row_major)
    return launch_status(launch_quant_1x128_cols(X, rows, cols, ldx, Q, scales, stream));
  // Row-major: [rows][cols]; column-major: [cols][rows] (for 128x128, rows = K, cols = N).
  CUtensorMap tm;
  const uint64_t inner = row_major ? cols : rows, outer = row_major ? rows : cols;
  if (!encode_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, X, inner, outer, static_cast<uint64_t>(ldx) * 4, 128,
                 group_rows == 1 ? 32 : 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SMGEMM_ERR_CUDA;
  cudaError_t e = group_rows == 1
                      ? launch_quant_1x128_tma(tm, rows, cols, Q, scales, d.sms, wait_limit(), stream)
                      : launch_quant_128x128_tma(tm, row_major, rows, cols, Q, scales, d.sms, wait_limit(), stream);
  return launch_status(e);
}

smgemm_status smgemm_check(smgemm_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return SMGEMM_ERR_CUDA;
  }
  const unsigned e = take_error_word_tc16() | take_error_word_fp8() | take_error_word_misc() | take_error_word_pair() |
                     take_error_word_fp8_pair() | take_error_word_grouped();
  return (e & kErrTimeout) ? SMGEMM_ERR_TIMEOUT : SMGEMM_OK;
}

smgemm_status smgemm_selftest_wait_timeout(uint32_t limit_us, smgemm_stream_t stream_) {
  DevInfo d;
  if (current_device(d) != SMGEMM_OK) return SMGEMM_ERR_CUDA;
  if (limit_us == 0 || limit_us > 10000000u) return SMGEMM_ERR_INVALID_ARG;
  return launch_status(
      launch_wait_selftest(static_cast<unsigned long long>(limit_us) * 1000ull, reinterpret_cast<cudaStream_t>(stream_)));
}

int64_t smgemm_schedule_dump(int64_t M, int64_t N, int64_t K, int kind, smgemm_layout layout_a, int num_sms,
                             int32_t* out, int64_t cap) {
  refresh_knobs();
  if (M <= 0 || N <= 0 || K <= 0 || num_sms <= 0) return 0;
  const Plan pl = kind == 1 ? plan_fp8(M, N, K, num_sms, fp8_tile_n(), num_sms / 2).pl
                            : plan_gemm16(M, N, K, layout_a, num_sms, num_sms / 2).pl;
  int64_t n = 0;
  for (int c = 0; c < pl.grid; ++c) {
    WorkIter it;
    it.init(pl.s, c);
    Seg seg;
    while (it.next(pl.s, seg)) {
      if (out != nullptr && n < cap) {
        int mt, nt;
        tile_coords(pl.s, seg.tile, mt, nt);
        int32_t* r = out + 7 * n;
        r[0] = c; r[1] = seg.tile; r[2] = mt; r[3] = nt; r[4] = seg.kb0; r[5] = seg.kb1;
        r[6] = seg.tile < pl.s.dp_tiles ? -1 : seg.slot;
      }
      ++n;
    }
  }
  return n;
}

}  // extern "C"
