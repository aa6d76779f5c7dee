// Internal interface between the C-ABI layer (api.cu) and the kernels. Not installed.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "epilogue.cuh"
#include "sm100.cuh"

namespace smg {

// Element types and activations, numerically equal to the public smgemm_* enums.
constexpr int kF32 = 0, kBF16 = 1, kF16 = 2, kE4M3 = 3;
constexpr int kActNone = 0, kActGeluTanh = 1, kActSilu = 2;

// Default limit of every bounded barrier wait inside the kernels, and the SM clock
// used to turn it into cycles (an upper bound of the B200 SM clock, so the real limit
// is at least the stated time).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
constexpr unsigned long long kCyclesPerNs = 2;

struct Tc16Params {
  TileSched s;
  EpiArgs e;                // output, bias, activation
  uint32_t idesc;           // tcgen05 instruction descriptor
  int a_mn_major;           // MMA "A" operand tile is MN-major (else K-major)
  int b_mn_major;           // MMA "B" operand tile is MN-major (else K-major)
  float* slots;             // stream-K partial tiles: [num_ctas][2][MMA_N][128] floats
  unsigned long long* counters;  // stream-K arrival counters (counter_arrive), one per stream-K tile
  unsigned long long gen;        // this call's counter generation
  unsigned long long wait_limit_cycles;
  // Swap-AB (skinny) kernels only, nullable: per 128-column tile of the output and per
  // token row, the tile's max logit and sum of exp(logit - max) (float2 [m_tiles][M]).
  float2* lse_part;
};

enum class Tc16Variant { kLarge, kSkinny16, kSkinny32, kSkinny64 };

cudaError_t launch_gemm_tc16(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const Tc16Params& p,
                             Tc16Variant v, int grid, cudaStream_t stream);
int tc16_mma_n(Tc16Variant v);
int tc16_bk(Tc16Variant v);

// CTA-pair large-tile kernel (256 x 256 per cluster of 2). p.s counts clusters;
// p.slots is [clusters][2][2 ranks][256][128] floats, p.counters [stream-K tiles][2].
// tm_c (nullable): a tensor map of C (box 32 x 32, 64-byte swizzle for 16-bit C, 128-byte
// for FP32) selects the epilogue that writes C with TMA tile stores.
cudaError_t launch_gemm_tc16_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap* tm_c,
                                  const Tc16Params& p, int clusters, cudaStream_t stream);
int tc16_pair_max_clusters();   // co-resident clusters of 2 on the current device (0 if unknown)
int tc16_pair_bk();

// Row log-softmax of an FP32 [M, N] logit matrix in place (logsoftmax.cu): lse[m] from the
// GEMM's per-tile partials (part != nullptr, [n_tiles][M]) or from the logits, then
// C[m, n] -= lse[m].
cudaError_t launch_log_softmax_rows(float* C, long long ldc, int M, int N, const float2* part, int n_tiles,
                                    float* lse, int sms, cudaStream_t stream);
// Per-128-column-tile (max, sum of exp) partials of an FP32 [M, N] logit matrix, part[t * M + m].
cudaError_t launch_lse_tile_partials(const float* C, long long ldc, int M, int N, float2* part, cudaStream_t stream);

// Grouped GEMM (gemm_grouped.cu): one record per group in device memory, 64-byte
// aligned (the TMA descriptors must be). tile0 = index of the group's first tile in the
// launch's tile order; groups with no tiles share their successor's tile0.
struct alignas(64) GroupDesc {
  CUtensorMap tm_a, tm_b;   // A: boxes of 64 rows (K-major) or 64 M x BK; B: 128 columns x BK
  long long tile0;
  int M, N, kb_total, m_tiles, n_tiles;
  int rem_t;                // 1: the last row of tiles (<= 128 rows) runs transposed
  const void* bias;         // nullable
  void* C;
  long long ldc;
};
static_assert(sizeof(GroupDesc) % 64 == 0, "GroupDesc keeps the descriptors 64-byte aligned in an array");

struct GroupedParams {
  const GroupDesc* groups;  // G records
  int G;
  long long total_tiles;
  int group_m;
  int bias_dtype, act, c_dtype;
  int a_mn_major, b_mn_major;
  uint32_t idesc;
  uint32_t idesc_t;         // transposed remainder tiles: M = 256 (B columns), N = 128 (A rows)
  unsigned long long wait_limit_cycles;
};

cudaError_t launch_gemm_grouped(const GroupedParams& p, int clusters, cudaStream_t stream);
int grouped_max_clusters();
int grouped_bk();

struct Fp8Params {
  TileSched s;
  EpiArgs e;
  int K;
  uint32_t idesc;
  const float* sa;          // [KB][M]
  const float* sb;          // [KB][NB]
  int nb_count;             // NB = ceil(N/128)
  float* slots;             // [num_ctas][2][128][128] floats
  unsigned long long* counters;  // stream-K arrival counters (counter_arrive)
  unsigned long long gen;        // this call's counter generation
  unsigned long long wait_limit_cycles;
};

cudaError_t launch_gemm_fp8(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const Fp8Params& p,
                            int grid, cudaStream_t stream);
constexpr int kFp8BM = 128, kFp8BN = 128, kFp8BK = 128;

// CTA-pair FP8 kernel (256 x tn per cluster of 2, tn = 256 or 128); p.s counts
// clusters, p.slots is [clusters][2][2 ranks][128][tn] floats, p.counters
// [stream-K tiles][2].
cudaError_t launch_gemm_fp8_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const Fp8Params& p,
                                 int clusters, int tn, cudaStream_t stream);
int fp8_pair_max_clusters(int tn);

// C[m, n] = act(bias[n]) (or act(0)) for the K == 0 degenerate GEMM.
cudaError_t launch_fill_epilogue(int M, int N, const void* bias, int bias_dtype, int act, void* C,
                                 int c_dtype, long long ldc, cudaStream_t stream);

// FP8 quantisers. Row-major 1x128 and both 128x128 layouts take a 2-D FLOAT32 tensor map
// without swizzle: 1x128 box {128 columns, 32 rows} over [rows][cols]; 128x128 box
// {128, 128} over [K][N] (n_contig) or [N][K]. Column-major 1x128 takes X itself.
cudaError_t launch_quant_1x128_tma(const CUtensorMap& tm_x, long long rows, long long cols, uint8_t* Q, float* S,
                                   int sms, unsigned long long limit, cudaStream_t stream);
cudaError_t launch_quant_1x128_cols(const float* X, long long rows, long long cols, long long ldx, uint8_t* Q,
                                    float* S, cudaStream_t stream);
cudaError_t launch_quant_128x128_tma(const CUtensorMap& tm_x, bool n_contig, long long K, long long N, uint8_t* Q,
                                     float* S, int sms, unsigned long long limit, cudaStream_t stream);

cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t stream);

// Per-translation-unit device error words (see sm100.cuh).
unsigned take_error_word_tc16();
unsigned take_error_word_fp8();
unsigned take_error_word_misc();
unsigned take_error_word_pair();
unsigned take_error_word_fp8_pair();
unsigned take_error_word_grouped();

}  // namespace smg
