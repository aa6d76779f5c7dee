/*
 * smgemm: dense GEMM C = epilogue(A*B) for NVIDIA B200 (sm_100a).
 *
 * The operation is the general matrix multiply that dominates LLM training and
 * inference ("从一次深夜的算力账单说起：为什么我们要死磕GEMM", kwkr.cn, sections
 * 2.1-3.1: projections, FFN up/down and the LM head are all C = X*W (+ b)), exported
 * as plain functions callable from any framework (DeepGEMM kernel-library
 * walkthrough, zwxr.cn, section 1.3).
 *
 * Conventions shared by every entry point:
 *  - All matrix, vector and workspace pointers are DEVICE pointers owned by the
 *    caller. The library allocates no device memory.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream). They return after enqueueing; they never synchronise.
 *  - Argument errors are detected on the host and returned before anything is
 *    enqueued. Launch failures return SMGEMM_ERR_CUDA. A kernel that gives up
 *    waiting on an internal pipeline barrier (about 2 s) records
 *    SMGEMM_ERR_TIMEOUT in a device-side word that smgemm_check() returns.
 *  - Shapes: M, N, K >= 0. M == 0 or N == 0 is a no-op. K == 0 writes
 *    act(bias) (or act(0)) to C.
 *  - TMA alignment: every matrix base pointer and every leading dimension in
 *    bytes must be a multiple of 16 (else SMGEMM_ERR_ALIGNMENT).
 *  - Layouts: SMGEMM_ROW_MAJOR means the second index is contiguous,
 *    SMGEMM_COL_MAJOR the first. C is always row-major with leading dimension ldc.
 *  - No exception crosses this interface. Thread-safe.
 *  - Tuning and test switches (SMGEMM_FORCE_CONFIG, SMGEMM_SPLITK, SMGEMM_SCHED,
 *    SMGEMM_GROUP_M, SMGEMM_EPI_STORE, SMGEMM_PDL, SMGEMM_LOG, ...) are read from the
 *    process environment once each time a call enters the library; each entry point
 *    opens an NVTX range named after it ("smgemm:<entry point>").
 */
#ifndef SMGEMM_H
#define SMGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* smgemm_stream_t;

typedef enum {
  SMGEMM_OK = 0,
  SMGEMM_ERR_INVALID_ARG = 1,   /* bad shape, null pointer, bad enum, ld too small */
  SMGEMM_ERR_UNSUPPORTED = 2,   /* valid but unsupported combination of types */
  SMGEMM_ERR_ALIGNMENT = 3,     /* a base pointer or ld*elem_size not a multiple of 16 B */
  SMGEMM_ERR_WORKSPACE = 4,     /* workspace smaller than smgemm_workspace_size() */
  SMGEMM_ERR_CUDA = 5,          /* a CUDA runtime/driver call failed, or no sm_100 device */
  SMGEMM_ERR_TIMEOUT = 6        /* a kernel abandoned a barrier wait (see smgemm_check) */
} smgemm_status;

typedef enum { SMGEMM_F32 = 0, SMGEMM_BF16 = 1, SMGEMM_F16 = 2, SMGEMM_E4M3 = 3 } smgemm_dtype;
typedef enum { SMGEMM_ROW_MAJOR = 0, SMGEMM_COL_MAJOR = 1 } smgemm_layout;
typedef enum { SMGEMM_ACT_NONE = 0, SMGEMM_ACT_GELU_TANH = 1, SMGEMM_ACT_SILU = 2 } smgemm_act;

/*
 * gemm_bf16: C[M,N] = cast_c( act( A[M,K] * B[K,N] + bias[N] ) ).
 *
 * 16-bit inputs with FP32 accumulation and one rounding (nearest-even) to the
 * output type (walkthrough section 2.4: low-precision inputs, high-precision
 * accumulator; section 5.1: bias and activation fused before the write-back).
 *   A        device, ab_dtype (SMGEMM_BF16 or SMGEMM_F16), logical [M,K] with
 *            layout_a; lda = distance in elements between consecutive rows
 *            (row-major, lda >= K) or columns (col-major, lda >= M).
 *   B        device, same dtype as A, logical [K,N] with layout_b; ldb likewise
 *            (row-major: ldb >= N; col-major, i.e. W^T stored [N,K]: ldb >= K).
 *   bias     device, nullable; bias_dtype SMGEMM_BF16 / SMGEMM_F16 / SMGEMM_F32; N entries.
 *   act      SMGEMM_ACT_NONE, SMGEMM_ACT_GELU_TANH (0.5x(1+tanh(sqrt(2/pi)(x+0.044715x^3))))
 *            or SMGEMM_ACT_SILU (x/(1+e^-x)), applied after the bias add, both as
 *            x*sigmoid(z) without cancellation: in FP32 for 16-bit outputs (relative error
 *            below 2^-16), in FP64 with one rounding for FP32 outputs (within one FP32 ulp).
 *   C        device, c_dtype SMGEMM_F32 / SMGEMM_BF16 / SMGEMM_F16, row-major, ldc >= N.
 *   workspace  device scratch of at least smgemm_workspace_size(M,N,K,0) bytes,
 *            16-byte aligned (may be NULL when that size is 0). The library uses it
 *            for split-K / stream-K partial tiles and their arrival counters; its
 *            contents on entry do not matter (no zeroing needed: the counters carry a
 *            per-call generation), and a completed call leaves every counter at zero, so
 *            a call captured in a CUDA graph can be replayed on the same workspace any
 *            number of times. It must not be shared by calls that can overlap on the GPU.
 * Small M (<= 64, row-major A) runs the memory-bound swap-AB path; everything else
 * the persistent tensor-core path. Results are deterministic run to run.
 */
smgemm_status gemm_bf16(int64_t M, int64_t N, int64_t K,
                        const void* A, smgemm_dtype ab_dtype, smgemm_layout layout_a, int64_t lda,
                        const void* B, smgemm_layout layout_b, int64_t ldb,
                        const void* bias, smgemm_dtype bias_dtype, smgemm_act act,
                        void* C, smgemm_dtype c_dtype, int64_t ldc,
                        void* workspace, size_t workspace_bytes, smgemm_stream_t stream);

/*
 * gemm_bf16_noalloc: gemm_bf16 without a workspace argument, for callers that cannot
 * allocate device memory - e.g. a plugin or custom-op host that is handed only its
 * input and output buffers, or a latency-critical decode loop that must not call
 * cudaMalloc (which can synchronise the device). The GEMM sources have no counterpart
 * for this entry point; it only changes where the scratch comes from.
 *   Arguments, results and errors are those of gemm_bf16 (same kernels, same schedule).
 *   Scratch is a fixed SMGEMM_NOALLOC_SCRATCH_BYTES (16 MiB) array inside the library's
 *   device image; every GPU that loads the library holds it until the process exits.
 *   A call whose schedule needs more scratch than that (at most smgemm_workspace_size)
 *   returns SMGEMM_ERR_WORKSPACE before enqueueing anything. The library allocates nothing.
 *   All calls share the array and it keeps the previous call's contents (nothing in it
 *   needs clearing); calls that can overlap on the GPU race on it.
 *   The first call on each device resolves the array's device address; under CUDA's
 *   default lazy module loading it also loads the library's device code there and
 *   reserves the array (milliseconds, may synchronise), so make it during warm-up,
 *   outside any latency-critical loop and before any stream capture. After
 *   cudaDeviceReset the next call resolves the address again in the new context.
 */
#define SMGEMM_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
smgemm_status gemm_bf16_noalloc(int64_t M, int64_t N, int64_t K,
                                const void* A, smgemm_dtype ab_dtype, smgemm_layout layout_a, int64_t lda,
                                const void* B, smgemm_layout layout_b, int64_t ldb,
                                const void* bias, smgemm_dtype bias_dtype, smgemm_act act,
                                void* C, smgemm_dtype c_dtype, int64_t ldc, smgemm_stream_t stream);

/*
 * gemm_bf16_grouped: for g < G, C_g[M_g,N_g] = cast_c( act( A_g[M_g,K_g] * B_g[K_g,N_g] + bias_g ) ),
 * all groups in one persistent launch ("为什么我们要死磕GEMM" (kwkr.cn), section 5.3:
 * batch many small GEMMs instead of launching them one by one).
 *   G          number of groups (0: no-op).
 *   M,N,K,lda,ldb,ldc   host arrays of G sizes / leading dimensions, meaning as in gemm_bf16.
 *   A,B,C      host arrays of G device pointers; bias: nullable host array of G
 *              (nullable) device pointers.
 *   ab_dtype, layout_a, layout_b, bias_dtype, act, c_dtype: shared by all groups, as in
 *              gemm_bf16. Groups with M or N = 0 are skipped; K = 0 writes act(bias).
 *   workspace  device, 16-byte aligned (else SMGEMM_ERR_ALIGNMENT), at least
 *              smgemm_grouped_workspace_size(G) bytes: with more than 16 groups the
 *              groups' TMA descriptors and sizes are written there before the launch (by
 *              small kernels on `stream` that carry them as parameters, so the call can be
 *              captured in a CUDA graph; up to 16 groups travel with the launch itself);
 *              the rest holds the partial tiles of a split last wave. Calls that can
 *              overlap on the GPU must not share it. A smaller workspace that still holds
 *              the table is accepted; the last wave is then not split.
 * Every group is validated, and every TMA descriptor encoded, before anything is
 * enqueued; the descriptor table is written first, then groups with K = 0 are filled,
 * then the GEMM launches. Errors as in gemm_bf16. Tiles of 256 x 256 run one per CTA
 * pair, the groups laid out with the most work (M N K) first; a group's last row of
 * tiles with at most 128 rows runs as 256 x 128 tiles of C_g^T = B_g^T A_g^T instead (half
 * the tensor work of a 256-row tile padded with zero rows). When the tiles do not fill a
 * whole last wave, the R tiles of that wave are each split along K into
 * S = min(P / R, KB / 8) pieces (P co-resident pairs, KB the smallest K-block count
 * among those tiles) that run side by side; the last piece to finish sums the partials
 * in piece order, so results are deterministic run to run and do not depend on the
 * groups' order.
 */
size_t smgemm_grouped_workspace_size(int G);
smgemm_status gemm_bf16_grouped(int G, const int64_t* M, const int64_t* N, const int64_t* K,
                                const void* const* A, smgemm_dtype ab_dtype, smgemm_layout layout_a,
                                const int64_t* lda, const void* const* B, smgemm_layout layout_b,
                                const int64_t* ldb, const void* const* bias, smgemm_dtype bias_dtype,
                                smgemm_act act, void* const* C, smgemm_dtype c_dtype, const int64_t* ldc,
                                void* workspace, size_t workspace_bytes, smgemm_stream_t stream);

/*
 * gemm_bf16_fp8out: the gemm_bf16 epilogue quantised to FP8 on the way out: with
 * Z = act(A[M,K] * B[K,N] + bias[N]) in FP32, every 1x128 row group of Z (columns
 * 128g .. 128g+127) is encoded as quantize_fp8_blockwise does (amax over the group's
 * present elements, s = amax/448 or 1 for an all-zero group, code = E4M3(z / s) with
 * a correctly rounded division, RN satfinite) - "fuse activation, quantization and
 * scaling" (DeepGEMM kernel-library walkthrough, zwxr.cn, sections 1.2 and 2.4). The
 * output is exactly the A operand gemm_fp8_blockscaled takes (K' = N).
 *   A, B, bias, act, lda, ldb, layouts, workspace: as in gemm_bf16.
 *   Cq      device uint8 E4M3 codes [M][N] row-major, 16-byte aligned, ldc >= N and a
 *           multiple of 16.
 *   scales  device float [ceil(N/128)][M], 4-byte aligned.
 * Runs on the CTA-pair kernel (any M); K = 0 returns SMGEMM_ERR_UNSUPPORTED.
 */
smgemm_status gemm_bf16_fp8out(int64_t M, int64_t N, int64_t K,
                               const void* A, smgemm_dtype ab_dtype, smgemm_layout layout_a, int64_t lda,
                               const void* B, smgemm_layout layout_b, int64_t ldb,
                               const void* bias, smgemm_dtype bias_dtype, smgemm_act act,
                               uint8_t* Cq, int64_t ldc, float* scales,
                               void* workspace, size_t workspace_bytes, smgemm_stream_t stream);

/*
 * gemm_bf16_logsoftmax: C[m,n] = z[m,n] - log sum_n' exp(z[m,n']), z = A[M,K] * B[K,N] + bias[N]
 * in FP32: the LM-head projection fused with the row log-softmax that follows it
 * ("为什么我们要死磕GEMM" (kwkr.cn), section 7.2, scheme B: GEMM + bias + LogSoftmax).
 *   A, B, bias, lda, ldb, layouts: as in gemm_bf16 (no activation).
 *   C          device float [M,N] row-major, ldc >= N (16-byte aligned rows): the
 *              log-probabilities (the logits are written there first and normalised in place).
 *   workspace  device, >= smgemm_logsoftmax_workspace_size(M,N,K) bytes, 16-byte aligned.
 * On the skinny path (M <= 64, row-major A) the GEMM epilogue also reduces every 128
 * logits of a row to (max, sum of exp) and the second pass only merges those and
 * subtracts; otherwise the second pass reads the row's logits. Deterministic.
 */
size_t smgemm_logsoftmax_workspace_size(int64_t M, int64_t N, int64_t K);
smgemm_status gemm_bf16_logsoftmax(int64_t M, int64_t N, int64_t K,
                                   const void* A, smgemm_dtype ab_dtype, smgemm_layout layout_a, int64_t lda,
                                   const void* B, smgemm_layout layout_b, int64_t ldb,
                                   const void* bias, smgemm_dtype bias_dtype,
                                   float* C, int64_t ldc,
                                   void* workspace, size_t workspace_bytes, smgemm_stream_t stream);

/*
 * Vocabulary-parallel LM head: the log-softmax of gemm_bf16_logsoftmax split in two steps,
 * so that each GPU can hold only its slice of the vocabulary (the columns of W) and the
 * ranks exchange nothing but the small per-row partials between the steps (the LM head is
 * the memory-bound "thin and tall" GEMM of "为什么我们要死磕GEMM" (kwkr.cn), sections 2.2
 * and 7.2; splitting its columns multiplies the HBM bandwidth that streams W).
 *
 * gemm_bf16_lse_partials: z = A[M,K] * B[K,N] + bias[N] in FP32, written to C (row-major,
 *   ldc >= N, 16-byte aligned rows), and for every 128-column tile t < ceil(N/128) and row
 *   m the pair part[2*(t*M + m) + 0/1] = (max of the tile's z, sum of exp(z - max)).
 *   A, B, bias, layouts, lda, ldb: as in gemm_bf16 (no activation). part: device float
 *   [ceil(N/128)][M][2], 16-byte aligned. workspace: smgemm_workspace_size(M,N,K,0) bytes.
 *   On the skinny path the GEMM epilogue forms the pairs; otherwise a light pass over C does.
 *
 * logsoftmax_apply_partials: lse[m] = log sum over every column of exp(z), merged from
 *   n_parts pairs part[2*(p*M + m) + 0/1], p < n_parts (for example every rank's partials,
 *   gathered one rank after another; a pair (-inf, 0) is neutral), with the rule
 *   (m1, s1) + (m2, s2) = (m, s1 e^(m1-m) + s2 e^(m2-m)), m = max(m1, m2), in a fixed order
 *   (deterministic); then C[m, n] -= lse[m] for n < N (this rank's slice; N may be 0).
 *   C: device float, ldc >= N, 16-byte aligned. part: device, 8-byte aligned. lse: device
 *   float [M], written. n_parts >= 1.
 * Errors as in gemm_bf16.
 */
smgemm_status gemm_bf16_lse_partials(int64_t M, int64_t N, int64_t K,
                                     const void* A, smgemm_dtype ab_dtype, smgemm_layout layout_a, int64_t lda,
                                     const void* B, smgemm_layout layout_b, int64_t ldb,
                                     const void* bias, smgemm_dtype bias_dtype,
                                     float* C, int64_t ldc, float* part,
                                     void* workspace, size_t workspace_bytes, smgemm_stream_t stream);
smgemm_status logsoftmax_apply_partials(float* C, int64_t ldc, int64_t M, int64_t N,
                                        const float* part, int64_t n_parts, float* lse, smgemm_stream_t stream);

/*
 * gemm_fp8_blockscaled: C[i,j] = cast_c( act( sum_kb sa[kb,i] * sb[kb, j/128] *
 *                                         sum_{k in kb} dec(Aq[i,k]) * dec(Bq[j,k]) + bias[j] ) )
 *
 * Group-scaled FP8 (walkthrough section 2.4): E4M3 codes with one FP32 scale per
 * 1x128 K-group of A and per 128x128 block of B; products are accumulated in FP32
 * per 128-wide K-block and promoted (scaled and added) into an FP32 accumulator.
 *   Aq  device uint8 E4M3 codes [M][K], K contiguous (leading dimension K).
 *   sa  device float [ceil(K/128)][M].
 *   Bq  device uint8 E4M3 codes of the weight B[K,N] stored transposed [N][K], K contiguous.
 *   sb  device float [ceil(K/128)][ceil(N/128)].
 *   bias/act/C/ldc/workspace as in gemm_bf16 (workspace size: smgemm_workspace_size(...,1)).
 * K must be a multiple of 16 (the TMA row pitch of the code matrices).
 */
smgemm_status gemm_fp8_blockscaled(int64_t M, int64_t N, int64_t K,
                                   const uint8_t* Aq, const float* sa,
                                   const uint8_t* Bq, const float* sb,
                                   const void* bias, smgemm_dtype bias_dtype, smgemm_act act,
                                   void* C, smgemm_dtype c_dtype, int64_t ldc,
                                   void* workspace, size_t workspace_bytes, smgemm_stream_t stream);

/*
 * quantize_fp8_blockwise: FP32 -> E4M3 codes + FP32 group scales (walkthrough section 2.4).
 * For each group: amax = max|x| over the group's elements, s = amax/448 (IEEE FP32
 * division; s = 1 for an all-zero group), q = E4M3(x/s) with an IEEE division, round
 * to nearest even, saturating at +-448, sign kept on zero. Bit-exact and deterministic.
 *   group_rows == 1   (activations) X is logical [rows, cols] = [M, K]; groups are
 *                     1x128 along cols. Writes Q[rows][cols] (ld = cols) and
 *                     scales[ceil(cols/128)][rows].
 *   group_rows == 128 (weights) X is logical [rows, cols] = [K, N]; groups are
 *                     128x128 blocks. Writes Q TRANSPOSED as [cols][rows] = [N][K]
 *                     (ld = rows) and scales[ceil(rows/128)][ceil(cols/128)] - exactly
 *                     the Bq/sb operands of gemm_fp8_blockscaled.
 *   X      device float, layout_x, ldx (row-major: ldx >= cols; col-major: ldx >= rows).
 *   Q      device uint8, 16-byte aligned; scales device float. X must be 16-byte aligned and
 *          ldx*4 a multiple of 16.
 * Input precondition: no NaN or infinity in X.
 */
smgemm_status quantize_fp8_blockwise(const float* X, int64_t rows, int64_t cols,
                                     smgemm_layout layout_x, int64_t ldx, int group_rows,
                                     uint8_t* Q, float* scales, smgemm_stream_t stream);

/* Bytes of workspace a call with these sizes needs (0 when none). kind: 0 = gemm_bf16,
 * 1 = gemm_fp8_blockscaled. Depends only on the arguments and the current device. */
size_t smgemm_workspace_size(int64_t M, int64_t N, int64_t K, int kind);

/* Static description of a status code. Never NULL. */
const char* smgemm_status_string(smgemm_status status);

/* Synchronises `stream`, then returns SMGEMM_ERR_TIMEOUT if any kernel of this library
 * on the current device recorded an abandoned barrier wait since the last check (and
 * clears the record), SMGEMM_ERR_CUDA if the stream reports an error, else SMGEMM_OK. */
smgemm_status smgemm_check(smgemm_stream_t stream);

/* Description of the kernel configuration the last gemm_* call on this thread chose
 * (path, tile, grid, split), for logs and tests. Never NULL. */
const char* smgemm_last_config(void);

/* Test hook for the bounded-wait machinery: launches one CTA that waits on an
 * mbarrier nothing will ever arrive on, with the given limit in microseconds, and
 * records SMGEMM_ERR_TIMEOUT exactly like a real pipeline stall. No GPU fault,
 * trap or hang is involved; smgemm_check() then reports the timeout. */
smgemm_status smgemm_selftest_wait_timeout(uint32_t limit_us, smgemm_stream_t stream);

/* Diagnostic view of the persistent schedule a gemm_* call with these sizes would
 * use on a GPU with `num_sms` SMs (no GPU needed): writes up to `cap` records of 7
 * int32 each - (cta, tile, m_tile, n_tile, kb_begin, kb_end, slot) - in each CTA's
 * processing order (slot = -1 for data-parallel tiles, else the stream-K partial slot), and returns the number of records (may exceed cap). kind as in
 * smgemm_workspace_size; layout_a selects the skinny path as gemm_bf16 does. */
int64_t smgemm_schedule_dump(int64_t M, int64_t N, int64_t K, int kind, smgemm_layout layout_a, int num_sms,
                             int32_t* out, int64_t cap);

#ifdef __cplusplus
}
#endif

#endif /* SMGEMM_H */
