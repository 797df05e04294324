/*
 * dg.h -- C ABI of libdg.so, an sm_100a (B200) implementation of the FP8 (E4M3)
 * GEMM with 128x128 block-wise scaling, C = A * B^T, FP32 accumulation with a
 * per-K-block scale promotion, BF16 output, in a dense and an MoE
 * grouped-contiguous form, plus the BF16 -> E4M3 block quantizer that makes its
 * inputs.
 *
 * The method, as the DeepGEMM pages describe it:
 *   - FP8 E4M3 inputs (1 sign, 4 exponent, 3 mantissa bits, largest value 448):
 *     DeepGEMM FP8 write-up (demingchina.com/news/60142) §3.1 format table;
 *     DeepGEMM library page (2kiu.com/news/5461879) §2.1.
 *   - A and B cut into 128x128 blocks, one FP32 scale per block; each output
 *     block's result is multiplied by the A-block and B-block scales:
 *     2kiu.com/news/5461879 §2.1, §3.3 (FP32 scale storage).
 *   - FP32 accumulation of FP8 products, long K accumulated in segments:
 *     2kiu.com/news/5461879 §3.3.  Here every 128-wide K block's partial sum is
 *     multiplied by sA[m/128][kb] * sB[n/128][kb] and added to an FP32 register
 *     accumulator, in ascending kb order.
 *   - Scales computed ahead of time and multiplied back at the output end:
 *     demingchina.com/news/60142 §3.1.
 *   - MoE experts stored contiguously by expert id as one long matrix, one
 *     launch for all experts: nxmr.cn/news/132300 §2.2; expert N and K fixed by
 *     the model, only the token count M varies: 2kiu.com/news/5461879 §2.2.
 *
 * Conventions for every entry point:
 *   - All matrix pointers are DEVICE pointers owned by the caller.  The library
 *     allocates nothing per call and never frees caller memory.
 *   - Matrices are dense row-major.  FP8 data is raw E4M3 bytes; scales are FP32;
 *     the output is BF16 (IEEE bfloat16 bit patterns).
 *   - Every call is asynchronous and ordered on `stream` (0 = legacy default
 *     stream).  Nothing synchronises the host.  Arguments are validated on the
 *     host before anything is enqueued; on an error nothing is enqueued.
 *   - A launch failure returns DG_ERR_CUDA.  Failures detected on the device
 *     (a pipeline wait that exceeded its time limit) are recorded in a
 *     per-process device status word; read it with dg_get_last_device_status().
 *   - The device must be compute capability 10.0 (B200, sm_100a); otherwise
 *     DG_ERR_UNSUPPORTED_DEVICE.  There is no fallback path.
 *   - Calls that overlap on the GPU are independent unless they write the same
 *     output.  Results are bitwise run-to-run deterministic.
 *   - Kernels are launched with programmatic stream serialisation: a kernel may
 *     start its set-up (barriers, tensor memory, descriptor and L2 prefetches of
 *     weights) while the previous kernel on `stream` finishes, and waits for that
 *     kernel to complete before it reads or writes any argument.  Stream order is
 *     unchanged.
 *   - Resources: the library allocates no device memory.  Its per-device state is
 *     a small status word in the module's global memory plus host-side caches of
 *     device attributes; they live until the process exits, so there is no
 *     initialisation or shutdown call.
 */
#ifndef DG_H_
#define DG_H_

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DG_OK = 0,
    DG_ERR_INVALID_ARG = 1,        /* null pointer where data is needed, bad enum */
    DG_ERR_SHAPE = 2,              /* a size outside the shape contract below */
    DG_ERR_ALIGNMENT = 3,          /* a pointer not aligned as required */
    DG_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not compute capability 10.0 */
    DG_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
    DG_ERR_TIMEOUT = 6,            /* device: a pipeline wait ran past its limit */
    DG_ERR_GROUP_OFFSETS = 7       /* device: group_offsets broke its contract; nothing was computed */
} dg_status_t;

/*
 * BF16 -> E4M3 block quantizer (2kiu.com/news/5461879 §2.1 block-wise scaling,
 * §3.3 FP32 scales; activation scales recomputed on every call, §4/§5).
 *
 * For each 128x128 block of X (edge blocks hold only the elements present):
 *   amax = max |x|;  s = amax / 448 rounded to FP32 (s = 1 when amax == 0);
 *   q = x / s rounded to FP32, then to the nearest E4M3 value (ties to the even
 *       code, magnitudes above 448 saturate to 448, the sign of zero is kept).
 *
 * X_bf16 : [rows][cols] BF16, 16-byte aligned.
 * Q      : [rows][cols] E4M3 bytes out, 16-byte aligned.
 * S      : [ceil(rows/128)][ceil(cols/128)] FP32 out, 4-byte aligned.
 * rows >= 0, cols >= 0, cols % 16 == 0.  rows == 0 or cols == 0 is a no-op.
 * The result is bit-identical to the definition above.
 */
dg_status_t dg_quantize_blockwise(const void *X_bf16, int64_t rows, int64_t cols,
                                  uint8_t *Q, float *S, cudaStream_t stream);

/*
 * dg_quantize_blockwise for the masked MoE layout (the activations of
 * dg_fp8_grouped_gemm_masked): X holds G slabs of M_max rows, slab g holds
 * masked_m[g] tokens in its first rows (counts outside [0, M_max] are clamped),
 * and each slab's tokens are quantized as dg_quantize_blockwise would quantize the
 * masked_m[g]-row matrix of them alone: the amax of the last token block covers
 * its tokens only, rows past the count are neither read nor written, and the
 * 128-row blocks at or past ceil(masked_m[g] / 128) are skipped (their scales are
 * not written).  So no code or scale depends on the rows past a count, which may
 * hold anything, and the work follows the tokens, not the slabs
 * (2kiu.com/news/5461879 §2.2: only M varies between experts and it changes from
 * call to call).
 *
 * X_bf16   : [G][M_max][cols] BF16, 16-byte aligned.
 * masked_m : DEVICE int32 [G], 4-byte aligned (may be produced on `stream`).
 * Q        : [G][M_max][cols] E4M3 out, 16-byte aligned.
 * S        : [G][ceil(M_max/128)][ceil(cols/128)] FP32 out, 4-byte aligned.
 * 1 <= G <= 1024, M_max >= 0, cols % 16 == 0.  M_max == 0 or cols == 0 is a no-op.
 */
dg_status_t dg_quantize_blockwise_masked(const void *X_bf16, int G, int64_t M_max, int64_t cols,
                                         const int32_t *masked_m, uint8_t *Q_e4m3, float *S,
                                         cudaStream_t stream);

/*
 * Dense block-scaled GEMM, C = A * B^T (2kiu.com/news/5461879 §2.1, §3.3;
 * demingchina.com/news/60142 §3.1, §3.3):
 *   C[m][n] = bf16( sum_kb sA[m/128][kb] * sB[n/128][kb] *
 *                   sum_{k in block kb} A[m][k] * B[n][k] )
 *
 * A  : [M][K] E4M3, 16-byte aligned.     sA : [ceil(M/128)][ceil(K/128)] FP32.
 * B  : [N][K] E4M3, 16-byte aligned.     sB : [ceil(N/128)][ceil(K/128)] FP32.
 * C  : [M][N] BF16 out, 16-byte aligned.
 * M >= 0, N >= 0 with N % 16 == 0, K > 0 with K % 16 == 0 (a row is a whole
 * number of 16-byte units).  When K % 128 != 0 the last K block is partial: it
 * holds the K % 128 columns present and has its own scales, as
 * dg_quantize_blockwise produces them (each K step clipped to what remains,
 * demingchina.com/news/60142 §6.3).
 * M == 0 or N == 0 is a no-op.  M <= 128 takes the skinny split-K kernel,
 * larger M the persistent single-CTA tile kernel (128 x 256 tiles; a last round
 * of tiles that would leave at least half the SMs idle runs as 128 x 128 halves);
 * both compute the same formula.
 */
dg_status_t dg_fp8_gemm_blockscaled(const uint8_t *A, const float *sA,
                                    const uint8_t *B, const float *sB, void *C_bf16,
                                    int64_t M, int64_t N, int64_t K, cudaStream_t stream);

/*
 * Block-scaled GEMM from BF16 activations: A is quantized per 128x128 block
 * exactly as dg_quantize_blockwise does (same codes, same scales, bit for bit),
 * then C = A * B^T as in dg_fp8_gemm_blockscaled.  Activation scales are
 * recomputed on every call while weight scales are computed once
 * (2kiu.com/news/5461879 §5), so this is the call a layer makes per step.
 *
 * A_bf16 : [M][K] BF16, 16-byte aligned.
 * B, sB  : as in dg_fp8_gemm_blockscaled (quantized once, e.g. by dg_quantize_blockwise).
 * C      : [M][N] BF16 out, 16-byte aligned.
 * QA     : [M][K] E4M3 out, 16-byte aligned; sA : [ceil(M/128)][ceil(K/128)] FP32 out.
 *          Caller-owned: they receive A's codes and scales (the library allocates
 *          nothing).
 * Shapes as in dg_fp8_gemm_blockscaled (N % 16 == 0, K % 16 == 0, K > 0).
 * Runs the block quantizer, then dg_fp8_gemm_blockscaled's kernel, on `stream`;
 * the quantizer lets the GEMM start its set-up and weight prefetch while it
 * runs.  (The one-launch form, DG_KERNEL_SKINNY_FUSED in
 * dg_fp8_gemm_blockscaled_bf16a_select, measured no faster for any M.)
 * M == 0 or N == 0 is a no-op.
 */
dg_status_t dg_fp8_gemm_blockscaled_bf16a(const void *A_bf16, const uint8_t *B, const float *sB,
                                          void *C_bf16, uint8_t *QA, float *sA,
                                          int64_t M, int64_t N, int64_t K, cudaStream_t stream);

/*
 * MoE grouped-contiguous block-scaled GEMM (nxmr.cn/news/132300 §2.2;
 * 2kiu.com/news/5461879 §2.2): expert g owns rows [off[g], off[g+1]) of A and
 * C, every off[g] a multiple of 128, and for those rows
 *   C[m][n] = bf16( sum_kb sA[m/128][kb] * sB[g][n/128][kb] *
 *                   sum_k A[m][k] * B[g][n][k] ).
 * Padding rows inside an expert's range are computed like real rows (zero rows
 * of A give zero rows of C).  Rows at or beyond off[G] are not written.
 *
 * A  : [M_total_capacity][K] E4M3.        sA : [M_total_capacity/128][ceil(K/128)] FP32.
 * B  : [G][N][K] E4M3.                    sB : [G][N/128][ceil(K/128)] FP32.
 * C  : [M_total_capacity][N] BF16 out.
 * group_offsets : DEVICE int32 [G+1], off[0] == 0, non-decreasing, each a
 *                 multiple of 128, off[G] <= M_total_capacity.  Read on the
 *                 device, so it may be produced by an earlier kernel on `stream`.
 *                 The kernel checks these rules before it computes anything; an
 *                 array that breaks one leaves C untouched and records
 *                 DG_ERR_GROUP_OFFSETS in the device status word
 *                 (dg_get_last_device_status); the call itself returns DG_OK.
 * M_total_capacity % 128 == 0, 1 <= G <= 1024, N % 128 == 0, K % 16 == 0, K > 0
 * (a partial last K block as in dg_fp8_gemm_blockscaled).
 * M_total_capacity == 0 or N == 0 is a no-op.
 */
dg_status_t dg_fp8_grouped_gemm_contiguous(const uint8_t *A, const float *sA,
                                           const uint8_t *B, const float *sB,
                                           void *C_bf16, const int32_t *group_offsets,
                                           int64_t M_total_capacity, int G,
                                           int64_t N, int64_t K, cudaStream_t stream);

/*
 * Per-token activation quantizer: one FP32 scale per row and 128-column group
 * ("per-group, 128 elements a group", demingchina.com/news/60142 §5.2), with the
 * same arithmetic as dg_quantize_blockwise on that 1 x 128 block:
 *   s = fl32(amax / 448) (1 if amax == 0);  q = E4M3_rn_satfinite(fl32(x / s)).
 *
 * X_bf16 : [rows][cols] BF16, 16-byte aligned.
 * Q      : [rows][cols] E4M3 out, 16-byte aligned.
 * S_t    : [ceil(cols/128)][rows] FP32 out, K-block-major (the transpose of the
 *          natural [rows][groups]): the layout dg_fp8_gemm_1x128 reads.
 * rows >= 0, cols >= 0, cols % 16 == 0; an empty matrix is a no-op.
 */
dg_status_t dg_quantize_1x128(const void *X_bf16, int64_t rows, int64_t cols,
                              uint8_t *Q, float *S_t, cudaStream_t stream);

/*
 * Block-scaled GEMM with per-token A scales (demingchina.com/news/60142 §5.2)
 * and 128x128 B scales:
 *   C[m][n] = bf16( sum_kb sA_t[kb][m] * sB[n/128][kb] *
 *                   sum_{k in block kb} A[m][k] * B[n][k] )
 *
 * A    : [M][K] E4M3.            sA_t : [ceil(K/128)][M] FP32 (from dg_quantize_1x128).
 * B, sB, C and the shape rules as in dg_fp8_gemm_blockscaled.
 * Runs the single-CTA tile kernel.
 */
dg_status_t dg_fp8_gemm_1x128(const uint8_t *A, const float *sA_t,
                              const uint8_t *B, const float *sB, void *C_bf16,
                              int64_t M, int64_t N, int64_t K, cudaStream_t stream);

/*
 * MoE masked grouped block-scaled GEMM (2kiu.com/news/5461879 §2.2: the experts
 * share N and K, only M varies, and from call to call): expert g owns a slab of
 * M_max rows of A and C and uses its first masked_m[g] rows, a count read on the
 * device (so an earlier kernel on `stream` may write it, with no host sync).
 * For those rows
 *   C[g][m][n] = bf16( sum_kb sA[g][m/128][kb] * sB[g][n/128][kb] *
 *                      sum_k A[g][m][k] * B[g][n][k] ).
 * Only m-blocks holding tokens are computed; rows at or past masked_m[g] of C
 * are not written, and rows past masked_m[g] of A may hold anything.
 *
 * A  : [G][M_max][K] E4M3, 16-byte aligned.  sA : [G][ceil(M_max/128)][ceil(K/128)] FP32.
 * B  : [G][N][K] E4M3.                       sB : [G][N/128][ceil(K/128)] FP32.
 * C  : [G][M_max][N] BF16 out.
 * masked_m : DEVICE int32 [G]; counts outside [0, M_max] are clamped to it.
 * 1 <= G <= 256, M_max >= 0, N % 128 == 0, K % 16 == 0, K > 0.
 * M_max == 0 or N == 0 is a no-op.
 */
dg_status_t dg_fp8_grouped_gemm_masked(const uint8_t *A, const float *sA,
                                       const uint8_t *B, const float *sB,
                                       void *C_bf16, const int32_t *masked_m, int G,
                                       int64_t M_max, int64_t N, int64_t K, cudaStream_t stream);

/*
 * Kernel selection for the dense GEMM, for tests and measurement.  AUTO is the
 * dispatch dg_fp8_gemm_blockscaled uses: SKINNY for M <= 128, else TILE.
 *   TILE    persistent single-CTA kernel, 128 x 256 (128 x 128 if N <= 128) tiles;
 *   SKINNY  split-K kernel for M <= 128 (larger M gives DG_ERR_SHAPE);
 *   PAIR    persistent CTA-pair kernel, 256 x 256 (256 x 128 if N <= 128) tiles.
 * TILE and PAIR run a last round that would leave at least half the SMs idle as
 * half-width tiles.
 */
typedef enum {
    DG_KERNEL_AUTO = 0,
    DG_KERNEL_TILE = 1,
    DG_KERNEL_SKINNY = 2,
    DG_KERNEL_PAIR = 3,
    DG_KERNEL_SKINNY_FUSED = 4 /* dg_fp8_gemm_blockscaled_bf16a_select only */
} dg_kernel_t;

dg_status_t dg_fp8_gemm_blockscaled_select(const uint8_t *A, const float *sA,
                                           const uint8_t *B, const float *sB, void *C_bf16,
                                           int64_t M, int64_t N, int64_t K,
                                           dg_kernel_t kernel, cudaStream_t stream);

/*
 * dg_fp8_gemm_blockscaled_bf16a with the kernel chosen, for tests and measurement.
 * AUTO, TILE, SKINNY, PAIR: the block quantizer, then that GEMM kernel.
 * SKINNY_FUSED (M <= 16, else DG_ERR_SHAPE): one launch of the skinny kernel,
 * whose four extra warps quantize A's K blocks straight into the MMA's stages
 * (same codes and scales, bit for bit; the CTAs of the first N block also write
 * QA and sA).  2kiu.com/news/5461879 §5: activation scales are recomputed on
 * every call.
 */
dg_status_t dg_fp8_gemm_blockscaled_bf16a_select(const void *A_bf16, const uint8_t *B, const float *sB,
                                                 void *C_bf16, uint8_t *QA, float *sA,
                                                 int64_t M, int64_t N, int64_t K,
                                                 dg_kernel_t kernel, cudaStream_t stream);

/* dg_fp8_gemm_1x128 with the kernel chosen: AUTO, TILE or PAIR (SKINNY gives
 * DG_ERR_INVALID_ARG), for tests and measurement. */
dg_status_t dg_fp8_gemm_1x128_select(const uint8_t *A, const float *sA_t,
                                     const uint8_t *B, const float *sB, void *C_bf16,
                                     int64_t M, int64_t N, int64_t K, dg_kernel_t kernel,
                                     cudaStream_t stream);

/* Human-readable name of a status code (static storage). */
const char *dg_status_string(dg_status_t status);

/*
 * Returns the device status word recorded by kernels of this library on the
 * current device since the previous call (DG_OK if none) and clears it: a small
 * kernel on `stream` swaps the word with zero atomically, so a failure recorded
 * concurrently is kept for the next call, not lost; then `stream` is
 * synchronised.  Failures of kernels on other streams are covered once those
 * kernels have completed (synchronise them first).
 */
dg_status_t dg_get_last_device_status(cudaStream_t stream);

/* Library ABI version (major * 100 + minor).  1.01 added the BF16-activation,
 * per-token-scale and masked-MoE calls; 1.02 added DG_ERR_GROUP_OFFSETS; 1.03
 * added dg_fp8_gemm_blockscaled_bf16a_select and DG_KERNEL_SKINNY_FUSED; 1.04 added
 * dg_quantize_blockwise_masked; 1.05: dg_quantize_blockwise_masked quantizes each
 * expert's tokens as a matrix of their own (rows past the count no longer enter the
 * last token block's amax).  Every 1.00 call is unchanged. */
int dg_version(void);

/*
 * Test-only control of the kernels' failure detection.  Every wait inside the
 * kernels gives up after timeout_ns nanoseconds (0 restores the default of 2 s),
 * records DG_ERR_TIMEOUT in the device status word and lets the kernel finish
 * cleanly.  debug_flags bit 0 makes the TMA producer of the tile, pair and skinny
 * kernels skip its first shared-memory stage, so that the MMA warp's wait runs
 * out: it exercises the timeout path without faulting or hanging the GPU.
 * Applies to launches made after the call, process-wide; not for production use.
 */
void dg_test_set_kernel_control(uint64_t timeout_ns, int debug_flags);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */
