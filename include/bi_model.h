/*
 * bi_model.h -- C ABI of the batch-invariant dense layers of the policy model: the bf16 GEMM of a
 * linear layer and RMSNorm.  Same library (libbi_isloss.so), status codes and conventions as
 * bi_isloss.h.
 *
 * Sources (page titles and sections):
 *   "Zero Mismatch, Simple Async RL", section "Only one probability gap comes from old weights":
 *       kernel selection by batch shape, reduction order and different prefill/decode arithmetic
 *       change logprobs although the parameters are the same.
 *   "Zero Mismatch, Simple Async RL", section "Large-model validation exposes concrete failure
 *       mechanisms": shape-selected library kernels are a source of batch variance.
 *   "REINFORCE Zero: 为什么内核对齐后...", the paragraph before Fig. 2: trainer-inference invariance
 *       removes the kernel-mismatch term with batch-invariant kernels and a matched forward pass.
 *
 * Batch invariance: every output row depends only on its own input row and the weights.  The same
 * kernel serves every M (one row alone, as in decode, or 10^5 packed rows, as in prefill or the
 * learner): one tile shape, a fixed reduction order, no split of the reduction across CTAs, no
 * atomics.  Rows are therefore bit-identical whatever batch they sit in and wherever they sit.
 *
 * Conventions: device pointers owned by the caller, bf16 passed as uint16_t bit patterns,
 * row-major; work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) without
 * synchronising; the library allocates nothing.  The return value reports host-visible errors
 * (nothing is launched unless it is BI_OK); *dev_status (device int32) is set to BI_OK and raised
 * by the kernel to BI_ERR_TIMEOUT if a bounded wait ran out (outputs then undefined).  Kernels
 * never trap.
 */
#ifndef BI_MODEL_H
#define BI_MODEL_H

#include "bi_isloss.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Y = X W^T: the linear layer y_m = W x_m.
 *   x   [M, K] bf16   input rows                       16-byte aligned
 *   w   [N, K] bf16   weight, one row per output        16-byte aligned
 *   y   [M, N] bf16   output, fp32 accumulation rounded to nearest even; overwritten
 *   M   >= 0 and <= 2^31 - 256 (M = 0 launches nothing and leaves *dev_status = BI_OK)
 *   N   > 0, a multiple of 8 and < 2^31;  K > 0, a multiple of 8 and < 2^31
 * Tiling: 256 x 256 output tiles on CTA pairs (tcgen05 M = 256 instructions), K in chunks of 64
 * taken in increasing order; the same for every M.
 * Returns BI_ERR_INVALID_ARG for a NULL or misaligned pointer, BI_ERR_UNSUPPORTED_SHAPE for N or
 * K outside the rules above, BI_ERR_CUDA when the device set-up or the launch fails.
 */
BI_API bi_status bi_gemm_bf16(const uint16_t* x, const uint16_t* w, uint16_t* y, int64_t M, int32_t N, int32_t K,
                              int32_t* dev_status, void* stream);

/*
 * RMSNorm: y_m = x_m / sqrt(mean_j x_mj^2 + eps) * g, row by row.
 *   x   [M, H] bf16   16-byte aligned;   g [H] bf16 gain, 16-byte aligned
 *   y   [M, H] bf16   output (may not alias x), 16-byte aligned
 *   eps >= 0 and finite;  M >= 0;  H > 0 and a multiple of 8
 * Arithmetic: fp32; the sum of squares of a row in a fixed order (a fixed per-lane order, then a
 * fixed shuffle tree whose lane-0 total the whole row uses), r = rsqrt(ss / H + eps),
 * y = bf16((x r) g).
 * Returns BI_ERR_INVALID_ARG for a NULL or misaligned pointer, aliasing x and y, or a negative or
 * non-finite eps; BI_ERR_UNSUPPORTED_SHAPE for H; BI_ERR_CUDA when the launch fails.
 */
BI_API bi_status bi_rmsnorm(const uint16_t* x, const uint16_t* g, float eps, uint16_t* y, int64_t M, int32_t H,
                            int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BI_MODEL_H */
