/*
 * bi_quantize.h -- C ABI of the e2m1 (FP4) weight quantisation (libbigemm.so).
 *
 * The pages' FP4 weights are quantised per output channel as W_fp4 = round((W - zero) / scale),
 * with a scale 2^-j (j = 1 .. 12) and a zero point that fp16 represents exactly, so that the
 * dequantisation W_fp4 * scale + zero is exact ("DeepSeek V4的batch invariance：大模型确定性推理的工程
 * 基石" (lshu.cn), section 4.3).  This call produces the packed e2m1 weights that
 * bi_gemm_run_w4a8 (bi_gemm.h) takes, with the same per-channel w_scale and w_zero.
 *
 * For every n < N and k < K:
 *   x = (W[n][k] - w_zero[n]) / w_scale[n], formed in fp64 from the 16-bit weight, and
 *   q[n][k] = the e2m1 value nearest x (0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6), a tie going to
 *             the value with fraction bit 0; |x| beyond 6 saturates to +-6; the sign bit follows
 *             the sign of x (a negative x that rounds to zero gives -0); NaN gives +0.
 * "round" is read as the IEEE round-to-nearest-even the pages fix for their GEMM
 * ("DeepSeek V4 的隐藏关键特性被挖出来了" (wmrh.cn), section 3.1), and saturation as the clamp any
 * finite format needs.  The codes are written packed: value k of row n in byte k/2 of row n of Q,
 * the even k in the low four bits.  The result depends on each weight and its channel's
 * constants only.
 *
 * Arguments (device pointers, owned by the caller; asynchronous on `stream`):
 *   W        16-bit weights [N][ldw]: bf16 (w_is_fp16 = 0) or fp16 (w_is_fp16 = 1), 2-byte aligned
 *   w_scale  fp32 [N] (any non-zero value is accepted here; bi_gemm_run_w4a8 requires 2^-j)
 *   w_zero   fp32 [N], or NULL for zero points 0
 *   Q        packed e2m1 [N][ldq / 2 bytes]; ldq (in values) >= K and even
 * K must be even.  N = 0 or K = 0 is a no-op returning BI_OK.
 * Errors: BI_ERR_INVALID_ARG (null pointers, negative sizes, odd K or ldq, ldw < K, ldq < K,
 * w_is_fp16 not 0 or 1), BI_ERR_ALIGNMENT (W not 2-byte, w_scale / w_zero not 4-byte aligned),
 * BI_ERR_NO_DEVICE, BI_ERR_CUDA.
 */
#ifndef BI_QUANTIZE_H
#define BI_QUANTIZE_H

#include <stdint.h>

#include <cuda_runtime.h>

#include "bi_gemm.h"

#ifdef __cplusplus
extern "C" {
#endif

bi_status_t bi_quantize_e2m1(const void *W, int w_is_fp16, int64_t ldw, int64_t N, int64_t K,
                             const float *w_scale, const float *w_zero, void *Q, int64_t ldq,
                             cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BI_QUANTIZE_H */
