/*
 * bi_attention.h -- C ABI of the dual-kernel decode attention (libbigemm.so).
 *
 * The pages pair their batch-invariant GEMM with decode attention built as two kernels: one
 * that splits a sequence's keys over several CTAs and merges the parts in a fixed binary tree,
 * and one that does not split, with bit-identical outputs, so that a runtime switch between them
 * changes no bit ("DeepSeek V4的batch invariance：大模型确定性推理的工程基石" (lshu.cn), section
 * 4.1; "DeepSeek V4 的隐藏关键特性被挖出来了" (wmrh.cn), section 3.3).
 *
 * Computation, for each sequence b and query head h (grouped-query attention: query head h reads
 * key/value head h / (Hq / Hkv)):
 *   s_j = scale * (q . k_j) over the sequence's keys j < L_b,
 *   O[b][h] = sum_j softmax(s)_j * v_j, rounded once to bf16.
 * The reduction order is fixed by L_b alone: the keys are cut into 4 chunks
 * [floor(c L_b / 4), floor((c+1) L_b / 4)), each chunk is reduced by the same code (blocks of 32
 * keys in ascending order, scores in a fixed summation order, an online softmax with fixed-order
 * warp reductions), and the 4 chunk
 * results are merged as ((c0 + c1) + (c2 + c3)).  `splits` only decides how many CTAs share a
 * sequence's chunks -- 1 (no split: one CTA walks all 4 chunks), 2 or 4 (split-KV: 2 or 4 CTAs,
 * then a merge kernel) -- so every value of `splits` gives the same bits, and a sequence's output
 * does not depend on the other sequences of the batch.
 */
#ifndef BI_ATTENTION_H
#define BI_ATTENTION_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime.h>

#include "bi_gemm.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of fp32 workspace bi_decode_attention needs: 0 for splits = 1, else
 * B * Hq * 4 * (D + 2) * 4 (one (max, sum, D-vector) partial per chunk). */
size_t bi_decode_attention_workspace_bytes(int64_t B, int Hq, int D, int splits);

/*
 * Decode attention, one query per sequence.  Device pointers, bf16 unless noted:
 *   Q [B][Hq][D], K and V [B][Lmax][Hkv][D] (sequence b's keys are rows 0 .. L_b - 1),
 *   lengths: int32 [B] on the device, 1 <= L_b <= Lmax,  O [B][Hq][D].
 * scale: the score scale (e.g. 1/sqrt(D)).  D = 128, Hq a multiple of Hkv with Hq / Hkv <= 8.
 * splits: 1, 2 or 4 (see above); workspace: fp32, at least
 * bi_decode_attention_workspace_bytes(B, Hq, D, splits) bytes (may be NULL for splits = 1).
 * Pointers 16-byte aligned.  Lengths outside [1, Lmax] make the sequence's output NaN.
 * Errors: BI_ERR_INVALID_ARG, BI_ERR_ALIGNMENT, BI_ERR_UNSUPPORTED_SHAPE (D != 128, bad head
 * counts), BI_ERR_NO_DEVICE, BI_ERR_CUDA.
 */
bi_status_t bi_decode_attention(const void *Q, const void *K, const void *V,
                                const int32_t *lengths, int64_t B, int Hq, int Hkv, int D,
                                int64_t Lmax, float scale, int splits, float *workspace,
                                size_t workspace_bytes, void *O, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BI_ATTENTION_H */
