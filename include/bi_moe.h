/*
 * bi_moe.h -- C ABI of the MoE steps either side of the grouped GEMM (libbigemm.so).
 *
 * The pages name MoE among DeepSeek V4's components ("DeepSeek不惜代价保住它！V4关键特性被挖出来了"
 * (QbitAI), on what V4 is built from) and require every token's output to be independent of the
 * batch it shares.  They give no routing formula.  The workload these steps serve routes each
 * token to the top k experts by router logit (softmax over all experts; k = 8 for the MoE
 * workload), groups the (token, slot) pairs by expert for bi_grouped_gemm_run, and combines the
 * k expert outputs of each token weighted by its softmax probabilities.
 *
 * Every step is deterministic and T-invariant: a token's experts, weights, rows and combined
 * output depend only on that token's logits and rows, never on T or on the other tokens; no step
 * uses atomics, and every reduction has a fixed order.
 *
 * Pointers are device pointers owned by the caller; calls are asynchronous on `stream`.  Status
 * codes are those of bi_gemm.h.  T = 0 is a no-op returning BI_OK.
 */
#ifndef BI_MOE_H
#define BI_MOE_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime.h>

#include "bi_gemm.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Router: for each token t (row t of logits [T][ld_logits], fp32, finite), the k experts with
 * the largest logits, in descending logit order, ties to the lower expert index, into
 * experts[t*k + j] (int32); and their softmax probabilities over all E experts,
 * p_e = exp(l_e - max) / sum_e' exp(l_e' - max), into weights[t*k + j] (fp32).  The sum runs in a
 * fixed order (each lane's experts in ascending index, then a fixed butterfly across lanes).
 * Limits: 1 <= k <= 8, k <= E <= 1024.
 * Errors: BI_ERR_INVALID_ARG (null pointers, bad sizes, ld_logits < E), BI_ERR_ALIGNMENT
 * (pointers not 4-byte aligned), BI_ERR_NO_DEVICE, BI_ERR_CUDA.
 */
bi_status_t bi_moe_route_topk(const float *logits, int64_t ld_logits, int64_t T, int E, int k,
                              int32_t *experts, float *weights, cudaStream_t stream);

/*
 * Dispatch: stable grouping of the T*k (token, slot) pairs by expert.  Pair i = t*k + j goes to
 * row r_i of the grouped order, where rows are ordered by expert and, inside an expert, by i.
 * Writes offsets[E+1] (offsets[0] = 0, offsets[e+1] - offsets[e] = pairs routed to e),
 * token_of_row[r_i] = t and row_of_slot[i] = r_i.  Expert ids outside [0, E) are not counted and
 * leave offsets[E] below T*k (their row_of_slot entries are not written).
 * Limits: 1 <= k <= 8, 1 <= E <= 1024, T*k < 2^31.
 * Errors: BI_ERR_INVALID_ARG, BI_ERR_ALIGNMENT, BI_ERR_NO_DEVICE, BI_ERR_CUDA.
 */
bi_status_t bi_moe_dispatch(const int32_t *experts, int64_t T, int E, int k, int32_t *offsets,
                            int32_t *token_of_row, int32_t *row_of_slot, cudaStream_t stream);

/*
 * Gather: A_perm[r][0:K] = X[token_of_row[r]][0:K] for r < R (bf16 rows; X [T][ldx], A_perm
 * [R][lda]), the grouped GEMM's A.  token_of_row entries must lie in [0, T) (not checked on the
 * device).  Pointers 16-byte aligned, ldx and lda multiples of 8 elements.
 * Errors: BI_ERR_INVALID_ARG, BI_ERR_ALIGNMENT, BI_ERR_NO_DEVICE, BI_ERR_CUDA.
 */
bi_status_t bi_moe_gather_rows(const void *X, int64_t ldx, int64_t K, const int32_t *token_of_row,
                               int64_t R, void *A_perm, int64_t lda, cudaStream_t stream);

/*
 * Combine: Y[t][n] = bf16_rne(acc) with acc = fma(w_{k-1}, c_{k-1}, ... fma(w_1, c_1,
 * fma(w_0, c_0, 0)) ...), w_j = weights[t*k + j] and c_j = C_perm[row_of_slot[t*k + j]][n]: the
 * token's expert outputs in slot order (descending router logit), fp32 accumulation.
 * C_perm [R][ldc] bf16 (the grouped GEMM's C), Y [T][ldy] bf16; pointers 16-byte aligned, ldc and
 * ldy multiples of 8 elements.  row_of_slot entries must be valid rows of C_perm.
 * Errors: BI_ERR_INVALID_ARG, BI_ERR_ALIGNMENT, BI_ERR_NO_DEVICE, BI_ERR_CUDA.
 */
bi_status_t bi_moe_combine(const void *C_perm, int64_t ldc, int64_t N, const int32_t *row_of_slot,
                           const float *weights, int64_t T, int k, void *Y, int64_t ldy,
                           cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BI_MOE_H */
