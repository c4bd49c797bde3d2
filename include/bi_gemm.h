/*
 * bi_gemm.h -- C ABI of libbigemm, a batch-invariant GEMM for NVIDIA B200 (sm_100a).
 *
 *   C[M,N] = A[M,K] . B[N,K]^T          (alpha = 1, beta = 0, fp32 accumulation, bf16 output)
 *
 * Batch invariance: for a fixed plan, the bits of output row C[m,:] are a function of A[m,:],
 * B (and, for FP8, the row's scales scale_a[:,m] and scale_b) only.  They do not depend on M,
 * on m, on the other rows of A, on the expert offsets of a grouped call, on the stream, on the
 * grid or on device occupancy.  This is the property defined in "DeepSeek不惜代价保住它！V4关键
 * 特性被挖出来了" (QbitAI), section "什么是batch invariance": one token's output is bit-identical
 * whatever its position in the batch, the batch size and its batch-mates.  The same article
 * (section "牺牲了什么") attributes it to dropping split-K in a custom GEMM: a split K axis is
 * summed in an order that changes with the split, and floating-point addition does not
 * associate.  The library therefore never splits K: one CTA owns the whole K range of its output
 * tile and walks it in ascending 128-byte blocks, and the tile shape, MMA instruction shape and
 * K order are fixed by the plan, a pure function of (N, K, dtype, num_experts) that never sees M.
 * There are no atomics on the data path.
 *
 * Memory and ownership.  The caller owns every buffer and the stream.  Device pointers must
 * point to memory of the current CUDA device.  A plan is host state plus, created lazily at the
 * first run on a device, one 4-byte device status word per device; nothing else allocates on
 * the run path.  All run calls are asynchronous on `stream` (NULL = the legacy default stream)
 * and do not synchronise.
 *
 * Errors.  Every entry point returns a bi_status_t; nothing throws across the ABI, calls exit or
 * abort, or traps on the device.  Invalid arguments are rejected before any launch.  Launch
 * failures map to BI_ERR_CUDA.  Device-side failures (a pipeline wait that exceeded its time
 * limit, malformed grouped offsets) are written to the plan's status word and reported by
 * bi_gemm_sync_status.
 *
 * Layouts (all row-major, strides in elements):
 *   A        [M][lda]   K-contiguous, bf16 or e4m3; lda >= K
 *   B        [N][ldb]   K-contiguous ("B^T" form, the weight layout); ldb >= K
 *   C        [M][ldc]   bf16, N-contiguous; ldc >= N
 *   scale_a  (FP8 only) fp32, K-block-major: the scale of row m and K block kb (columns
 *            128*kb .. 128*kb+127) is scale_a[kb*ld_sa + m]; ld_sa >= M
 *   scale_b  (FP8 only) fp32 [ceil(N/128)][ceil(K/128)] row-major: one scale per 128x128 block
 * Alignment: A, B, C must be 16-byte aligned, and lda*elt, ldb*elt, ldc*2 must be multiples of
 * 16 bytes (elt = 2 for bf16, 1 for e4m3).  scale_a and scale_b need 4-byte alignment.
 */
#ifndef BI_GEMM_H
#define BI_GEMM_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BI_GEMM_ABI_VERSION 1

typedef enum {
    BI_DTYPE_BF16 = 0,              /* A, B bf16; C bf16 */
    BI_DTYPE_E4M3_BLOCKSCALED = 1,  /* A, B e4m3 (fn) with fp32 block scales; C bf16 */
    BI_DTYPE_E2M1_W4A8 = 2          /* A e4m3 with fp32 block scales, B packed e2m1 weights with a
                                       power-of-two scale and a zero point per output column;
                                       C bf16 (bi_gemm_run_w4a8) */
} bi_dtype_t;

typedef enum {
    BI_OK = 0,
    BI_ERR_INVALID_ARG = 1,         /* null pointer, negative size, stride below the extent */
    BI_ERR_ALIGNMENT = 2,           /* pointer or stride not 16-byte aligned */
    BI_ERR_UNSUPPORTED_SHAPE = 3,   /* a size outside what the plan supports */
    BI_ERR_DTYPE_MISMATCH = 4,      /* scales given to a bf16 plan, missing for FP8, ... */
    BI_ERR_CUDA = 5,                /* a CUDA runtime/driver call failed */
    BI_ERR_DEVICE_TIMEOUT = 6,      /* a device pipeline wait exceeded its limit */
    BI_ERR_BAD_OFFSETS = 7,         /* grouped offsets not 0 .. total_rows non-decreasing */
    BI_ERR_NO_DEVICE = 8            /* no CUDA device, or the device is not sm_100 */
} bi_status_t;

/* Opaque, library-owned plan. */
typedef struct bi_plan_s *bi_plan_t;

/* What a plan fixed.  None of it depends on M, except the scheduling, which is reported for a
 * full-height tile: a launch whose whole problem has fewer rows than one tile sizes its A slots
 * to those rows and deepens both rings; a bf16 64 x 32 (FP8 128 x 64) plan groups 8 (4) K chunks
 * per pipeline stage when A has at most 32 (64) rows, and the bf16 plan 16 below 8 rows; and a
 * launch with more tiles than SMs runs two or four adjacent tiles in lockstep, with one
 * instruction as wide as those tiles together.  The tile, the instruction's M and K and the K
 * order are fixed, and tcgen05 computes each output element the same way whatever the
 * instruction's N, so no row's result changes. */
typedef struct {
    int64_t n, k;              /* the plan's N and K */
    int dtype;                 /* bi_dtype_t */
    int num_experts;           /* 1 = dense */
    int block_m;               /* output rows per tile */
    int block_n;               /* output columns per tile */
    int block_k;               /* K elements per pipeline stage (1, 2 or 4 chunks of 128 bytes) for
                                  a full-height tile */
    int cta_group;             /* CTAs that share one MMA (1 or 2) */
    int mma_m, mma_n, mma_k;   /* tcgen05.mma instruction shape */
    int stages;                /* depth of the B (weight) shared-memory ring */
    int k_order_id;            /* 0 = ascending K blocks, whole K per CTA, no split-K;
                                  1 = fixed split-K research plan (see bi_gemm_plan_splitk);
                                  2 = whole K per CTA in two fixed interleaved chains: the
                                      128-byte K chunks 0, 2, 4, ... and 1, 3, 5, ... are each
                                      accumulated in ascending K, then C = chain0 + chain1 once;
                                  3 = whole K per CTA in four fixed interleaved chains: chain c
                                      accumulates the chunks c, c + 4, c + 8, ... in ascending K,
                                      then C = (chain0 + chain1) + (chain2 + chain3) once, chains
                                      that K leaves empty left out (dense bf16 plans of
                                      32-column tiles).
                                  Every order is fixed by K alone: the same for every M, row
                                  position and scheduling form. */
    int threads_per_cta;
    int smem_bytes;            /* dynamic shared memory per CTA */
    int tmem_columns;          /* tensor-memory columns allocated per CTA */
    int stages_a;              /* depth of the A shared-memory ring (<= stages) */
    int k_splits;              /* 1, or the split count of a split-K research plan */
} bi_plan_info_t;

/* Library version check: returns BI_GEMM_ABI_VERSION. */
int bi_gemm_abi_version(void);

/* Human-readable name of a status code (static string; never NULL). */
const char *bi_status_string(bi_status_t status);

/*
 * Create a plan for C = A . B^T with the given N, K and dtype.  num_experts = 1 makes a dense
 * plan; num_experts > 1 makes a grouped (MoE) plan for bi_grouped_gemm_run (bf16 only).
 * The plan is a pure function of its arguments: the same (N, K, dtype, num_experts) gives the
 * same tile configuration in every process and on every device.  It touches no device and can
 * be created on a machine without a GPU.
 * Errors: BI_ERR_INVALID_ARG (out == NULL, N < 0, K < 0, num_experts < 1),
 * BI_ERR_UNSUPPORTED_SHAPE (num_experts > 1024, grouped with FP8 or e2m1, or e2m1 with K not a
 * multiple of 128).
 */
bi_status_t bi_gemm_plan(bi_plan_t *out, int64_t N, int64_t K, bi_dtype_t dtype,
                         int num_experts);

/*
 * A plan for the output columns [n_begin, n_end) of a dense plan (column-parallel sharding: one
 * GPU per column shard, "DeepSeek V4的batch invariance：大模型确定性推理的工程基石" (lshu.cn),
 * section 2.2, on every device computing the same thing).  It keeps `full`'s tile, MMA
 * instruction and K order (and scheduling forms), so column n of C computed with it, from rows
 * [n_begin, n_end) of B, is bit-identical to column n_begin + n of the full GEMM.  (A plan made
 * for the shard's own (N, K) may choose a different tile and K order, and then differ in the
 * last bits.)  Run it like any dense plan with N = n_end - n_begin: B is the shard's [N][ldb]
 * rows, C its [M][ldc] columns; for FP8, scale_b starts at block row n_begin / 128.
 * Errors: BI_ERR_INVALID_ARG for a grouped or split-K plan or a range outside [0, N];
 * BI_ERR_UNSUPPORTED_SHAPE for an FP8 plan and n_begin not a multiple of 128.  The shard plan is
 * independent of `full` once made; destroy it with bi_gemm_plan_destroy.
 */
bi_status_t bi_gemm_plan_column_shard(bi_plan_t *out, bi_plan_t full, int64_t n_begin, int64_t n_end);

/* Destroy a plan and free its device status words.  NULL is accepted. */
bi_status_t bi_gemm_plan_destroy(bi_plan_t plan);

/* Copy the plan's fixed configuration into *info. */
bi_status_t bi_gemm_plan_describe(bi_plan_t plan, bi_plan_info_t *info);

/*
 * Dense GEMM on device memory: C[0:M, 0:N] = A[0:M, 0:K] . B[0:N, 0:K]^T, rounded to bf16 (RNE).
 * For BI_DTYPE_E4M3_BLOCKSCALED the operands are dequantised inside the kernel: the product of
 * K block kb is scaled by scale_a[kb*ld_sa + m] * scale_b[(n/128)*ceil(K/128) + kb] and added to
 * the fp32 accumulator in ascending kb (the fused dequantisation of "DeepSeek V4的batch
 * invariance：大模型确定性推理的工程基石" (lshu.cn), section 3.2).  For bf16, pass
 * scale_a = scale_b = NULL and ld_sa = 0.
 * M = 0 (or N = 0) is a no-op returning BI_OK.  K = 0 writes zeros.
 * Errors: BI_ERR_INVALID_ARG, BI_ERR_ALIGNMENT, BI_ERR_DTYPE_MISMATCH, BI_ERR_NO_DEVICE,
 * BI_ERR_CUDA; a grouped plan returns BI_ERR_INVALID_ARG, a BI_DTYPE_E2M1_W4A8 plan
 * BI_ERR_DTYPE_MISMATCH (it runs through bi_gemm_run_w4a8).
 */
bi_status_t bi_gemm_run(bi_plan_t plan, int64_t M,
                        const void *A, int64_t lda,
                        const void *B, int64_t ldb,
                        void *C, int64_t ldc,
                        const float *scale_a, int64_t ld_sa,
                        const float *scale_b,
                        cudaStream_t stream);

/*
 * Grouped (MoE) GEMM, bf16: rows of A are grouped by expert; expert e owns the rows
 * [offsets[e], offsets[e+1]) and multiplies them with its weight matrix
 * B_e[n][k] = B[(e*N + n)*ldb + k]:   C[r, :] = A[r, :] . B_e^T.
 * expert_offsets is a DEVICE array of E+1 int32 with offsets[0] = 0, non-decreasing,
 * offsets[E] = total_rows; it is read only by the kernel (no host synchronisation).  Malformed
 * offsets make the kernel compute nothing and set BI_ERR_BAD_OFFSETS in the status word.
 * Every row's bits are fixed by the grouped plan alone: they do not depend on total_rows, on the
 * offsets or on the other rows of its expert.  (A grouped plan may choose a different tile from
 * the dense plan of the same N and K; when the two plans' bi_plan_info_t agree, a row also gets
 * the bits a dense call with its expert's B_e would give it.)
 * Errors: as bi_gemm_run; a dense plan returns BI_ERR_INVALID_ARG.
 */
bi_status_t bi_grouped_gemm_run(bi_plan_t plan, int64_t total_rows,
                                const void *A, int64_t lda,
                                const void *B, int64_t ldb,
                                void *C, int64_t ldc,
                                const int32_t *expert_offsets,
                                cudaStream_t stream);

/*
 * e2m1 (FP4) weights x e4m3 (FP8) activations, plan dtype BI_DTYPE_E2M1_W4A8.
 *
 * The weights follow the quantisation of "DeepSeek V4的batch invariance：大模型确定性推理的工程
 * 基石" (lshu.cn), section 4.3: W[n][k] = q[n][k] * w_scale[n] + w_zero[n], where q is an e2m1
 * value (1 sign, 2 exponent bits with bias 1, 1 fraction bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6), the
 * per-channel scale is 2^-j with j in [1, 12] and the zero point is a value fp16 represents
 * exactly, so every dequantised weight is exact.  The activations are as for
 * BI_DTYPE_E4M3_BLOCKSCALED: a[m][k] = e4m3(A[m][k]) * scale_a[(k/128)*ld_sa + m].
 *
 *   C[m][n] = bf16( sum_k a[m][k] * W[n][k] )
 *
 * computed as: the MMA takes the e2m1 codes directly (tcgen05 kind::f8f6f4), each 128-wide K
 * block's partial product is promoted with scale_a alone in ascending kb (acc = fma(P_kb,
 * scale_a[m,kb], acc)), and the column's constants are applied once at the end:
 * C = fma(w_zero[n], rowsum[m], w_scale[n] * acc), with rowsum[m] = sum_k a[m][k] in fp32 in an
 * order fixed by K (32 interleaved slices, each accumulated over kb ascending, then a fixed tree).
 * A power-of-two scale multiplies exactly, so it can leave the K sum.  The bits of C[m, :] depend on row m of A and scale_a, W and the column constants only.
 *
 * Device pointers:
 *   A        e4m3 [M][lda] (lda >= K, 16-byte aligned rows)
 *   scale_a  fp32, K-block-major [K/128][ld_sa], ld_sa >= M
 *   W        packed e2m1 [N][ldw / 2 bytes]: value k of row n is in byte k/2 of the row, the even
 *            k in the low four bits.  ldw (in values) >= K and a multiple of 64; W 32-byte aligned.
 *   w_scale  fp32 [N], each 2^-j with j in [1, 12]
 *   w_zero   fp32 [N] of fp16-exact values, or NULL for no zero points (then C = w_scale * acc)
 *   workspace  fp32 scratch of at least bi_gemm_w4a8_workspace_bytes(M) bytes (16-byte aligned)
 *              for the row sums; needed only with w_zero (may be NULL otherwise)
 *   C        bf16 [M][ldc]
 * K must be a multiple of 128 (the plan refuses others).  A scale outside {2^-1 .. 2^-12} or a
 * zero point fp16 cannot represent is reported on the device: the launch completes and
 * bi_gemm_sync_status returns BI_ERR_INVALID_ARG.
 * Errors: BI_ERR_INVALID_ARG, BI_ERR_ALIGNMENT, BI_ERR_DTYPE_MISMATCH (not a W4A8 plan),
 * BI_ERR_NO_DEVICE, BI_ERR_CUDA.
 */
size_t bi_gemm_w4a8_workspace_bytes(int64_t M);

bi_status_t bi_gemm_run_w4a8(bi_plan_t plan, int64_t M,
                             const void *A, int64_t lda,
                             const float *scale_a, int64_t ld_sa,
                             const void *W, int64_t ldw,
                             const float *w_scale, const float *w_zero,
                             float *workspace, size_t workspace_bytes,
                             void *C, int64_t ldc,
                             cudaStream_t stream);

/*
 * Dense GEMM from host memory: copies A (and scale_a) from the host buffers into the caller's
 * device staging buffers, runs bi_gemm_run on them, and copies C back into C_host, all enqueued
 * on `stream` (cudaMemcpyAsync; pinned host memory makes the copies asynchronous).  B and
 * scale_b are device pointers (resident weights).  A_dev / C_dev / scale_a_dev must be large
 * enough for M*lda, M*ldc and ceil(K/128)*ld_sa elements.  The call returns once everything is
 * enqueued; synchronise `stream` before reading C_host.  Every argument is checked before the
 * first copy is enqueued, so a refused call has enqueued nothing.
 * Errors: as bi_gemm_run, plus BI_ERR_INVALID_ARG for missing staging buffers.
 */
bi_status_t bi_gemm_run_host(bi_plan_t plan, int64_t M,
                             const void *A_host, int64_t lda,
                             const void *B, int64_t ldb,
                             void *C_host, int64_t ldc,
                             const float *scale_a_host, int64_t ld_sa,
                             const float *scale_b,
                             void *A_dev, void *C_dev, float *scale_a_dev,
                             cudaStream_t stream);

/*
 * A batch of dense GEMMs from host memory, pipelined behind the ABI.
 *
 * Each call is the GEMM of bi_gemm_run (C = A . B^T, "DeepSeek V4的batch invariance：大模型确定性
 * 推理的工程基石" (lshu.cn), section 2.1; every row of C bit-identical to the same row computed in
 * any other batch, "DeepSeek不惜代价保住它！V4关键特性被挖出来了" (QbitAI), section "什么是batch
 * invariance") with A, scale_a and C in host memory and B, scale_b on the device:
 *   M, A_host [M][lda], B [N][ldb] (device), C_host [M][ldc] bf16, scale_a_host
 *   [ceil(K/128)][ld_sa] and scale_b (device) as bi_gemm_run (FP8 plans only; NULL for bf16).
 * Each batch owns one region of the staging buffer (batch count % S).  On copy_in its calls' A
 * (and scale_a) are copied into it; with BI_PLAN_HOST_ROW_BLOCKS, calls whose host A rows begin
 * where the previous call's end (a batch laid out back to back in host memory) share one copy.  Once all of the batch's
 * copy-ins have landed, its GEMMs run on compute in call order, writing C into the region.  The
 * C results are copied back to the C_host buffers on copy_out (with that flag, again one copy
 * for calls whose host C rows follow each other) by the second batch call of this plan after it (or by
 * bi_gemm_host_batch_flush): they are queued after that batch's copy-ins and wait for this
 * batch's kernels, which by then have finished.  (A copy-out queued while its kernel is still
 * running holds up the copies queued after it; deferring it lets later copy-ins run under the
 * kernels.)  A region is refilled only after its previous batch's copy-outs have completed.
 * S is the number of regions the staging buffer holds (2 to 32): give it three.  At most 1024
 * calls per batch.
 * The call returns once everything is enqueued.  A batch's results are in host memory once
 * copy_out reaches the copy-outs that a later batch call (or the flush) enqueued:
 * synchronise copy_out after bi_gemm_host_batch_flush to wait for all of them.  Host buffers
 * must stay valid until then; pinned host memory makes the copies asynchronous.  The three
 * streams may be the same stream (no overlap).
 * Staging: caller-owned device memory, 256-byte aligned; bi_gemm_host_batch_staging_bytes(plan,
 * n, calls, S) gives the bytes for S regions of these calls (0 for invalid arguments, more than
 * 1024 calls or S outside 2..32); the library allocates nothing.  Passing a different staging
 * buffer (or a batch whose region has another size) first flushes and makes the copy-ins wait
 * for every copy-out issued so far.  One batch per plan at a time (a plan-wide lock).
 * Stream capture: when compute is capturing, the first batch of the capture forks copy_in and
 * copy_out from compute (copy-outs pending from before the capture must have been flushed, else
 * BI_ERR_INVALID_ARG), the regions are ordered among the capture's own batches, and
 * bi_gemm_host_batch_flush, called before the capture ends, enqueues the last copy-outs and
 * joins both copy streams back into compute.  Replays of the graph are ordered by their stream.
 * Errors: every call's arguments are checked before anything is enqueued (as bi_gemm_run; the
 * scale_a of a call is only copied and may have any alignment); BI_ERR_INVALID_ARG for a
 * missing or short staging buffer, BI_ERR_ALIGNMENT for a misaligned one.  A CUDA failure while
 * enqueueing returns BI_ERR_CUDA with the work before it enqueued.  BI_ERR_INVALID_ARG also for
 * a staging buffer of fewer than two regions or more than 1024 calls.  Grouped, split-K and
 * e2m1 plans are refused.
 */
typedef struct {
    int64_t M;
    const void *A_host;         /* host [M][lda] */
    int64_t lda;
    const void *B;              /* device [N][ldb] */
    int64_t ldb;
    void *C_host;               /* host [M][ldc] bf16 */
    int64_t ldc;
    const float *scale_a_host;  /* FP8: host [ceil(K/128)][ld_sa]; NULL for bf16 */
    int64_t ld_sa;
    const float *scale_b;       /* FP8: device [ceil(N/128)][ceil(K/128)]; NULL for bf16 */
} bi_host_gemm_t;

size_t bi_gemm_host_batch_staging_bytes(bi_plan_t plan, int n, const bi_host_gemm_t *calls,
                                        int regions);

bi_status_t bi_gemm_run_host_batch(bi_plan_t plan, int n, const bi_host_gemm_t *calls,
                                   void *staging, size_t staging_bytes,
                                   cudaStream_t copy_in, cudaStream_t compute,
                                   cudaStream_t copy_out);

/* Enqueue the copy-outs still pending from the plan's last host batches on copy_out (each after
 * its batch's kernels); under stream capture also join copy_in and copy_out back into compute.
 * Returns BI_OK when nothing is pending. */
bi_status_t bi_gemm_host_batch_flush(bi_plan_t plan, cudaStream_t copy_in, cudaStream_t compute,
                                     cudaStream_t copy_out);

/*
 * Dense GEMM from host memory for callers that must not allocate device memory.
 *
 * Some callers cannot call cudaMalloc: their device memory is owned by another allocator (a
 * framework's caching allocator or an inference server's arena that has reserved the GPU), so
 * a stray allocation fails or breaks the owner's accounting, or they run where allocating after
 * start-up is not allowed.  This entry point does what bi_gemm_run_host does, but it takes no
 * device staging buffers and allocates nothing: the device copies of A, scale_a and C and the
 * kernel's status word live in one file-scope device array of BI_NOALLOC_SCRATCH_BYTES (8 MiB),
 * which every GPU that loads the library holds until the process exits.  The paper has no
 * counterpart to this entry point.
 *
 * Sizes: the call needs 256 bytes for the status word plus M*lda*elt (A), M*ldc*2 (C) and, for
 * FP8, ceil(K/128)*ld_sa*4 (scale_a) bytes, each rounded up to 256; a call that needs more than
 * BI_NOALLOC_SCRATCH_BYTES returns BI_ERR_UNSUPPORTED_SHAPE before touching the device.  (The
 * decode shape N = 4096, K = 7168 in bf16 fits up to M = 372 rows.)
 * Behaviour: copies A (and scale_a) in, runs the GEMM, copies C out, then synchronises `stream`
 * and returns the kernel's status (BI_OK or BI_ERR_DEVICE_TIMEOUT), so C_host is ready on
 * return.  B and scale_b are device pointers (resident weights).  The status word is cleared
 * before every launch.  All calls share the one array and it keeps the last call's contents:
 * calls that overlap on the GPU (from several host threads or streams) race on it and must be
 * serialised by the caller.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before any stream
 * capture begins, so that the look-up never happens inside a capture.  The status word is read
 * back on `stream` ahead of the one synchronisation, so the call touches no other stream.
 * Dense plans only (a grouped plan returns BI_ERR_INVALID_ARG).
 * Errors: as bi_gemm_run_host (scale_b must be 4-byte aligned; scale_a_host may have any
 * alignment, it is only copied), plus BI_ERR_UNSUPPORTED_SHAPE when the scratch is too small
 * or when M, lda, ldc or ld_sa alone exceeds BI_NOALLOC_SCRATCH_BYTES.
 */
#define BI_NOALLOC_SCRATCH_BYTES (8u << 20)
bi_status_t bi_gemm_run_host_noalloc(bi_plan_t plan, int64_t M,
                                     const void *A_host, int64_t lda,
                                     const void *B, int64_t ldb,
                                     void *C_host, int64_t ldc,
                                     const float *scale_a_host, int64_t ld_sa,
                                     const float *scale_b,
                                     cudaStream_t stream);

/*
 * Synchronise `stream`, then read and clear the plan's device status word for the current
 * device.  Returns BI_OK, BI_ERR_DEVICE_TIMEOUT, BI_ERR_BAD_OFFSETS or BI_ERR_CUDA.  All runs
 * of one plan on one device share the status word.
 */
bi_status_t bi_gemm_sync_status(bi_plan_t plan, cudaStream_t stream);

/*
 * Set the time limit, in nanoseconds, of every device-side pipeline wait of this plan's
 * kernels (default 2e9, i.e. 2 s; 0 restores the default).  The device counts the limit in SM
 * clock cycles at 2 cycles per ns, at or above the highest B200 SM clock, so a wait lasts at least
 * timeout_ns (longer when the clock runs lower).  A wait that runs out sets
 * BI_ERR_DEVICE_TIMEOUT, lets the CTA drain its own copies in flight, frees its tensor memory
 * and returns, so the context stays usable.
 */
bi_status_t bi_gemm_set_wait_timeout(bi_plan_t plan, uint64_t timeout_ns);

/*
 * Fixed-split-K research variant.  NOT the batch-invariant product path: the pages drop split-K
 * from the GEMM because a split count chosen by heuristics (per batch size, occupancy or memory
 * pressure) changes the reduction order ("DeepSeek V4 的隐藏关键特性被挖出来了" (wmrh.cn), section
 * 2.2).  This plan fixes the split instead: splits = 2, 4 or 8, chosen by the caller, and the tile
 * (128 x BN, BN the widest of 128 / 64 / 32 that gives at least 100 work units) follow from
 * (N, K, splits) alone.  Split s of a tile accumulates the K chunks (128 bytes each)
 * [s*nkb/splits, (s+1)*nkb/splits) (integer division) in ascending K into an fp32 workspace, and a
 * second kernel adds the splits in a fixed pairwise tree, ((p0 + p1) + (p2 + p3)) + ..., then
 * rounds once to bf16.  The split points and the merge order depend on (N, K, splits) only, so a
 * row's bits still do not depend on M, but they differ from the product plan's bits for the same
 * (N, K).  bf16 only.  bi_gemm_run refuses such a plan; bi_gemm_run_splitk refuses any other.
 * Errors: BI_ERR_INVALID_ARG (splits not 2, 4 or 8), BI_ERR_UNSUPPORTED_SHAPE (fewer K chunks
 * than splits).
 */
bi_status_t bi_gemm_plan_splitk(bi_plan_t *out, int64_t N, int64_t K, int splits);

/* Bytes of fp32 workspace bi_gemm_run_splitk needs for M rows: splits * M * roundup(N, 4) * 4
 * (0 for a plan that is not a split-K plan, or M <= 0). */
size_t bi_gemm_splitk_workspace_bytes(bi_plan_t plan, int64_t M);

/* C = A . B^T with a split-K plan.  Arguments as bi_gemm_run (bf16, no scales), plus a caller-
 * owned, 16-byte aligned device workspace of at least bi_gemm_splitk_workspace_bytes(plan, M)
 * bytes, which the call overwrites.  Two kernels on `stream`: the split GEMM and the merge. */
bi_status_t bi_gemm_run_splitk(bi_plan_t plan, int64_t M,
                               const void *A, int64_t lda,
                               const void *B, int64_t ldb,
                               void *C, int64_t ldc,
                               void *workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/*
 * Plan flags; 0 clears them all.
 * BI_PLAN_RESIDENT_WEIGHTS: the caller promises that no kernel enqueued on a launch's stream
 * before that launch writes the launch's B or scale_b (weights loaded once and then only read,
 * as in inference).  A dense launch may then request its first pipeline groups of B while the
 * previous kernel in the stream is still running; it still waits for that kernel to complete
 * before it reads A or scale_a or writes C or the status word.  The flag changes when B is
 * read, never a result.  Off by default; grouped plans ignore it.
 * BI_PLAN_HOST_ROW_BLOCKS: the caller promises that, within one bi_gemm_run_host_batch, host
 * buffers of consecutive calls that touch end to start (A_host after A_host, C_host after
 * C_host) belong to one host allocation.  The batch then moves each such run of calls with one
 * copy (a copy may not span two allocations).  Off by default: one copy per call.
 * Errors: BI_ERR_INVALID_ARG (plan == NULL or an unknown flag bit).
 */
#define BI_PLAN_RESIDENT_WEIGHTS 1u
#define BI_PLAN_HOST_ROW_BLOCKS 2u
bi_status_t bi_gemm_plan_set_flags(bi_plan_t plan, uint32_t flags);

/*
 * Test-only fault injection on the host side of the launch.  BI_DEBUG_SKIP_FIRST_LOAD makes
 * the producer of every CTA skip its very first operand load, so that the first MMA wait of
 * the CTA can never complete and must end by its time limit.  0 clears all flags.  Never set in
 * production.
 */
#define BI_DEBUG_SKIP_FIRST_LOAD 1u
bi_status_t bi_gemm_debug_set_flags(bi_plan_t plan, uint32_t flags);

#ifdef __cplusplus
}
#endif

#endif /* BI_GEMM_H */
