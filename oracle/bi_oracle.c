/*
 * bi_oracle.c -- plain, slow, obviously correct CPU oracle for the batch-invariant GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file:
 * only the tests, the package's smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (plain definitions, fp64, one rounding at the end):
 *
 *   Dense GEMM, alpha = 1, beta = 0:   C[m][n] = sum_k A[m][k] * B[n][k]
 *     -- the K-axis accumulation C[i][j] = sum_K A[i][k] x B[k][j] of
 *        "DeepSeek V4的batch invariance：大模型确定性推理的工程基石" (lshu.cn), section 2.1,
 *        with B stored as [N][K] (the B^T form), and the alpha = 1, beta = 0 restriction of the
 *        wmrh.cn article "DeepSeek V4 的隐藏关键特性被挖出来了", section 3.1.
 *   FP8 block-scaled GEMM: the e4m3 codes are dequantised exactly (code value times the fp32
 *     scale of its block: A per 1x128 K-block, B per 128x128 block), then the dense GEMM above.
 *     The pages only say that the dequantisation is fused into the GEMM (lshu.cn article,
 *     section 3.2); the block shapes are those of the FP8 workload this library targets.
 *   e2m1 weights x e4m3 activations (W4A8): the weights are dequantised as
 *     W[n][k] = e2m1(Q[n][k]) * scale[n] + zero[n], the quantisation of the lshu.cn article,
 *     section 4.3 (one scale 2^-j, j in [1, 12], and one fp16-exact zero point per output
 *     channel), the activations as in the FP8 GEMM (per 1x128 K-block scales); then the dense
 *     GEMM above.  Every dequantised weight is exact in fp64 (a 2-bit significand times a power
 *     of two plus an 11-bit one, spanning at most 2^15 .. 2^-24).
 *   e2m1 weight quantisation, the same section's W_fp4 = round((W - zero) / scale): x is formed
 *     in fp64 from the 16-bit weight (bf16 or fp16), the zero point and the scale, and rounded to
 *     the nearest e2m1 value, ties to the even fraction bit (the IEEE default the pages fix for
 *     their GEMM, wmrh.cn article section 3.1); values beyond +-6 saturate to +-6, NaN gives +0.
 *   Grouped (MoE) GEMM: for expert e and every row r in [offsets[e], offsets[e+1]),
 *     C[r][n] = sum_k A[r][k] * B_e[n][k].  MoE is listed among the V4 components in
 *     "DeepSeek不惜代价保住它！V4关键特性被挖出来了" (QbitAI), section "什么是batch invariance".
 *
 * Every sum runs k = 0, 1, ..., K-1 in fp64 with a plain scalar loop.  Products of two bf16
 * values are exact in fp64; products of two dequantised e4m3 values carry at most 8 + 48
 * significant bits, so fp64 rounds them by at most 2^-53 relative.  The result is rounded once,
 * round-to-nearest-even, from fp64 straight to bf16 (no intermediate fp32 step).
 *
 * Codecs are written from the format definitions:
 *   bf16  = 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits (upper half of binary32).
 *   e4m3  = 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits; exponent field 0 is
 *           subnormal (value = fraction * 2^-9); S.1111.111 is NaN; no infinities; max 448.
 *   fp16  = 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; exponent field 0 is
 *           subnormal (value = fraction * 2^-24); exponent field 31 is infinity or NaN.
 *   e2m1  = 1 sign bit, 2 exponent bits (bias 1), 1 fraction bit; exponent field 0 is
 *           subnormal (value = fraction * 2^-1); no infinities or NaN; max 6.  Packed two per
 *           byte, value k of a row in byte k/2, the even k in the low four bits.
 *
 * Threads: output rows are split across POSIX threads; every output element is still one
 * sequential fp64 loop, so the oracle is itself deterministic and batch-invariant.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC -pthread bi_oracle.c -lm
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ----------------------------------------------------------------------------------------- */
/* Codecs                                                                                      */
/* ----------------------------------------------------------------------------------------- */

/* bf16 bit pattern -> exact fp64 value, from the sign/exponent/fraction fields. */
double oracle_bf16_to_f64(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 7) & 0xFF;
    int frac = bits & 0x7F;
    double v;
    if (expo == 0xFF) {
        v = frac ? NAN : INFINITY;
    } else if (expo == 0) {
        v = ldexp((double)frac, -126 - 7);            /* subnormal: 0.frac * 2^-126 */
    } else {
        v = ldexp((double)(128 + frac), expo - 127 - 7); /* 1.frac * 2^(e-127) */
    }
    return sign ? -v : v;
}

/* e4m3 ("fn" variant: no infinities) bit pattern -> exact fp64 value. */
double oracle_e4m3_to_f64(uint8_t bits)
{
    int sign = (bits >> 7) & 1;
    int expo = (bits >> 3) & 0xF;
    int frac = bits & 0x7;
    double v;
    if (expo == 0xF && frac == 0x7) {
        v = NAN;
    } else if (expo == 0) {
        v = ldexp((double)frac, -9);                   /* 0.frac * 2^-6 = frac * 2^-9 */
    } else {
        v = ldexp((double)(8 + frac), expo - 7 - 3);   /* 1.frac * 2^(e-7) */
    }
    return sign ? -v : v;
}

/* e2m1 4-bit code (the low four bits of `code`) -> exact fp64 value. */
double oracle_e2m1_to_f64(uint8_t code)
{
    int sign = (code >> 3) & 1;
    int expo = (code >> 1) & 0x3;
    int frac = code & 0x1;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -1);                   /* 0.frac * 2^0 = frac * 2^-1 */
    else
        v = ldexp((double)(2 + frac), expo - 1 - 1);   /* 1.frac * 2^(e-1) */
    return sign ? -v : v;
}

/* fp16 bit pattern -> exact fp64 value. */
double oracle_fp16_to_f64(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 10) & 0x1F;
    int frac = bits & 0x3FF;
    double v;
    if (expo == 0x1F)
        v = frac ? NAN : INFINITY;
    else if (expo == 0)
        v = ldexp((double)frac, -24);                  /* 0.frac * 2^-14 */
    else
        v = ldexp((double)(1024 + frac), expo - 15 - 10);   /* 1.frac * 2^(e-15) */
    return sign ? -v : v;
}

/* fp64 -> e2m1 4-bit code: round to nearest, ties to the even fraction bit, saturating at +-6;
 * NaN gives +0.  The e2m1 values in [0, 2) are 0.5 apart, in [2, 4) 1 apart and in [4, 8) 2
 * apart (6 being the largest); the sign bit follows the sign of x, so a negative x that rounds to
 * zero gives -0. */
uint8_t oracle_f64_to_e2m1(double x)
{
    if (isnan(x))
        return 0;
    uint8_t sign = signbit(x) ? 8 : 0;
    double a = fabs(x);
    double q = a < 2.0 ? 0.5 : (a < 4.0 ? 1.0 : 2.0);   /* spacing in a's binade */
    double v = nearbyint(a / q) * q;                      /* ties to an even multiple of q */
    if (v > 6.0)
        v = 6.0;
    static const double values[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    uint8_t code = 0;
    for (uint8_t c = 0; c < 8; ++c)
        if (values[c] == v)
            code = c;
    return (uint8_t)(sign | code);
}

/* fp64 -> bf16 bit pattern, round to nearest, ties to even; overflow goes to +-inf,
 * results below the smallest normal become bf16 subnormals.  NaN maps to the quiet NaN 0x7FC0
 * with the input's sign. */
uint16_t oracle_f64_to_bf16_rne(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x))
        return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(x);
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0)
        return sign;

    int e2;                     /* a = f * 2^e2 with f in [0.5, 1) */
    (void)frexp(a, &e2);
    int e = e2 - 1;             /* a in [2^e, 2^(e+1)) */
    if (e < -126)
        e = -126;               /* subnormal range shares the quantum of the smallest binade */
    /* bf16 keeps 8 significant bits: the quantum in the binade [2^e, 2^(e+1)) is 2^(e-7). */
    double q = ldexp(1.0, e - 7);
    double n = a / q;           /* exact: division by a power of two */
    double r = nearbyint(n);    /* default rounding mode: to nearest, ties to even */

    uint32_t field;
    if (a < ldexp(1.0, -126)) {
        /* subnormal input: the integer r (0..128) is exactly the 8-bit pattern; r = 128 is the
         * smallest normal 0x0080. */
        field = (uint32_t)r;
    } else {
        /* normal: r in [128, 256]; r = 256 carries into the exponent field. */
        field = ((uint32_t)(e + 127) << 7) + ((uint32_t)r - 128u);
        if (field >= 0x7F80u)
            field = 0x7F80u;    /* overflow to infinity */
    }
    return (uint16_t)(sign | field);
}

/* Array forms of the codecs: the scalar codecs above applied to each element in turn (no other
 * arithmetic), so that whole tensors convert without one foreign call per element. */
void oracle_bf16_to_f64_array(const uint16_t *bits, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_to_f64(bits[i]);
}

void oracle_e4m3_to_f64_array(const uint8_t *bits, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_to_f64(bits[i]);
}

void oracle_f64_to_bf16_rne_array(const double *x, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f64_to_bf16_rne(x[i]);
}

/* ----------------------------------------------------------------------------------------- */
/* Row-parallel driver                                                                         */
/* ----------------------------------------------------------------------------------------- */

typedef struct {
    const double *a;        /* [rows][K] fp64 */
    const double *b;        /* [N][K]    fp64 (for grouped: [E][N][K]) */
    const int64_t *row_b;   /* per row: offset of its B matrix in b (elements), or NULL */
    int64_t rows, n_cols, k;
    double *cref;           /* [rows][N] fp64, may be NULL */
    uint16_t *cbits;        /* [rows][N] bf16 bits, may be NULL */
    int64_t row_begin, row_end;
} oracle_job_t;

static void *oracle_rows(void *arg)
{
    const oracle_job_t *j = (const oracle_job_t *)arg;
    for (int64_t m = j->row_begin; m < j->row_end; ++m) {
        const double *arow = j->a + m * j->k;
        const double *bmat = j->b + (j->row_b ? j->row_b[m] : 0);
        for (int64_t n = 0; n < j->n_cols; ++n) {
            const double *brow = bmat + n * j->k;
            double s = 0.0;
            for (int64_t kk = 0; kk < j->k; ++kk)
                s += arow[kk] * brow[kk];
            if (j->cref)
                j->cref[m * j->n_cols + n] = s;
            if (j->cbits)
                j->cbits[m * j->n_cols + n] = oracle_f64_to_bf16_rne(s);
        }
    }
    return NULL;
}

static int run_rows(const double *a, const double *b, const int64_t *row_b, int64_t rows,
                    int64_t n_cols, int64_t k, double *cref, uint16_t *cbits, int threads)
{
    if (threads < 1)
        threads = 1;
    if (threads > 1024)
        threads = 1024;
    if ((int64_t)threads > rows)
        threads = rows > 0 ? (int)rows : 1;
    oracle_job_t *jobs = (oracle_job_t *)calloc((size_t)threads, sizeof(oracle_job_t));
    pthread_t *tids = (pthread_t *)calloc((size_t)threads, sizeof(pthread_t));
    if (!jobs || !tids) {
        free(jobs);
        free(tids);
        return -1;
    }
    for (int t = 0; t < threads; ++t) {
        oracle_job_t *j = &jobs[t];
        j->a = a; j->b = b; j->row_b = row_b;
        j->rows = rows; j->n_cols = n_cols; j->k = k;
        j->cref = cref; j->cbits = cbits;
        j->row_begin = rows * t / threads;
        j->row_end = rows * (t + 1) / threads;
    }
    int started = 0;
    for (int t = 1; t < threads; ++t) {
        if (pthread_create(&tids[t], NULL, oracle_rows, &jobs[t]) != 0)
            break;
        started = t;
    }
    oracle_rows(&jobs[0]);
    for (int t = 1; t <= started; ++t)
        pthread_join(tids[t], NULL);
    /* rows of threads that could not be started run here, serially */
    for (int t = started + 1; t < threads; ++t)
        oracle_rows(&jobs[t]);
    free(jobs);
    free(tids);
    return 0;
}

/* ----------------------------------------------------------------------------------------- */
/* Public oracle entry points (all host memory, row-major, caller-owned)                       */
/* ----------------------------------------------------------------------------------------- */

/* Dense bf16:  A [M][K] bf16 bits, B [N][K] bf16 bits  ->  cref [M][N] fp64 (unrounded sum)
 * and cbits [M][N] bf16 bits (cref rounded once, RNE).  Either output may be NULL.
 * Returns 0, or -1 on allocation failure. */
int oracle_gemm_bf16(int64_t M, int64_t N, int64_t K, const uint16_t *A, const uint16_t *B,
                     double *cref, uint16_t *cbits, int threads)
{
    double *a = (double *)malloc(sizeof(double) * (size_t)(M * K > 0 ? M * K : 1));
    double *b = (double *)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
    if (!a || !b) {
        free(a);
        free(b);
        return -1;
    }
    for (int64_t i = 0; i < M * K; ++i)
        a[i] = oracle_bf16_to_f64(A[i]);
    for (int64_t i = 0; i < N * K; ++i)
        b[i] = oracle_bf16_to_f64(B[i]);
    int rc = run_rows(a, b, NULL, M, N, K, cref, cbits, threads);
    free(a);
    free(b);
    return rc;
}

/* FP8 e4m3 with fp32 block scales, dequantised exactly and then multiplied:
 *   a_deq[m][k] = e4m3(QA[m][k]) * SA[m][k/128]          SA is [M][ceil(K/128)] row-major
 *   b_deq[n][k] = e4m3(QB[n][k]) * SB[n/128][k/128]      SB is [ceil(N/128)][ceil(K/128)]
 *   cref[m][n]  = sum_k a_deq[m][k] * b_deq[n][k]
 * Each dequantised value (4 + 24 significant bits) is exact in fp64. */
int oracle_gemm_fp8_blockscaled(int64_t M, int64_t N, int64_t K, const uint8_t *QA,
                                const uint8_t *QB, const float *SA, const float *SB,
                                double *cref, uint16_t *cbits, int threads)
{
    int64_t kb = (K + 127) / 128;
    double *a = (double *)malloc(sizeof(double) * (size_t)(M * K > 0 ? M * K : 1));
    double *b = (double *)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
    if (!a || !b) {
        free(a);
        free(b);
        return -1;
    }
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k)
            a[m * K + k] = oracle_e4m3_to_f64(QA[m * K + k]) * (double)SA[m * kb + k / 128];
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            b[n * K + k] = oracle_e4m3_to_f64(QB[n * K + k]) * (double)SB[(n / 128) * kb + k / 128];
    int rc = run_rows(a, b, NULL, M, N, K, cref, cbits, threads);
    free(a);
    free(b);
    return rc;
}

/* e2m1 weights x e4m3 activations:
 *   a_deq[m][k] = e4m3(QA[m][k]) * SA[m][k/128]           SA is [M][ceil(K/128)] row-major
 *   w_deq[n][k] = e2m1(QW[n][k]) * WS[n] + WZ[n]          QW packed [N][K/2] bytes; WZ may be NULL
 *   cref[m][n]  = sum_k a_deq[m][k] * w_deq[n][k]
 * K must be even.  Returns 0, or -1 on allocation failure. */
int oracle_gemm_w4a8(int64_t M, int64_t N, int64_t K, const uint8_t *QA, const float *SA,
                     const uint8_t *QW, const float *WS, const float *WZ, double *cref,
                     uint16_t *cbits, int threads)
{
    int64_t kb = (K + 127) / 128;
    double *a = (double *)malloc(sizeof(double) * (size_t)(M * K > 0 ? M * K : 1));
    double *b = (double *)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
    if (!a || !b) {
        free(a);
        free(b);
        return -1;
    }
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k)
            a[m * K + k] = oracle_e4m3_to_f64(QA[m * K + k]) * (double)SA[m * kb + k / 128];
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = QW[n * (K / 2) + k / 2];
            uint8_t code = (k % 2 == 0) ? (uint8_t)(byte & 0xF) : (uint8_t)(byte >> 4);
            double w = oracle_e2m1_to_f64(code) * (double)WS[n];
            if (WZ)
                w += (double)WZ[n];
            b[n * K + k] = w;
        }
    int rc = run_rows(a, b, NULL, M, N, K, cref, cbits, threads);
    free(a);
    free(b);
    return rc;
}

/* e2m1 quantisation of 16-bit weights W [N][K] (bf16 bits, or fp16 bits when is_fp16):
 *   q[n][k] = e2m1_rne((W[n][k] - WZ[n]) / WS[n])   (WZ may be NULL: zero points 0)
 * written packed, Q [N][K/2] bytes, value k in byte k/2, the even k in the low four bits.  K must
 * be even. */
void oracle_quantize_e2m1(int64_t N, int64_t K, const uint16_t *W, int is_fp16, const float *WS,
                          const float *WZ, uint8_t *Q)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; k += 2) {
            uint8_t code[2];
            for (int h = 0; h < 2; ++h) {
                uint16_t bits = W[n * K + k + h];
                double w = is_fp16 ? oracle_fp16_to_f64(bits) : oracle_bf16_to_f64(bits);
                double z = WZ ? (double)WZ[n] : 0.0;
                code[h] = oracle_f64_to_e2m1((w - z) / (double)WS[n]);
            }
            Q[n * (K / 2) + k / 2] = (uint8_t)(code[0] | (code[1] << 4));
        }
}

/* Grouped bf16 (MoE):  A [R][K] rows grouped by expert, B [E][N][K], offsets [E+1] with
 * offsets[0] = 0, non-decreasing, offsets[E] = R.  Row r in [offsets[e], offsets[e+1]) is
 * multiplied with B_e.  Returns -2 if the offsets break those rules. */
int oracle_grouped_gemm_bf16(int64_t R, int64_t N, int64_t K, int64_t E, const uint16_t *A,
                             const uint16_t *B, const int32_t *offsets, double *cref,
                             uint16_t *cbits, int threads)
{
    if (E < 1 || offsets[0] != 0 || offsets[E] != R)
        return -2;
    for (int64_t e = 0; e < E; ++e)
        if (offsets[e + 1] < offsets[e])
            return -2;
    double *a = (double *)malloc(sizeof(double) * (size_t)(R * K > 0 ? R * K : 1));
    double *b = (double *)malloc(sizeof(double) * (size_t)(E * N * K > 0 ? E * N * K : 1));
    int64_t *row_b = (int64_t *)malloc(sizeof(int64_t) * (size_t)(R > 0 ? R : 1));
    if (!a || !b || !row_b) {
        free(a);
        free(b);
        free(row_b);
        return -1;
    }
    for (int64_t i = 0; i < R * K; ++i)
        a[i] = oracle_bf16_to_f64(A[i]);
    for (int64_t i = 0; i < E * N * K; ++i)
        b[i] = oracle_bf16_to_f64(B[i]);
    for (int64_t e = 0; e < E; ++e)
        for (int64_t r = offsets[e]; r < offsets[e + 1]; ++r)
            row_b[r] = e * N * K;
    int rc = run_rows(a, b, row_b, R, N, K, cref, cbits, threads);
    free(a);
    free(b);
    free(row_b);
    return rc;
}
