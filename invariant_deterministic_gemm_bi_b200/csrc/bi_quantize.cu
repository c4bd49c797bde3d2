// bi_quantize.cu -- e2m1 (FP4) quantisation of 16-bit weights with a per-channel scale and zero
// point (include/bi_quantize.h).  Elementwise and HBM-bound.  Rows whose weights start on 16 bytes
// and whose codes start on 4 bytes take the vector kernel: one CTA per row at a time, each thread
// turning 8 weights (one 16-byte load) into 4 code bytes (one 4-byte store), four such loads in
// flight.  Other layouts take a scalar kernel with one thread per code byte.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bi_quantize.h"

namespace {

// The e2m1 code of x: the nearest of 0, 0.5, 1, 1.5, 2, 3, 4, 6 to |x| (ties to the value with
// fraction bit 0), saturating at 6, with x's sign in bit 3; NaN gives 0.  The magnitude code is
// the number of decision points |x| lies above -- the midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5
// and 5 between neighbouring values -- each inclusive when the value above it has fraction bit 0
// (0.75, 1.75, 3.5) and exclusive otherwise.
//
// The comparisons run on one 32-bit key: key = 2 * (high word of |x|) + (low word != 0).  For
// non-negative doubles the bit patterns are ordered like the values, and every decision point t
// has a zero low word, so |x| >= t  <=>  key >= 2 * hi(t)  and  |x| > t  <=>  key > 2 * hi(t).
// NaN is the only case with key > 2 * hi(inf).
__device__ __forceinline__ uint32_t e2m1_code(double x)
{
    const uint32_t hi = static_cast<uint32_t>(__double2hiint(x));
    const uint32_t lo = static_cast<uint32_t>(__double2loint(x));
    const uint32_t key = ((hi & 0x7FFFFFFFu) << 1) | (lo != 0u ? 1u : 0u);
    if (key > 0xFFE00000u)                        // 2 * hi(inf): NaN
        return 0u;
    const uint32_t c = (key > 0x7FA00000u ? 1u : 0u) +    // |x| >  0.25
                       (key >= 0x7FD00000u ? 1u : 0u) +   // |x| >= 0.75
                       (key > 0x7FE80000u ? 1u : 0u) +    // |x| >  1.25
                       (key >= 0x7FF80000u ? 1u : 0u) +   // |x| >= 1.75
                       (key > 0x80080000u ? 1u : 0u) +    // |x| >  2.5
                       (key >= 0x80180000u ? 1u : 0u) +   // |x| >= 3.5
                       (key > 0x80280000u ? 1u : 0u);     // |x| >  5
    return (hi >> 31) * 8u + c;
}

template <bool FP16>
__device__ __forceinline__ double weight_value(uint32_t bits16)
{
    if constexpr (FP16)
        return static_cast<double>(__half2float(__ushort_as_half(static_cast<uint16_t>(bits16))));
    else
        return static_cast<double>(__uint_as_float(bits16 << 16));
}

// One channel's constants.  x = (w - zero) / scale in fp64.  When the scale (as a double) has no
// mantissa bits -- a power of two, +-0 or +-inf -- its reciprocal is exact and d * (1 / scale)
// equals d / scale bit for bit (no product here can overflow or underflow fp64: |d| < 2^130 and
// the scale lies in the fp32 range), so the multiply replaces the division.
struct Channel {
    double zero, scale, recip;
    bool pow2;
};

__device__ __forceinline__ Channel channel(const float *scale, const float *zero, int64_t r)
{
    Channel ch;
    ch.scale = static_cast<double>(scale[r]);
    ch.zero = zero ? static_cast<double>(zero[r]) : 0.0;
    ch.pow2 = (static_cast<uint64_t>(__double_as_longlong(ch.scale)) & 0x000FFFFFFFFFFFFFull) == 0;
    ch.recip = 1.0 / ch.scale;
    return ch;
}

template <bool FP16, bool POW2>
__device__ __forceinline__ uint32_t code_of(uint32_t bits16, const Channel &ch)
{
    const double d = weight_value<FP16>(bits16) - ch.zero;
    return e2m1_code(POW2 ? d * ch.recip : d / ch.scale);
}

// One row's whole 8-value groups: thread t converts groups t, t + blockDim, ..., four loads in
// flight.  The scale's kind is a template parameter so that the loop of a power-of-two row holds
// no division code.
template <bool FP16, bool POW2>
__device__ __forceinline__ void quantize_row_groups(const uint4 *wr, uint32_t *qr, int64_t vecs,
                                                    const Channel &ch)
{
    constexpr int kUnroll = 4;
    for (int64_t v0 = threadIdx.x; v0 < vecs; v0 += kUnroll * blockDim.x) {
        uint4 x[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t v = v0 + u * static_cast<int64_t>(blockDim.x);
            x[u] = v < vecs ? __ldg(wr + v) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t v = v0 + u * static_cast<int64_t>(blockDim.x);
            if (v < vecs) {
                const uint32_t in[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
                uint32_t out = 0u;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // weights 2j (low half) and 2j + 1 (high half) -> byte j
                    const uint32_t lo = code_of<FP16, POW2>(in[j] & 0xFFFFu, ch);
                    const uint32_t hi = code_of<FP16, POW2>(in[j] >> 16, ch);
                    out |= (lo | (hi << 4)) << (8 * j);
                }
                qr[v] = out;
            }
        }
    }
}

// Rows with 16-byte-aligned weights and 4-byte-aligned codes: CTA b handles rows b, b + grid, ...
template <bool FP16>
__global__ void __launch_bounds__(256) quantize_e2m1_vec_kernel(const uint16_t *w, int64_t ldw,
                                                                int64_t n_rows, int64_t k,
                                                                const float *scale, const float *zero,
                                                                uint8_t *q, int64_t ldq_bytes)
{
    const int64_t vecs = k / 8;   // whole 8-value groups of a row
    for (int64_t r = blockIdx.x; r < n_rows; r += gridDim.x) {
        const Channel ch = channel(scale, zero, r);
        const uint4 *wr = reinterpret_cast<const uint4 *>(w + r * ldw);
        uint32_t *qr = reinterpret_cast<uint32_t *>(q + r * ldq_bytes);
        if (ch.pow2)
            quantize_row_groups<FP16, true>(wr, qr, vecs, ch);
        else
            quantize_row_groups<FP16, false>(wr, qr, vecs, ch);
        // the pairs past the last whole group (K % 8 != 0)
        const int64_t pairs = k / 2;
        for (int64_t c = vecs * 4 + threadIdx.x; c < pairs; c += blockDim.x) {
            const uint16_t *wp = w + r * ldw + 2 * c;
            const uint32_t lo = ch.pow2 ? code_of<FP16, true>(wp[0], ch) : code_of<FP16, false>(wp[0], ch);
            const uint32_t hi = ch.pow2 ? code_of<FP16, true>(wp[1], ch) : code_of<FP16, false>(wp[1], ch);
            q[r * ldq_bytes + c] = static_cast<uint8_t>(lo | (hi << 4));
        }
    }
}

// Any layout: one thread per code byte (two weights), grid-stride.
template <bool FP16>
__global__ void quantize_e2m1_kernel(const uint16_t *w, int64_t ldw, int64_t n_rows, int64_t k,
                                     const float *scale, const float *zero, uint8_t *q,
                                     int64_t ldq_bytes)
{
    const int64_t pairs = k / 2;
    const int64_t total = n_rows * pairs;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / pairs;
        const int64_t c = i - r * pairs;
        const Channel ch = channel(scale, zero, r);
        const uint16_t *wr = w + r * ldw + 2 * c;
        const uint32_t lo = ch.pow2 ? code_of<FP16, true>(wr[0], ch) : code_of<FP16, false>(wr[0], ch);
        const uint32_t hi = ch.pow2 ? code_of<FP16, true>(wr[1], ch) : code_of<FP16, false>(wr[1], ch);
        q[r * ldq_bytes + c] = static_cast<uint8_t>(lo | (hi << 4));
    }
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

} // namespace

extern "C" {

bi_status_t bi_quantize_e2m1(const void *W, int w_is_fp16, int64_t ldw, int64_t N, int64_t K,
                             const float *w_scale, const float *w_zero, void *Q, int64_t ldq,
                             cudaStream_t stream)
{
    if (N < 0 || K < 0 || (w_is_fp16 != 0 && w_is_fp16 != 1))
        return BI_ERR_INVALID_ARG;
    if (K % 2 != 0)
        return BI_ERR_INVALID_ARG;
    if (N == 0 || K == 0)
        return BI_OK;
    if (!W || !Q || !w_scale || ldw < K || ldq < K || ldq % 2 != 0)
        return BI_ERR_INVALID_ARG;
    if (!aligned(W, 2) || !aligned(w_scale, 4) || (w_zero && !aligned(w_zero, 4)))
        return BI_ERR_ALIGNMENT;
    int count = 0, dev = 0, major = 0, sms = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess || count <= 0) {
        cudaGetLastError();
        return BI_ERR_NO_DEVICE;
    }
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return BI_ERR_CUDA;
    if (major != 10)
        return BI_ERR_NO_DEVICE;
    const uint16_t *w = static_cast<const uint16_t *>(W);
    uint8_t *q = static_cast<uint8_t *>(Q);
    const int64_t ldq_bytes = ldq / 2;
    // every row's weights on 16 bytes and codes on 4 bytes
    const bool vec = aligned(W, 16) && ldw % 8 == 0 && aligned(Q, 4) && ldq_bytes % 4 == 0;
    if (vec) {
        const int grid = static_cast<int>(N < sms * 4 ? N : sms * 4);
        if (w_is_fp16)
            quantize_e2m1_vec_kernel<true><<<grid, 256, 0, stream>>>(w, ldw, N, K, w_scale, w_zero, q, ldq_bytes);
        else
            quantize_e2m1_vec_kernel<false><<<grid, 256, 0, stream>>>(w, ldw, N, K, w_scale, w_zero, q, ldq_bytes);
    } else {
        const int64_t total = N * (K / 2);
        const int64_t blocks = (total + 255) / 256;
        const int grid = static_cast<int>(blocks < sms * 32 ? blocks : sms * 32);
        if (w_is_fp16)
            quantize_e2m1_kernel<true><<<grid, 256, 0, stream>>>(w, ldw, N, K, w_scale, w_zero, q, ldq_bytes);
        else
            quantize_e2m1_kernel<false><<<grid, 256, 0, stream>>>(w, ldw, N, K, w_scale, w_zero, q, ldq_bytes);
    }
    return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

} // extern "C"
