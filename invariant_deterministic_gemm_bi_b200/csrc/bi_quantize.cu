// bi_quantize.cu -- e2m1 (FP4) quantisation of 16-bit weights with a per-channel scale and zero
// point (include/bi_quantize.h).  Elementwise and HBM-bound: one thread per output byte (two
// values), grid-stride over the weights.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bi_quantize.h"

namespace {

// The e2m1 code of x: the nearest of 0, 0.5, 1, 1.5, 2, 3, 4, 6 to |x| (ties to the value with
// fraction bit 0), saturating at 6, with x's sign in bit 3; NaN gives 0.  The magnitude code is
// the number of decision points |x| lies above: the midpoints between neighbouring values, each
// inclusive when the value above it has fraction bit 0 (0.75, 1.75, 3.5) and exclusive otherwise.
__device__ __forceinline__ uint32_t e2m1_code(double x)
{
    if (x != x)
        return 0u;
    const uint32_t sign = (__double_as_longlong(x) < 0) ? 8u : 0u;
    const double a = fabs(x);
    const uint32_t c = (a > 0.25 ? 1u : 0u) + (a >= 0.75 ? 1u : 0u) + (a > 1.25 ? 1u : 0u) +
                       (a >= 1.75 ? 1u : 0u) + (a > 2.5 ? 1u : 0u) + (a >= 3.5 ? 1u : 0u) +
                       (a > 5.0 ? 1u : 0u);
    return sign | c;
}

template <bool FP16>
__device__ __forceinline__ double weight_value(uint16_t bits)
{
    if constexpr (FP16)
        return static_cast<double>(__half2float(__ushort_as_half(bits)));
    else
        return static_cast<double>(__uint_as_float(static_cast<uint32_t>(bits) << 16));
}

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
        const double s = static_cast<double>(scale[r]);
        const double z = zero ? static_cast<double>(zero[r]) : 0.0;
        const uint16_t *wr = w + r * ldw + 2 * c;
        const uint32_t lo = e2m1_code((weight_value<FP16>(wr[0]) - z) / s);
        const uint32_t hi = e2m1_code((weight_value<FP16>(wr[1]) - z) / s);
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
    const int64_t total = N * (K / 2);
    const int64_t blocks = (total + 255) / 256;
    const int grid = static_cast<int>(blocks < sms * 32 ? blocks : sms * 32);
    const uint16_t *w = static_cast<const uint16_t *>(W);
    uint8_t *q = static_cast<uint8_t *>(Q);
    if (w_is_fp16)
        quantize_e2m1_kernel<true><<<grid, 256, 0, stream>>>(w, ldw, N, K, w_scale, w_zero, q, ldq / 2);
    else
        quantize_e2m1_kernel<false><<<grid, 256, 0, stream>>>(w, ldw, N, K, w_scale, w_zero, q, ldq / 2);
    return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

} // extern "C"
