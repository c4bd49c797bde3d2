// bi_moe.cu -- the MoE steps either side of the grouped GEMM: top-k routing with softmax
// weights, the stable dispatch into expert segments, the row gather and the weighted combine
// (include/bi_moe.h).  All of them are HBM- or latency-bound elementwise work on CUDA cores; none
// uses atomics, and every floating-point reduction has a fixed order, so every token's results
// depend on that token alone.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <type_traits>

#include "bi_moe.h"

namespace {

constexpr int kMaxE = 1024;
constexpr int kMaxK = 8;
constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------------------------
// Router: one warp per token.  Lane l holds the logits of experts l, l + 32, l + 64, ...
// ---------------------------------------------------------------------------------------------

// PL = logit slots per lane (ceil(E / 32) rounded up to a power of two)
template <int PL>
__global__ void __launch_bounds__(256) moe_route_kernel(const float *logits, int64_t ld, int64_t T,
                                                        int E, int k, int32_t *experts,
                                                        float *weights)
{
    const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T)
        return;   // warp-uniform
    const float *row = logits + t * ld;
    float v[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) {
        const int e = i * 32 + lane;
        v[i] = e < E ? row[e] : -INFINITY;
    }
    // max over all experts (exact whatever the order)
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < PL; ++i)
        m = fmaxf(m, v[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
    // sum of exp(l - max): each lane in ascending expert index, then a fixed butterfly (every
    // lane adds the same pairs, so all lanes end with the same bits)
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < PL; ++i)
        if (i * 32 + lane < E)
            s = s + expf(v[i] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        s = s + __shfl_xor_sync(kFull, s, off);
    // top k: k rounds of a warp arg-max over (logit descending, expert index ascending)
    uint32_t used = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const int e = i * 32 + lane;
            if (e < E && !((used >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
                bv = v[i];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, off);
            const int oe = __shfl_xor_sync(kFull, be, off);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane)
            used |= 1u << (be >> 5);
        if (lane == 0) {
            experts[t * k + j] = be;
            weights[t * k + j] = expf(bv - m) / s;
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Dispatch: counts per expert, their exclusive scan, then each expert's rows in pair order.
// One block per expert, of 8 or 32 warps; warp w owns the contiguous pairs [w * seg, (w + 1) * seg) (seg a
// multiple of 128) and walks them 128 at a time, lane l holding pairs 4l .. 4l+3 of each step (one
// coalesced 16-byte load per lane when the id array is 16-byte aligned).  Ranks follow pair order:
// warps in order, steps in order, lanes in order, a lane's four pairs in order.
// ---------------------------------------------------------------------------------------------

constexpr int kDispatchSteps = 8;   // 128-pair steps loaded per batch
// Warps per expert block: 8 for up to kFewPairs pairs, else 32 (enough loads in flight per SM).
constexpr int kFewPairs = 16384;

template <int WARPS>
__device__ __forceinline__ int64_t dispatch_segment(int64_t n)
{
    const int64_t per = (n + WARPS - 1) / WARPS;
    return (per + 127) & ~static_cast<int64_t>(127);
}

// The four ids of pairs i .. i+3 (-1 past n, which matches no expert).  VEC: experts is 16-byte
// aligned and i is a multiple of 4.
template <bool VEC>
__device__ __forceinline__ int4 load_ids(const int32_t *__restrict__ experts, int64_t i, int64_t n)
{
    if (VEC && i + 4 <= n)
        return __ldg(reinterpret_cast<const int4 *>(experts + i));
    int4 v;
    v.x = i < n ? __ldg(experts + i) : -1;
    v.y = i + 1 < n ? __ldg(experts + i + 1) : -1;
    v.z = i + 2 < n ? __ldg(experts + i + 2) : -1;
    v.w = i + 3 < n ? __ldg(experts + i + 3) : -1;
    return v;
}

__device__ __forceinline__ uint32_t hit_mask(const int4 &v, int e)
{
    return (v.x == e ? 1u : 0u) | (v.y == e ? 2u : 0u) | (v.z == e ? 4u : 0u) | (v.w == e ? 8u : 0u);
}

// Hits of expert e in this warp's segment (every lane gets the total).
template <bool VEC>
__device__ __forceinline__ int warp_count(const int32_t *__restrict__ experts, int64_t lo, int64_t hi,
                                          int64_t n, int e)
{
    const int lane = threadIdx.x & 31;
    int c = 0;
    for (int64_t base = lo; base < hi; base += kDispatchSteps * 128) {
        int4 v[kDispatchSteps];
#pragma unroll
        for (int u = 0; u < kDispatchSteps; ++u) {
            const int64_t i = base + 128 * u + 4 * lane;
            v[u] = (base + 128 * u < hi) ? load_ids<VEC>(experts, i, n) : make_int4(-1, -1, -1, -1);
        }
#pragma unroll
        for (int u = 0; u < kDispatchSteps; ++u)
            c += __popc(hit_mask(v[u], e));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        c += __shfl_xor_sync(kFull, c, off);
    return c;
}

// Exclusive prefix of one count per warp, in warp order, and the block total.
template <int WARPS>
__device__ __forceinline__ int warp_prefix(int warp_total, int *total)
{
    __shared__ int sums[WARPS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
        sums[warp] = warp_total;
    __syncthreads();
    int before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
        before += w < warp ? sums[w] : 0;
        all += sums[w];
    }
    *total = all;
    return before;
}

template <bool VEC, int WARPS>
__global__ void __launch_bounds__(WARPS * 32) moe_count_kernel(const int32_t *__restrict__ experts,
                                                               int64_t n, int32_t *offsets)
{
    const int e = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int64_t seg = dispatch_segment<WARPS>(n);
    const int64_t lo = warp * seg;
    const int64_t hi = lo + seg < n ? lo + seg : n;
    const int c = warp_count<VEC>(experts, lo, hi, n, e);
    int total = 0;
    (void)warp_prefix<WARPS>(c, &total);
    if (threadIdx.x == 0)
        offsets[e + 1] = total;
}

__global__ void __launch_bounds__(kMaxE) moe_scan_kernel(int32_t *offsets, int E)
{
    __shared__ int32_t sc[kMaxE];
    const int i = threadIdx.x;
    sc[i] = i < E ? offsets[i + 1] : 0;
    __syncthreads();
    for (int w = 1; w < kMaxE; w <<= 1) {   // inclusive Hillis-Steele scan (integers)
        const int32_t add = i >= w ? sc[i - w] : 0;
        __syncthreads();
        sc[i] += add;
        __syncthreads();
    }
    if (i < E)
        offsets[i + 1] = sc[i];
    if (i == 0)
        offsets[0] = 0;
}

template <bool VEC, int WARPS>
__global__ void __launch_bounds__(WARPS * 32) moe_fill_kernel(const int32_t *__restrict__ experts,
                                                              int64_t n, int k,
                                                              const int32_t *__restrict__ offsets,
                                                              int32_t *__restrict__ token_of_row,
                                                              int32_t *__restrict__ row_of_slot)
{
    const int e = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t seg = dispatch_segment<WARPS>(n);
    const int64_t lo = warp * seg;
    const int64_t hi = lo + seg < n ? lo + seg : n;
    const int c = warp_count<VEC>(experts, lo, hi, n, e);
    int total = 0;
    int32_t r = offsets[e] + warp_prefix<WARPS>(c, &total);   // this warp's first row
    if (c == 0)
        return;
    for (int64_t base = lo; base < hi; base += kDispatchSteps * 128) {
        int4 v[kDispatchSteps];
#pragma unroll
        for (int u = 0; u < kDispatchSteps; ++u) {
            const int64_t i = base + 128 * u + 4 * lane;
            v[u] = (base + 128 * u < hi) ? load_ids<VEC>(experts, i, n) : make_int4(-1, -1, -1, -1);
        }
#pragma unroll
        for (int u = 0; u < kDispatchSteps; ++u) {
            const uint32_t m = hit_mask(v[u], e);
            const int h = __popc(m);
            int incl = h;   // rows of the lanes before this one in the step, then this lane's
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(kFull, incl, off);
                if (lane >= off)
                    incl += y;
            }
            int32_t row = r + incl - h;
            const int64_t i0 = base + 128 * u + 4 * lane;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if ((m >> j) & 1u) {
                    token_of_row[row] = static_cast<int32_t>((i0 + j) / k);
                    row_of_slot[i0 + j] = row;
                    ++row;
                }
            r += __shfl_sync(kFull, incl, 31);   // the step's hits
        }
    }
}

// Few pairs (up to kPassPairs): one block per expert walks all pairs in passes of 256 x 8
// consecutive pairs (thread t owns pairs 8t .. 8t+7 of a pass), ranking its hits with one block
// scan per pass.  Same grouping as the segment kernels above; fewer steps when there are few pairs.
constexpr int kPerThread = 8;
constexpr int64_t kPassPairs = 4096;

__global__ void __launch_bounds__(256) moe_count_pass_kernel(const int32_t *experts, int64_t n,
                                                        int32_t *offsets)
{
    const int e = blockIdx.x;
    int c = 0;
    for (int64_t base = static_cast<int64_t>(threadIdx.x) * kPerThread; base < n;
         base += static_cast<int64_t>(blockDim.x) * kPerThread) {
#pragma unroll
        for (int q = 0; q < kPerThread; ++q)
            c += (base + q < n && experts[base + q] == e) ? 1 : 0;
    }
    __shared__ int part[256];
    part[threadIdx.x] = c;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w)
            part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0)
        offsets[e + 1] = part[0];
}

__global__ void __launch_bounds__(256) moe_fill_pass_kernel(const int32_t *experts, int64_t n, int k,
                                                       const int32_t *offsets, int32_t *token_of_row,
                                                       int32_t *row_of_slot)
{
    // One block per expert.  A pass covers 256 * 8 consecutive pairs: thread t owns the 8 pairs
    // [base + 8t, base + 8t + 8), so an exclusive scan of the per-thread hit counts in thread
    // order places the expert's rows in ascending pair order.
    const int e = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ int32_t wsum[8];
    int32_t running = offsets[e];
    const int64_t span = static_cast<int64_t>(blockDim.x) * kPerThread;
    for (int64_t base = 0; base < n; base += span) {
        const int64_t i0 = base + static_cast<int64_t>(threadIdx.x) * kPerThread;
        uint32_t hits = 0;
#pragma unroll
        for (int q = 0; q < kPerThread; ++q)
            if (i0 + q < n && experts[i0 + q] == e)
                hits |= 1u << q;
        const int cnt = __popc(hits);
        int incl = cnt;   // inclusive scan inside the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, off);
            if (lane >= off)
                incl += y;
        }
        if (lane == 31)
            wsum[warp] = incl;
        __syncthreads();
        int32_t before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            before += w < warp ? wsum[w] : 0;
            total += wsum[w];
        }
        int32_t r = running + before + incl - cnt;
#pragma unroll
        for (int q = 0; q < kPerThread; ++q)
            if ((hits >> q) & 1u) {
                token_of_row[r] = static_cast<int32_t>((i0 + q) / k);
                row_of_slot[i0 + q] = r;
                ++r;
            }
        running += total;
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------------------------
// Gather and combine: 16-byte vectors of 8 bf16
// ---------------------------------------------------------------------------------------------

__global__ void __launch_bounds__(256) moe_gather_kernel(const __nv_bfloat16 *X, int64_t ldx,
                                                         int64_t vecs_per_row, const int32_t *tok,
                                                         int64_t R, __nv_bfloat16 *A, int64_t lda)
{
    const int64_t total = R * vecs_per_row;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = idx / vecs_per_row;
        const int64_t v = idx - r * vecs_per_row;
        const uint4 *src = reinterpret_cast<const uint4 *>(X + static_cast<int64_t>(tok[r]) * ldx) + v;
        uint4 *dst = reinterpret_cast<uint4 *>(A + r * lda) + v;
        *dst = __ldg(src);
    }
}

__global__ void __launch_bounds__(256) moe_combine_kernel(const __nv_bfloat16 *C, int64_t ldc,
                                                          int64_t vecs_per_row,
                                                          const int32_t *row_of_slot,
                                                          const float *weights, int64_t T, int k,
                                                          __nv_bfloat16 *Y, int64_t ldy)
{
    const int64_t total = T * vecs_per_row;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = idx / vecs_per_row;
        const int64_t v = idx - t * vecs_per_row;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            acc[q] = 0.0f;
        for (int j = 0; j < k; ++j) {   // slot order: descending router logit
            const int64_t r = row_of_slot[t * k + j];
            const float w = weights[t * k + j];
            const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(C + r * ldc) + v);
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = __bfloat1622float2(h[q]);
                acc[2 * q] = fmaf(w, f.x, acc[2 * q]);
                acc[2 * q + 1] = fmaf(w, f.y, acc[2 * q + 1]);
            }
        }
        uint4 out;
        uint32_t *o = reinterpret_cast<uint32_t *>(&out);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            __nv_bfloat162 hh = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
            o[q] = *reinterpret_cast<uint32_t *>(&hh);
        }
        *(reinterpret_cast<uint4 *>(Y + t * ldy) + v) = out;
    }
}

// ---------------------------------------------------------------------------------------------
// host helpers
// ---------------------------------------------------------------------------------------------

bi_status_t moe_device(int *num_sms)
{
    int count = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess || count <= 0) {
        cudaGetLastError();
        return BI_ERR_NO_DEVICE;
    }
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return BI_ERR_CUDA;
    return major == 10 ? BI_OK : BI_ERR_NO_DEVICE;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int grid_for(int64_t work, int num_sms)
{
    const int64_t blocks = (work + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms) * 16;
    return static_cast<int>(blocks < 1 ? 1 : blocks < cap ? blocks : cap);
}

bi_status_t last_launch() { return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA; }

} // namespace

extern "C" {

bi_status_t bi_moe_route_topk(const float *logits, int64_t ld_logits, int64_t T, int E, int k,
                              int32_t *experts, float *weights, cudaStream_t stream)
{
    if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > kMaxK || k > E || ld_logits < E)
        return BI_ERR_INVALID_ARG;
    if (T == 0)
        return BI_OK;
    if (!logits || !experts || !weights)
        return BI_ERR_INVALID_ARG;
    if (!aligned(logits, 4) || !aligned(experts, 4) || !aligned(weights, 4))
        return BI_ERR_ALIGNMENT;
    if (T > (INT64_C(1) << 31) / k)
        return BI_ERR_UNSUPPORTED_SHAPE;
    int sms = 0;
    bi_status_t st = moe_device(&sms);
    if (st != BI_OK)
        return st;
    const unsigned blocks = static_cast<unsigned>((T * 32 + 255) / 256);
    const int pl = (E + 31) / 32;
    if (pl <= 1)
        moe_route_kernel<1><<<blocks, 256, 0, stream>>>(logits, ld_logits, T, E, k, experts, weights);
    else if (pl <= 2)
        moe_route_kernel<2><<<blocks, 256, 0, stream>>>(logits, ld_logits, T, E, k, experts, weights);
    else if (pl <= 4)
        moe_route_kernel<4><<<blocks, 256, 0, stream>>>(logits, ld_logits, T, E, k, experts, weights);
    else if (pl <= 8)
        moe_route_kernel<8><<<blocks, 256, 0, stream>>>(logits, ld_logits, T, E, k, experts, weights);
    else if (pl <= 16)
        moe_route_kernel<16><<<blocks, 256, 0, stream>>>(logits, ld_logits, T, E, k, experts, weights);
    else
        moe_route_kernel<32><<<blocks, 256, 0, stream>>>(logits, ld_logits, T, E, k, experts, weights);
    return last_launch();
}

bi_status_t bi_moe_dispatch(const int32_t *experts, int64_t T, int E, int k, int32_t *offsets,
                            int32_t *token_of_row, int32_t *row_of_slot, cudaStream_t stream)
{
    if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > kMaxK)
        return BI_ERR_INVALID_ARG;
    if (!offsets)
        return BI_ERR_INVALID_ARG;
    if (T > 0 && (!experts || !token_of_row || !row_of_slot))
        return BI_ERR_INVALID_ARG;
    if (!aligned(offsets, 4) || !aligned(experts, 4) || !aligned(token_of_row, 4) ||
        !aligned(row_of_slot, 4))
        return BI_ERR_ALIGNMENT;
    if (T > ((INT64_C(1) << 31) - 1) / k)
        return BI_ERR_UNSUPPORTED_SHAPE;
    int sms = 0;
    bi_status_t st = moe_device(&sms);
    if (st != BI_OK)
        return st;
    const int64_t n = T * k;
    if (n <= kPassPairs) {
        moe_count_pass_kernel<<<E, 256, 0, stream>>>(experts, n, offsets);
        if ((st = last_launch()) != BI_OK)
            return st;
        moe_scan_kernel<<<1, kMaxE, 0, stream>>>(offsets, E);
        if ((st = last_launch()) != BI_OK)
            return st;
        if (n == 0)
            return BI_OK;
        moe_fill_pass_kernel<<<E, 256, 0, stream>>>(experts, n, k, offsets, token_of_row, row_of_slot);
        return last_launch();
    }
    const bool vec = aligned(experts, 16);
    const bool few = n <= kFewPairs;
    auto count = [&](auto vec_tag, auto warps_tag) {
        constexpr bool V = decltype(vec_tag)::value;
        constexpr int W = decltype(warps_tag)::value;
        moe_count_kernel<V, W><<<E, W * 32, 0, stream>>>(experts, n, offsets);
    };
    auto fill = [&](auto vec_tag, auto warps_tag) {
        constexpr bool V = decltype(vec_tag)::value;
        constexpr int W = decltype(warps_tag)::value;
        moe_fill_kernel<V, W><<<E, W * 32, 0, stream>>>(experts, n, k, offsets, token_of_row, row_of_slot);
    };
    using T8 = std::integral_constant<int, 8>;
    using T32 = std::integral_constant<int, 32>;
    using VT = std::true_type;
    using VF = std::false_type;
    if (vec)
        few ? count(VT{}, T8{}) : count(VT{}, T32{});
    else
        few ? count(VF{}, T8{}) : count(VF{}, T32{});
    if ((st = last_launch()) != BI_OK)
        return st;
    moe_scan_kernel<<<1, kMaxE, 0, stream>>>(offsets, E);
    if ((st = last_launch()) != BI_OK)
        return st;
    if (n == 0)
        return BI_OK;
    if (vec)
        few ? fill(VT{}, T8{}) : fill(VT{}, T32{});
    else
        few ? fill(VF{}, T8{}) : fill(VF{}, T32{});
    return last_launch();
}

bi_status_t bi_moe_gather_rows(const void *X, int64_t ldx, int64_t K, const int32_t *token_of_row,
                               int64_t R, void *A_perm, int64_t lda, cudaStream_t stream)
{
    if (R < 0 || K < 0 || ldx < K || lda < K)
        return BI_ERR_INVALID_ARG;
    if (R == 0 || K == 0)
        return BI_OK;
    if (!X || !token_of_row || !A_perm)
        return BI_ERR_INVALID_ARG;
    if (K % 8 != 0)
        return BI_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(X, 16) || !aligned(A_perm, 16) || !aligned(token_of_row, 4) || ldx % 8 || lda % 8)
        return BI_ERR_ALIGNMENT;
    int sms = 0;
    bi_status_t st = moe_device(&sms);
    if (st != BI_OK)
        return st;
    const int64_t vpr = K / 8;
    moe_gather_kernel<<<grid_for(R * vpr, sms), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(X), ldx, vpr, token_of_row, R,
        static_cast<__nv_bfloat16 *>(A_perm), lda);
    return last_launch();
}

bi_status_t bi_moe_combine(const void *C_perm, int64_t ldc, int64_t N, const int32_t *row_of_slot,
                           const float *weights, int64_t T, int k, void *Y, int64_t ldy,
                           cudaStream_t stream)
{
    if (T < 0 || N < 0 || k < 1 || k > kMaxK || ldc < N || ldy < N)
        return BI_ERR_INVALID_ARG;
    if (T == 0 || N == 0)
        return BI_OK;
    if (!C_perm || !row_of_slot || !weights || !Y)
        return BI_ERR_INVALID_ARG;
    if (N % 8 != 0)
        return BI_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(C_perm, 16) || !aligned(Y, 16) || !aligned(row_of_slot, 4) || !aligned(weights, 4) ||
        ldc % 8 || ldy % 8)
        return BI_ERR_ALIGNMENT;
    int sms = 0;
    bi_status_t st = moe_device(&sms);
    if (st != BI_OK)
        return st;
    const int64_t vpr = N / 8;
    moe_combine_kernel<<<grid_for(T * vpr, sms), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(C_perm), ldc, vpr, row_of_slot, weights, T, k,
        static_cast<__nv_bfloat16 *>(Y), ldy);
    return last_launch();
}

} // extern "C"
