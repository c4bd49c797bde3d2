// bi_attention.cu -- dual-kernel decode attention (include/bi_attention.h).
//
// One CTA serves one (sequence, key/value head) pair -- or, split-KV, a part of its chunks --
// with one warp per query head of the group (grouped-query attention).  A sequence's keys are cut
// into kChunks = 4 chunks by its own length, and every chunk is reduced by chunk_attention():
// blocks of 32 keys in ascending order, lane j scoring key j (q . k_j as two partial sums over
// the even and the odd d, each ascending, then added),
// an online softmax whose block max and block sum are fixed butterflies, and the value sum
// o = o * corr + sum_j p_j v_j with j ascending.  merge() combines two chunk results, always as
// ((c0 + c1) + (c2 + c3)).  The no-split kernel and the split-KV kernels run exactly this
// arithmetic, so their outputs are bitwise equal.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "bi_attention.h"

namespace {

constexpr int kD = 128;             // head dimension
constexpr int kChunks = 4;          // chunks per sequence (fixed: the merge tree has 4 leaves)
constexpr int kBlockKeys = 32;      // keys per block = lanes of a warp
constexpr int kMaxGroup = 8;        // query heads per key/value head
constexpr int kRowStride = kD * 2 + 16;   // bytes per key row in shared memory (bank spread)
constexpr unsigned kFull = 0xffffffffu;

// The running state of one query head: max, sum of exp, and this lane's 4 output dimensions
// (unnormalised).
struct Partial {
    float m, l;
    float o[4];
};

__device__ __forceinline__ Partial empty_partial()
{
    Partial p;
    p.m = -INFINITY;
    p.l = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        p.o[i] = 0.0f;
    return p;
}

// a + b of two partials of the same query head (same lane's dimensions).
__device__ __forceinline__ Partial merge(const Partial &a, const Partial &b)
{
    const float m = fmaxf(a.m, b.m);
    if (m == -INFINITY)
        return a;   // both empty
    const float fa = expf(a.m - m);
    const float fb = expf(b.m - m);
    Partial r;
    r.m = m;
    r.l = fmaf(b.l, fb, a.l * fa);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        r.o[i] = fmaf(b.o[i], fb, a.o[i] * fa);
    return r;
}

// Two fused multiply-adds in one instruction (sm_100's packed fp32 pipe): r.x = fma(a.x, b.x, c.x)
// and r.y = fma(a.y, b.y, c.y), each rounded to nearest like fmaf.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool valid)
{
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const int n = valid ? 16 : 0;   // 0: fill the 16 bytes with zeros
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

struct AttnArgs {
    const __nv_bfloat16 *q, *k, *v;
    const int32_t *lengths;
    int64_t lmax;
    int hq, hkv, group;
    float scale;
};

// A group of `nthreads` threads of the CTA (thread `tid` of the group; one warp per query head)
// that synchronises on named barrier `bar` (0: the whole CTA).
struct Group {
    int tid, nthreads, bar;
};

__device__ __forceinline__ void group_sync(const Group &g)
{
    if (g.bar == 0)
        __syncthreads();
    else
        asm volatile("bar.sync %0, %1;" ::"r"(g.bar), "r"(g.nthreads) : "memory");
}

// Keys [k0, k1) of sequence b, key/value head kvh, into this warp's partial.  Every thread of the
// group calls it with the same arguments (it loads shared K/V blocks into kv_s and synchronises
// the group).  The K/V blocks stream through S shared-memory stages, S - 1 blocks ahead of the one
// being reduced; the depth changes when a block arrives, never the arithmetic.
template <int S>
__device__ Partial chunk_attention(const AttnArgs &a, int64_t b, int kvh, int k0, int k1,
                                   const float *q_s, uint8_t *kv_s, const Group &grp)
{
    static_assert(S >= 2, "at least double buffering");
    const int warp = grp.tid >> 5, lane = grp.tid & 31;
    const int nthreads = grp.nthreads;
    Partial st = empty_partial();
    const int nblk = (k1 - k0 + kBlockKeys - 1) / kBlockKeys;
    const int64_t row_pitch = static_cast<int64_t>(a.hkv) * kD;   // elements between keys
    const __nv_bfloat16 *kbase = a.k + (b * a.lmax * a.hkv + kvh) * kD;
    const __nv_bfloat16 *vbase = a.v + (b * a.lmax * a.hkv + kvh) * kD;
    auto load_block = [&](int blk, int buf) {
        uint8_t *ks = kv_s + buf * 2 * kBlockKeys * kRowStride;
        uint8_t *vs = ks + kBlockKeys * kRowStride;
        // 32 keys x 16 pieces of 16 bytes, for K and for V
        for (int i = grp.tid; i < kBlockKeys * 16; i += nthreads) {
            const int j = i >> 4, piece = i & 15;
            const int key = k0 + blk * kBlockKeys + j;
            const bool ok = key < k1;
            const int64_t off = (ok ? key : k0) * row_pitch + piece * 8;
            cp_async16(ks + j * kRowStride + piece * 16, kbase + off, ok);
            cp_async16(vs + j * kRowStride + piece * 16, vbase + off, ok);
        }
    };
    // blocks 0 .. S-2 first, one commit group each (empty groups past the end keep the count)
#pragma unroll
    for (int i = 0; i < S - 1; ++i) {
        if (i < nblk)
            load_block(i, i);
        cp_async_commit();
    }
    for (int blk = 0; blk < nblk; ++blk) {
        // block blk + S - 1 into the stage block blk - 1 used (freed by the barrier that ended
        // the previous iteration)
        if (blk + S - 1 < nblk)
            load_block(blk + S - 1, (blk + S - 1) % S);
        cp_async_commit();
        cp_async_wait<S - 1>();   // block blk's group (number blk) has landed
        group_sync(grp);
        const uint8_t *ks = kv_s + (blk % S) * 2 * kBlockKeys * kRowStride;
        const uint8_t *vs = ks + kBlockKeys * kRowStride;
        if (warp < a.group) {
            // lane j: the score of key j of the block, as two partial sums -- even d and odd d,
            // each in ascending d -- added at the end
            const int key = k0 + blk * kBlockKeys + lane;
            const float2 *qh = reinterpret_cast<const float2 *>(q_s + warp * kD);
            const uint4 *krow = reinterpret_cast<const uint4 *>(ks + lane * kRowStride);
            float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll 4
            for (int piece = 0; piece < 16; ++piece) {
                const uint4 raw = krow[piece];
                const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    s2 = fma2(qh[piece * 4 + t], __bfloat1622float2(h2[t]), s2);
            }
            float s = s2.x + s2.y;
            s = key < k1 ? s * a.scale : -INFINITY;
            float mb = s;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, off));
            const float m_new = fmaxf(st.m, mb);
            const float corr = expf(st.m - m_new);   // 0 for the first block (st.m = -inf)
            const float p = expf(s - m_new);         // 0 for masked keys
            float ps = p;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                ps = ps + __shfl_xor_sync(kFull, ps, off);
            st.l = fmaf(st.l, corr, ps);
            // o = o * corr + sum_j p_j v_j, j ascending (two dimensions per packed FMA: the same
            // roundings as four fmaf)
            float2 acc01 = make_float2(st.o[0] * corr, st.o[1] * corr);
            float2 acc23 = make_float2(st.o[2] * corr, st.o[3] * corr);
            for (int j = 0; j < kBlockKeys; ++j) {
                const float pj = __shfl_sync(kFull, p, j);
                const float2 pp = make_float2(pj, pj);
                const __nv_bfloat162 *vrow =
                    reinterpret_cast<const __nv_bfloat162 *>(vs + j * kRowStride) + lane * 2;
                acc01 = fma2(pp, __bfloat1622float2(vrow[0]), acc01);
                acc23 = fma2(pp, __bfloat1622float2(vrow[1]), acc23);
            }
            st.o[0] = acc01.x;
            st.o[1] = acc01.y;
            st.o[2] = acc23.x;
            st.o[3] = acc23.y;
            st.m = m_new;
        }
        group_sync(grp);   // the stage is refilled in the next iteration
    }
    return st;
}

__device__ __forceinline__ int chunk_begin(int c, int L) { return static_cast<int>((static_cast<int64_t>(c) * L) / kChunks); }

// Load the group's query heads into shared memory as fp32.
__device__ void load_q(const AttnArgs &a, int64_t b, int kvh, float *q_s)
{
    for (int i = threadIdx.x; i < a.group * kD; i += blockDim.x) {
        const int h = kvh * a.group + i / kD;
        q_s[i] = __bfloat162float(a.q[(b * a.hq + h) * kD + (i % kD)]);
    }
    __syncthreads();
}

__device__ __forceinline__ int valid_length(const AttnArgs &a, int64_t b)
{
    const int L = a.lengths[b];
    return (L >= 1 && L <= a.lmax) ? L : -1;
}

__device__ __forceinline__ void store_output(const AttnArgs &a, int64_t b, int h, const Partial &p,
                                             bool valid, __nv_bfloat16 *out)
{
    const int lane = threadIdx.x & 31;
    __nv_bfloat16 *o = out + (b * a.hq + h) * kD + lane * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        o[i] = __float2bfloat16_rn(valid ? p.o[i] / p.l : NAN);
}

// No split: one CTA per (sequence, key/value head) walks the 4 chunks and merges them.
template <int S>
__global__ void __launch_bounds__(256, 2) attn_nosplit_kernel(AttnArgs a, __nv_bfloat16 *out)
{
    extern __shared__ __align__(16) uint8_t smem[];
    float *q_s = reinterpret_cast<float *>(smem);
    uint8_t *kv_s = smem + kMaxGroup * kD * 4;
    const int64_t b = blockIdx.x / a.hkv;
    const int kvh = blockIdx.x % a.hkv;
    const int L = valid_length(a, b);
    load_q(a, b, kvh, q_s);
    Partial c[kChunks];
#pragma unroll
    for (int ci = 0; ci < kChunks; ++ci)
        c[ci] = L > 0 ? chunk_attention<S>(a, b, kvh, chunk_begin(ci, L), chunk_begin(ci + 1, L), q_s, kv_s,
                                           Group{static_cast<int>(threadIdx.x), static_cast<int>(blockDim.x), 0})
                      : empty_partial();
    const int warp = threadIdx.x >> 5;
    if (warp < a.group)
        store_output(a, b, kvh * a.group + warp, merge(merge(c[0], c[1]), merge(c[2], c[3])), L > 0, out);
}

// No split, the four chunks at once (query groups of up to 4 heads): warp group c -- one warp per
// query head -- reduces chunk c with its own K/V stages and named barrier 1 + c; the four partials
// meet in shared memory and group 0 merges them as ((c0 + c1) + (c2 + c3)).  Each chunk is the
// same chunk_attention() call as in the kernels above, so the outputs are bitwise equal to theirs.
constexpr int kParStages = 3;
constexpr int kStageBytes = 2 * kBlockKeys * kRowStride;   // one K block and one V block

__global__ void __launch_bounds__(kChunks * 4 * 32, 1) attn_nosplit_par_kernel(AttnArgs a,
                                                                              __nv_bfloat16 *out)
{
    extern __shared__ __align__(16) uint8_t smem[];
    float *q_s = reinterpret_cast<float *>(smem);
    uint8_t *kv_base = smem + kMaxGroup * kD * 4;
    const int64_t b = blockIdx.x / a.hkv;
    const int kvh = blockIdx.x % a.hkv;
    const int L = valid_length(a, b);
    load_q(a, b, kvh, q_s);
    const int gthreads = 32 * a.group;
    const int c = static_cast<int>(threadIdx.x) / gthreads;
    const Group grp{static_cast<int>(threadIdx.x) - c * gthreads, gthreads, 1 + c};
    const Partial r = L > 0 ? chunk_attention<kParStages>(a, b, kvh, chunk_begin(c, L), chunk_begin(c + 1, L), q_s,
                                                          kv_base + c * kParStages * kStageBytes, grp)
                            : empty_partial();
    __syncthreads();   // every group is done with its stages: they now hold the partials
    float *part = reinterpret_cast<float *>(kv_base);   // [chunk][head][m, l, o[kD]]
    const int warp = grp.tid >> 5, lane = threadIdx.x & 31;
    float *w = part + (c * kMaxGroup + warp) * (kD + 2);
    if (lane == 0) {
        w[0] = r.m;
        w[1] = r.l;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[2 + lane * 4 + i] = r.o[i];
    __syncthreads();
    if (c == 0) {
        Partial p[kChunks];
#pragma unroll
        for (int ci = 0; ci < kChunks; ++ci) {
            const float *q = part + (ci * kMaxGroup + warp) * (kD + 2);
            p[ci].m = q[0];
            p[ci].l = q[1];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                p[ci].o[i] = q[2 + lane * 4 + i];
        }
        store_output(a, b, kvh * a.group + warp, merge(merge(p[0], p[1]), merge(p[2], p[3])), L > 0, out);
    }
}

// Split-KV: CTA `part` of `splits` for (sequence, key/value head) reduces chunks
// [part * 4 / splits, (part + 1) * 4 / splits) (merging them pairwise when it has two) and writes
// its partial to ws[((b * hq + h) * 4 + part) * (kD + 2)].
template <int S>
__global__ void __launch_bounds__(256, 2) attn_split_kernel(AttnArgs a, int splits, float *ws)
{
    extern __shared__ __align__(16) uint8_t smem[];
    float *q_s = reinterpret_cast<float *>(smem);
    uint8_t *kv_s = smem + kMaxGroup * kD * 4;
    const int part = blockIdx.x % splits;
    const int64_t pair = blockIdx.x / splits;
    const int64_t b = pair / a.hkv;
    const int kvh = static_cast<int>(pair % a.hkv);
    const int L = valid_length(a, b);
    load_q(a, b, kvh, q_s);
    const int per = kChunks / splits;
    const Group all{static_cast<int>(threadIdx.x), static_cast<int>(blockDim.x), 0};
    Partial r = empty_partial();
    if (L > 0) {
        if (per == 1) {
            r = chunk_attention<S>(a, b, kvh, chunk_begin(part, L), chunk_begin(part + 1, L), q_s, kv_s, all);
        } else {
            const Partial c0 = chunk_attention<S>(a, b, kvh, chunk_begin(2 * part, L), chunk_begin(2 * part + 1, L), q_s, kv_s, all);
            const Partial c1 = chunk_attention<S>(a, b, kvh, chunk_begin(2 * part + 1, L), chunk_begin(2 * part + 2, L), q_s, kv_s, all);
            r = merge(c0, c1);
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < a.group) {
        const int h = kvh * a.group + warp;
        float *w = ws + ((b * a.hq + h) * kChunks + part) * (kD + 2);
        if (lane == 0) {
            w[0] = r.m;
            w[1] = r.l;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[2 + lane * 4 + i] = r.o[i];
    }
}

// Merge of the split partials: one warp per (sequence, query head).
__global__ void __launch_bounds__(256) attn_merge_kernel(AttnArgs a, int splits, const float *ws,
                                                         __nv_bfloat16 *out, int64_t B)
{
    const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= B * a.hq)
        return;
    const int64_t b = wid / a.hq;
    const int h = static_cast<int>(wid % a.hq);
    Partial p[kChunks];
    for (int part = 0; part < splits; ++part) {
        const float *w = ws + (wid * kChunks + part) * (kD + 2);
        p[part].m = w[0];
        p[part].l = w[1];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            p[part].o[i] = w[2 + lane * 4 + i];
    }
    const Partial r = splits == 4 ? merge(merge(p[0], p[1]), merge(p[2], p[3])) : merge(p[0], p[1]);
    store_output(a, b, h, r, valid_length(a, b) > 0, out);
}

bi_status_t attn_device(int *num_sms)
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

template <int S>
constexpr int smem_bytes() { return kMaxGroup * kD * 4 + S * 2 * kBlockKeys * kRowStride; }

// Stage depths: a launch with at most two CTAs per SM takes the deep pipeline (6 stages, 108 KB,
// two CTAs per SM), any other the shallow one (2 stages, 39 KB, five CTAs per SM): with few CTAs a
// CTA needs many blocks in flight, with many CTAs occupancy matters more.
constexpr int kDeep = 6, kShallow = 2;
constexpr int kParSmemBytes = kMaxGroup * kD * 4 + kChunks * kParStages * kStageBytes;
static_assert(kChunks * kMaxGroup * (kD + 2) * 4 <= kChunks * kParStages * kStageBytes,
              "the partials fit in the stages");

// Both kernels at both depths need more than the default 48 KB of dynamic shared memory; the
// opt-in is set once per device.
std::mutex g_attr_mu;
bool g_attr_set[64] = {};

bi_status_t ensure_attributes(int dev)
{
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (dev < 0 || dev >= 64)
        return BI_ERR_CUDA;
    if (g_attr_set[dev])
        return BI_OK;
    const cudaFuncAttribute attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
    if (cudaFuncSetAttribute(attn_nosplit_par_kernel, attr, kParSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(attn_nosplit_kernel<kDeep>, attr, smem_bytes<kDeep>()) != cudaSuccess ||
        cudaFuncSetAttribute(attn_nosplit_kernel<kShallow>, attr, smem_bytes<kShallow>()) != cudaSuccess ||
        cudaFuncSetAttribute(attn_split_kernel<kDeep>, attr, smem_bytes<kDeep>()) != cudaSuccess ||
        cudaFuncSetAttribute(attn_split_kernel<kShallow>, attr, smem_bytes<kShallow>()) != cudaSuccess)
        return BI_ERR_CUDA;
    g_attr_set[dev] = true;
    return BI_OK;
}

} // namespace

extern "C" {

size_t bi_decode_attention_workspace_bytes(int64_t B, int Hq, int D, int splits)
{
    if (B <= 0 || Hq <= 0 || D <= 0 || splits <= 1)
        return 0;
    return static_cast<size_t>(B) * static_cast<size_t>(Hq) * kChunks * static_cast<size_t>(D + 2) * 4u;
}

bi_status_t bi_decode_attention(const void *Q, const void *K, const void *V,
                                const int32_t *lengths, int64_t B, int Hq, int Hkv, int D,
                                int64_t Lmax, float scale, int splits, float *workspace,
                                size_t workspace_bytes, void *O, cudaStream_t stream)
{
    if (B < 0 || Hq < 1 || Hkv < 1 || Lmax < 1 || (splits != 0 && splits != 1 && splits != 2 && splits != 4))
        return BI_ERR_INVALID_ARG;
    if (D != kD || Hq % Hkv != 0 || Hq / Hkv > kMaxGroup)
        return BI_ERR_UNSUPPORTED_SHAPE;
    if (B == 0)
        return BI_OK;
    if (!Q || !K || !V || !lengths || !O)
        return BI_ERR_INVALID_ARG;
    auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!al16(Q) || !al16(K) || !al16(V) || !al16(O) || (reinterpret_cast<uintptr_t>(lengths) & 3u))
        return BI_ERR_ALIGNMENT;
    if (Lmax > INT32_MAX / 4 || B * Hkv > INT32_MAX / 4)
        return BI_ERR_UNSUPPORTED_SHAPE;
    int sms = 0;
    bi_status_t st = attn_device(&sms);
    if (st != BI_OK)
        return st;
    if (splits == 0) {   // automatic: the fewest splits that give every SM a CTA (no bit changes)
        splits = 4;
        for (int s = 1; s <= 2; s *= 2)
            if (B * Hkv * s >= sms) {
                splits = s;
                break;
            }
    }
    if (splits > 1) {
        if (!workspace || workspace_bytes < bi_decode_attention_workspace_bytes(B, Hq, D, splits))
            return BI_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(workspace) & 15u)
            return BI_ERR_ALIGNMENT;
    }
    AttnArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(Q);
    a.k = static_cast<const __nv_bfloat16 *>(K);
    a.v = static_cast<const __nv_bfloat16 *>(V);
    a.lengths = lengths;
    a.lmax = Lmax;
    a.hq = Hq;
    a.hkv = Hkv;
    a.group = Hq / Hkv;
    a.scale = scale;
    const int threads = 32 * a.group;
    const int64_t pairs = B * Hkv;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || (st = ensure_attributes(dev)) != BI_OK)
        return st == BI_OK ? BI_ERR_CUDA : st;
    const bool deep = pairs * splits <= 2LL * sms;
    // No split with at most one CTA per SM: the four chunks at once (with more CTAs the shallow
    // sequential kernel keeps five CTAs per SM instead)
    if (splits == 1 && a.group <= 4 && pairs <= sms) {
        attn_nosplit_par_kernel<<<static_cast<unsigned>(pairs), kChunks * threads, kParSmemBytes, stream>>>(
            a, static_cast<__nv_bfloat16 *>(O));
        return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
    }
    if (splits == 1) {
        if (deep)
            attn_nosplit_kernel<kDeep><<<static_cast<unsigned>(pairs), threads, smem_bytes<kDeep>(), stream>>>(
                a, static_cast<__nv_bfloat16 *>(O));
        else
            attn_nosplit_kernel<kShallow><<<static_cast<unsigned>(pairs), threads, smem_bytes<kShallow>(), stream>>>(
                a, static_cast<__nv_bfloat16 *>(O));
        return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
    }
    if (deep)
        attn_split_kernel<kDeep><<<static_cast<unsigned>(pairs * splits), threads, smem_bytes<kDeep>(), stream>>>(
            a, splits, workspace);
    else
        attn_split_kernel<kShallow><<<static_cast<unsigned>(pairs * splits), threads, smem_bytes<kShallow>(), stream>>>(
            a, splits, workspace);
    if (cudaGetLastError() != cudaSuccess)
        return BI_ERR_CUDA;
    const int64_t warps = B * Hq;
    attn_merge_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, stream>>>(
        a, splits, workspace, static_cast<__nv_bfloat16 *>(O), B);
    return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

} // extern "C"
