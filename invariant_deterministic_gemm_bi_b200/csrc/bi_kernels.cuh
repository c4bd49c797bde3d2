// bi_kernels.cuh -- persistent, warp-specialised tcgen05 GEMM kernels for sm_100a.
//
//   C[M,N] = A[M,K] . B[N,K]^T,  fp32 accumulation in tensor memory, bf16 output.
//
// Batch invariance ("DeepSeek不惜代价保住它！V4关键特性被挖出来了" (QbitAI), sections
// "什么是batch invariance" and "牺牲了什么"): the bits of C[m,:] must not depend on M, on m or on
// the other rows.  A split K axis would be summed in an order that changes with the split, so
// here one CTA owns the whole K range of its 128 x BN output tile: the MMA warp issues the
// K-slices of the tile in ascending order into one TMEM accumulator (no split-K, no atomics,
// no cross-CTA reduction).  The tile shape, the MMA instruction shape and the K order are
// template constants chosen by the host plan from (N, K, dtype) only.  Rows past the end of A
// are zero-filled by TMA and never stored.  When the whole problem has fewer rows than a tile,
// TMA brings only those rows of the A tile; the MMA still runs on all BM rows, and the rows never
// loaded feed only output rows that are never stored (every output element depends on its own A
// row alone).  The CTA <-> tile mapping does depend on M, which is
// harmless: it decides where a tile is computed, not how.
//
// Roles inside a CTA (6 warps = 192 threads):
//   warp 0, lane 0 : TMA producer -- A tiles [BM x 128 B] and B tiles [BN x 128 B] into two
//                    shared-memory rings (128-byte swizzle).  The B (weight) ring is deeper
//                    than the A ring: B streams from HBM and needs many bytes in flight, A is
//                    small and L2-resident when the batch is small, so B loads run SB - SA
//                    K blocks ahead of the A loads of the same K block.
//   warp 1         : allocates tensor memory; lane 0 issues tcgen05.mma and commits
//   warps 2..5     : epilogue -- tcgen05.ld from TMEM, fp32 -> bf16 (RNE), masked stores
//   (FP8 tiles at least 64 wide have 8 epilogue warps, 2..9; the dense wide lockstep form adds
//   one more warp after the epilogue warps whose lane 0 issues the second column half's MMAs)
// bf16: the accumulator is double-buffered in TMEM so the epilogue of tile i overlaps the
// MMAs of tile i+1.  FP8 (e4m3, block scales): each 128-wide K block is accumulated by the MMA
// into its own TMEM partial buffer (a ring of NPART), and the epilogue warps promote it into
// fp32 registers as acc = fma(partial, scale_a[m,kb] * scale_b[n/128,kb], acc), kb ascending --
// the dequantisation fused into the GEMM ("DeepSeek V4的batch invariance：大模型确定性推理的工程
// 基石" (lshu.cn), section 3.2).  The scales are arbitrary fp32 values, which the UE8M0 /
// UE4M3 block-scaled MMA kinds cannot take, so the promotion runs on the CUDA cores.
//
// Failure handling: every mbarrier wait is bounded (see ptx::mbar_wait).  A wait that runs out
// records BI_ERR_DEVICE_TIMEOUT in the status word, raises a CTA-wide abort flag so the other
// roles stop, and the CTA then drains its own TMA loads and MMAs in flight (with the same
// bound), frees its tensor memory and returns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "ptx_sm100.cuh"

namespace bi {

constexpr int kBlockM = 128;        // largest output-tile height = largest MMA M (cta_group::1)
constexpr int kRowBytes = 128;      // K bytes per stage per row: one 128-byte swizzle row
constexpr int kRingBytes = 200 * 1024;   // shared memory for the two operand rings of a CTA pair
// One-CTA kernels: as much of the 227 KB (232 448 bytes) a CTA may hold as the rest leaves: the
// static shared memory (1 KB: the 1024-byte alignment of the dynamic array pads it), the
// alignment slack, the barriers and (grouped) the expert tables.
constexpr int kRingBytes1 = 224 * 1024;
constexpr int kRingBytesGrouped = 214 * 1024;
constexpr int kEpilogueWarps = 4;                       // bf16 (and narrow FP8) epilogue warps
constexpr int kThreads = (2 + kEpilogueWarps) * 32;

// FP8 tiles at least 64 wide split each lane quarter's columns in two halves across 8 epilogue
// warps, so the per-K-chunk promotion keeps up with the MMAs.
template <bool FP8, int BN>
struct Epi {
    static constexpr int kHalves = (FP8 && BN >= 64) ? 2 : 1;
    static constexpr int kWarps = 4 * kHalves;
    static constexpr int kThreads = (2 + kWarps) * 32;
    static constexpr int kCols = BN / kHalves;             // columns per epilogue thread
};

// MMA-issuing threads of a kernel.  A thread's next tcgen05.mma waits on the issue of its previous
// one, which costs ~57 cycles whatever the instruction's shape; several issuing threads overlap
// that cost.  The K chunks of a group are dealt to the issuers round robin (chunk c to issuer
// c % kIssuers), so that every accumulator still receives its instructions from one thread in
// ascending K:
//   - in the dense FP8 kernels with an even number of chunks per group (four issuers when the
//     count is a multiple of 4, else two): each 128-wide K chunk has its own partial-product
//     buffer, and the epilogue promotes the buffers in ascending kb whoever issued them;
//   - in the dense bf16 kernels with CH = 2 or 4 K chains: chain c accumulates the chunks with
//     chunk % CH == c into an accumulator of its own, and the epilogue adds the chains once.  As
//     many issuers as chains when a group's chunk count allows it (kIssuers divides both CH and
//     KC), so each chain belongs to one issuer.
// Grouped kernels keep one issuer: their 128 x 128 instructions are wide enough for one thread
// to keep the tensor pipe fed.  The extra issuers are the warps after the epilogue
// warps.
template <bool FP8, int BN, int NSPLIT, bool GROUPED = false, int KC = 1, int CH = 1>
struct Issue {
    static constexpr int kIssuers = GROUPED ? 1
                                    : FP8   ? (KC % 4 == 0 ? 4 : KC % 2 == 0 ? 2 : 1)
                                    : (CH == 4 && KC % 4 == 0) ? 4
                                    : (CH >= 2 && KC % 2 == 0) ? 2 : 1;
    static constexpr bool kByChunk = kIssuers > 1;
    static constexpr int kSecondWarp = 2 + Epi<FP8, BN>::kWarps;
    static constexpr int kThreads = Epi<FP8, BN>::kThreads + (kIssuers - 1) * 32;
};
constexpr int kMaxExperts = 1024;

// Device status codes (the same values as bi_status_t).
constexpr int kStatusInvalidArg = 1;
constexpr int kStatusTimeout = 6;
constexpr int kStatusBadOffsets = 7;

struct GemmParams {
    int32_t rows;            // M (dense) or total_rows (grouped)
    int32_t n;               // N
    int32_t k;               // K (elements)
    int32_t num_k_blocks;    // ceil(K * elt / 128)
    int32_t num_n_blocks;    // ceil(N / BN)
    int32_t num_m_blocks;    // dense: ceil(M / BM)
    int32_t num_experts;     // grouped: E
    int32_t raster_m;        // dense raster band height in m-blocks
    int32_t a_box_rows;      // rows of A one TMA load brings: BM, or, when the whole dense problem
                             // has fewer rows, exactly its rows (no load reaches past the end of
                             // A; TMA fills such rows slowly).  Chunk c of an A slot then starts
                             // c * a_box_rows * 128 bytes in, inside a 1024-byte swizzle atom when
                             // a_box_rows is not a multiple of 8: tcgen05 applies the 128-byte
                             // swizzle to the absolute shared-memory address, as TMA does when it
                             // writes the box, so the descriptors need no base offset.
    int32_t sa, sb;          // ring depths in groups (2..kMaxSA, sa..kMaxSB)
    uint32_t a_stride;       // bytes between A slots (KC * a_box_rows * 128, rounded up to 1024)
    uint32_t b_offset;       // byte offset of the B ring in the ring region
    int32_t pair_a1;         // CTA pair: 1 if the peer CTA loads A rows (the problem has > 128)
    int32_t prefetch_b;      // dense, resident weights: request the first B groups before the
                             // previous kernel in the stream has completed
    __nv_bfloat16 *c;
    int64_t ldc;
    const float *scale_a;    // FP8: [kb][ld_sa]
    int64_t ld_sa;
    const float *scale_b;    // FP8: [ceil(N/128)][kb_scale]
    int32_t kb_scale;        // ceil(K / 128)
    // e2m1 weights (W4 kernels) only, per output column n: the scale w_scale[n] = 2^-j with j in
    // [1, 12] and the zero point w_zero[n] (a value fp16 represents exactly; null for none);
    // w_rowsum[m] = the sum over k of row m of the dequantised A (read only with w_zero)
    const float *w_scale;
    const float *w_zero;
    const float *w_rowsum;
    const int32_t *offsets;  // grouped: [E+1] (device)
    int *status;             // device status word
    uint64_t timeout_cycles; // limit of every pipeline wait, in SM clock cycles
    uint32_t debug_flags;    // bit 0: skip the first load (fault-injection tests)
    // fixed-split-K research variant only (SPLIT kernels): K chunks [s nkb / S, (s+1) nkb / S)
    // (integer division; S = k_splits <= nkb) of a tile form split s; its fp32 partial goes to
    // ws[s*ws_split_stride + row*ld_ws + col]
    int32_t k_splits;
    float *ws;
    int64_t ld_ws;
    int64_t ws_split_stride;
};

struct TileCoord {
    int32_t m0;       // first output row of the tile
    int32_t row_end;  // one past the last row that belongs to this tile's problem
    int32_t n0;       // first output column
    int32_t b_row0;   // row of the tile's first B row in the (grouped: stacked) B tensor
    int32_t kb0;      // first K chunk of this work unit (0 except for the split-K variant)
    int32_t nkb;      // K chunks of this work unit
    int32_t split;    // split index (split-K variant)
};

// Operand rings.  A pipeline stage ("group") carries KC 128-byte K chunks: KC chunks of A rows
// and KC chunks of BN B rows.  The ring depths and the A slot size are chosen per launch by the
// host (GemmParams::sa, sb, a_stride, b_offset) inside the kernel's ring bytes (ring_bytes_1cta):
// when a dense problem has fewer rows than the tile, an A slot only holds the rows TMA brings,
// which leaves more of shared memory to the B (weight) ring.  The MMA still reads BM rows from
// every A chunk; the rows past the loaded ones lie in the next chunk, slot or the B ring (the host
// keeps them inside the ring) and feed only output rows that are never stored.  The ring geometry
// decides how far ahead loads run, never what the MMA computes.
constexpr int kMaxSA = 8;
constexpr int kMaxSB = 32;

template <bool GROUPED>
__host__ __device__ constexpr int ring_bytes_1cta()
{
    return GROUPED ? kRingBytesGrouped : kRingBytes1;
}
static_assert(1024 + 1024 + kRingBytes1 + 1024 <= 232448, "one-CTA dense ring too large");
static_assert(1024 + 1024 + kRingBytesGrouped + 1024 + 2 * (kMaxExperts + 1) * 4 <= 232448,
              "one-CTA grouped ring too large");

template <int BM, int BN, int KC>
struct Rings {
    static constexpr int kAChunkBytes = BM * kRowBytes;   // one full-height A chunk
    static constexpr int kBChunkBytes = BN * kRowBytes;
    static constexpr int kABytesMax = KC * kAChunkBytes;  // one A group at full height
    static constexpr int kBBytes = KC * kBChunkBytes;     // one B group
};

// Dense tile id -> coordinates.  Tiles are rastered in bands of `raster_m` m-blocks; inside a
// band the m-block varies fastest, so the CTAs running at the same time share B tiles in L2.
__device__ __forceinline__ TileCoord dense_tile(const GemmParams &p, int bm, int bn, int t)
{
    const int band_tiles = p.raster_m * p.num_n_blocks;
    const int band = t / band_tiles;
    const int within = t - band * band_tiles;
    const int m_first = band * p.raster_m;
    int g = p.num_m_blocks - m_first;
    if (g > p.raster_m)
        g = p.raster_m;
    const int m_blk = m_first + within % g;
    const int n_blk = within / g;
    TileCoord tc;
    tc.m0 = m_blk * bm;
    tc.row_end = p.rows;
    tc.n0 = n_blk * bn;
    tc.b_row0 = tc.n0;
    tc.kb0 = 0;
    tc.nkb = p.num_k_blocks;
    tc.split = 0;
    return tc;
}

// Grouped tiles whose segment has at most kShortSegmentRows rows from the tile's first row load
// their A rows as ceil(rows / 8) boxes of 8 rows x KC chunks instead of one full box; the
// shared-memory layout is then [8-row group][chunk][8 rows], which the MMA reads with a stride byte
// offset of KC * 1024.  (More small boxes per stage cost more than the rows they save: TMA issues
// small boxes slowly.)  Returns the number of 8-row boxes, or 0 for a full box.
constexpr int kShortSegmentRows = 16;
__device__ __forceinline__ int short_segment_boxes(const TileCoord &tc, int limit_rows)
{
    const int rows = tc.row_end - tc.m0;
    return rows <= limit_rows ? (rows + 7) >> 3 : 0;
}

// Split-K variant: work unit u is split u % S of dense tile u / S.  The split points are fixed
// by (K, S): split s owns the K chunks [s nkb / S, (s+1) nkb / S), never empty for S <= nkb.
__device__ __forceinline__ TileCoord split_unit(const GemmParams &p, int bm, int bn, int u)
{
    TileCoord tc = dense_tile(p, bm, bn, u / p.k_splits);
    tc.split = u % p.k_splits;
    const int64_t nkb = p.num_k_blocks;
    tc.kb0 = static_cast<int32_t>(tc.split * nkb / p.k_splits);
    tc.nkb = static_cast<int32_t>((tc.split + 1) * nkb / p.k_splits) - tc.kb0;
    return tc;
}

// Grouped tile id -> coordinates.  prefix[e] = number of tiles of experts < e (E+1 entries,
// shared memory).  Inside an expert the m-block varies fastest (the segment's CTAs share B_e).
__device__ __forceinline__ TileCoord grouped_tile(const GemmParams &p, int bm, int bn, int t,
                                                  const int32_t *prefix, const int32_t *offs)
{
    int lo = 0, hi = p.num_experts;   // invariant: prefix[lo] <= t < prefix[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= t)
            lo = mid;
        else
            hi = mid;
    }
    const int e = lo;
    const int local = t - prefix[e];
    const int seg0 = offs[e];
    const int seg1 = offs[e + 1];
    const int mb = (seg1 - seg0 + bm - 1) / bm;
    const int m_blk = local % mb;
    const int n_blk = local / mb;
    TileCoord tc;
    tc.m0 = seg0 + m_blk * bm;
    tc.row_end = seg1;
    tc.n0 = n_blk * bn;
    tc.b_row0 = e * p.n + tc.n0;
    tc.kb0 = 0;
    tc.nkb = p.num_k_blocks;
    tc.split = 0;
    return tc;
}

__device__ __forceinline__ void record_failure(const GemmParams &p, volatile int *abort_flag,
                                               int code)
{
    *abort_flag = 1;
    atomicCAS(p.status, 0, code);
}

// Store 32 consecutive fp32 values of one output row as bf16 (RNE), columns [col0, col0+32),
// masked to col < n.
__device__ __forceinline__ void store_row_chunk32(__nv_bfloat16 *crow, int col0, int n,
                                                  const float (&v)[32])
{
    if (col0 + 32 <= n) {
        uint32_t packed[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
            packed[j] = *reinterpret_cast<uint32_t *>(&h);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(crow + col0);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                                packed[4 * j + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (col0 + j < n)
                crow[col0 + j] = __float2bfloat16_rn(v[j]);
    }
}

// Split-K variant: 32 consecutive fp32 partial sums of one row (row pitch a multiple of 4).
__device__ __forceinline__ void store_row_chunk32_f32(float *wrow, int col0, int n, const float (&v)[32])
{
    if (col0 + 32 <= n) {
        float4 *dst = reinterpret_cast<float4 *>(wrow + col0);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (col0 + j < n)
                wrow[col0 + j] = v[j];
    }
}

// ---------------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------------
//
// BM      : output rows per tile = MMA M (64 or 128).  With M = 64 the accumulator's row i sits
//           in TMEM lane (i % 16) + 32 * (i / 16), so each epilogue warp owns 16 rows.
// FP8: the scales one epilogue thread needs for the KC chunks of group kg -- scale_a of its row
// and (kBlockB) scale_b of each of its 32-column blocks (32 columns never straddle a 128-column
// scale block: the tile origin, the thread's first column and c * 32 are all multiples of 32).
// Chunks past the end of K and columns past N read nothing and get 0.
template <int KC, int kLoads, bool kBlockB = true>
__device__ __forceinline__ void load_group_scales(const GemmParams &p, const float *sa_col, bool row_ok,
                                                  int col_first, int kg, int nkb, float (&sa)[KC],
                                                  float (&sb)[KC][kLoads])
{
#pragma unroll
    for (int cc = 0; cc < KC; ++cc) {
        const int kb = kg * KC + cc;
        const bool kb_ok = kb < nkb;
        sa[cc] = (row_ok && kb_ok) ? __ldg(sa_col + static_cast<int64_t>(kb) * p.ld_sa) : 0.0f;
        if constexpr (kBlockB) {
#pragma unroll
            for (int c = 0; c < kLoads; ++c) {
                const int col = col_first + c * 32;
                sb[cc][c] = (kb_ok && col < p.n)
                                ? __ldg(p.scale_b + static_cast<int64_t>(col >> 7) * p.kb_scale + kb)
                                : 0.0f;
            }
        }
    }
}

// e2m1 weights: the column constants of one epilogue thread's kLoads 32-column blocks, loaded
// once per tile and spread over the warp (lane j holds column col_first + 32 c + j), and the
// zero-point row sum of the thread's row.  A scale that is not 2^-j (j in [1, 12]) or a zero point
// fp16 cannot represent sets BI_ERR_INVALID_ARG in the status word (the columns are computed all
// the same).  Columns past N get scale 1 and zero 0 and are never stored.
template <int kLoads>
struct W4Consts {
    float scale[kLoads];
    float zero[kLoads];
    float rowsum;
};

template <int kLoads>
__device__ __forceinline__ W4Consts<kLoads> w4_load_consts(const GemmParams &p, int row, bool row_ok,
                                                           int col_first, uint32_t lane)
{
    W4Consts<kLoads> w;
    const bool zp = p.w_zero != nullptr;
    bool bad = false;
#pragma unroll
    for (int c = 0; c < kLoads; ++c) {
        const int col = col_first + c * 32 + static_cast<int>(lane);
        const bool ok = col < p.n;
        w.scale[c] = ok ? __ldg(p.w_scale + col) : 1.0f;
        w.zero[c] = (ok && zp) ? __ldg(p.w_zero + col) : 0.0f;
        const uint32_t sbits = __float_as_uint(w.scale[c]);
        const uint32_t e = sbits >> 23;   // sign 0 and a biased exponent in [115, 126]
        bad |= ok && ((sbits & 0x7FFFFFu) != 0u || e < 127u - 12u || e > 127u - 1u);
        bad |= ok && zp && __half2float(__float2half_rn(w.zero[c])) != w.zero[c];
    }
    w.rowsum = (zp && row_ok) ? __ldg(p.w_rowsum + row) : 0.0f;
    if (bad)
        atomicCAS(p.status, 0, kStatusInvalidArg);
    return w;
}

// C = fma(zero[n], rowsum[m], scale[n] * acc), or scale[n] * acc without zero points, for the
// thread's 32 kLoads promoted sums.  Warp-collective (the constants come by shuffle).
template <int kLoads>
__device__ __forceinline__ void w4_finish(const GemmParams &p, const W4Consts<kLoads> &w,
                                          float (&acc)[32 * kLoads])
{
    const bool zp = p.w_zero != nullptr;
#pragma unroll
    for (int c = 0; c < kLoads; ++c) {
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
            const float s = __shfl_sync(0xFFFFFFFFu, w.scale[c], jj);
            const float z = __shfl_sync(0xFFFFFFFFu, w.zero[c], jj);
            const float v = s * acc[c * 32 + jj];
            acc[c * 32 + jj] = zp ? fmaf(z, w.rowsum, v) : v;
        }
    }
}

// e2m1 weights with zero points: rowsum[m] = sum_k a[m][k] in fp32, in an order fixed by K alone
// (so rowsum[m] depends on row m only).  Lane l of a 32-lane group owns the values 4l .. 4l+3 of
// every 128-value K chunk kb: it adds the four e4m3 values of its slice of the chunk in order,
// p = ((v0 + v1) + v2) + v3, and accumulates r_l = fma(p, scale_a[m,kb], r_l) over kb ascending;
// the 32 lane sums are then added in a fixed butterfly.  The two kernels below split the work
// differently and compute the same bits.  K is a multiple of 128.
__device__ __forceinline__ float e4m3x4_sum(uint32_t w)
{
    float t = 0.0f;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        __nv_fp8_e4m3 q;
        q.__x = static_cast<__nv_fp8_storage_t>((w >> (8 * b)) & 0xFFu);
        t += static_cast<float>(q);
    }
    return t;
}

__device__ __forceinline__ float lane_butterfly_sum(float r)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        r += __shfl_xor_sync(0xFFFFFFFFu, r, o);
    return r;
}

// Many rows: one warp per row (8 rows per CTA), 16 chunks in flight per batch; 4 CTAs per SM
// (at most 64 registers a thread) keep the rows of a 4096-row batch in one wave.
__global__ void __launch_bounds__(256, 4) bi_w4_rowsum_warp_kernel(const uint8_t *a, int64_t lda,
                                                                const float *scale_a, int64_t ld_sa,
                                                                int32_t m_rows, int32_t k, float *rowsum)
{
    constexpr int kBatch = 16;
    ptx::grid_dependency_wait();
    if (threadIdx.x == 0)
        ptx::launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= m_rows)
        return;
    const uint8_t *arow = a + row * lda;
    const int nkb = k / 128;
    float r = 0.0f;
    for (int c0 = 0; c0 < nkb; c0 += kBatch) {
        uint32_t wv[kBatch];
        float sv[kBatch];
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            const bool ok = c0 + i < nkb;
            wv[i] = ok ? __ldg(reinterpret_cast<const uint32_t *>(arow + static_cast<int64_t>(c0 + i) * 128) + lane)
                       : 0u;
            sv[i] = ok ? __ldg(scale_a + static_cast<int64_t>(c0 + i) * ld_sa + row) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < kBatch; ++i)
            if (c0 + i < nkb)
                r = fmaf(e4m3x4_sum(wv[i]), sv[i], r);
    }
    r = lane_butterfly_sum(r);
    if (lane == 0)
        rowsum[row] = r;
}

// Few rows: one CTA per row.  Its 8 warps take the chunks in turn and leave each lane's slice sum
// in shared memory; warp 0 then runs the 32 per-lane chains in kb order.
__global__ void __launch_bounds__(256) bi_w4_rowsum_kernel(const uint8_t *a, int64_t lda,
                                                           const float *scale_a, int64_t ld_sa,
                                                           int32_t m_rows, int32_t k, float *rowsum)
{
    constexpr int kSeg = 128;   // chunks per pass through shared memory
    constexpr int kWarps = 8;
    __shared__ float s_p[kSeg][32];
    __shared__ float s_s[kSeg];
    ptx::grid_dependency_wait();
    if (threadIdx.x == 0)
        ptx::launch_dependents();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t row = blockIdx.x;
    if (row >= m_rows)
        return;
    const uint8_t *arow = a + row * lda;
    const int nkb = k / 128;
    float r = 0.0f;
    for (int kb0 = 0; kb0 < nkb; kb0 += kSeg) {
        const int nseg = nkb - kb0 < kSeg ? nkb - kb0 : kSeg;
        for (int c0 = warp; c0 < nseg; c0 += 8 * kWarps) {
            uint32_t wv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = c0 + i * kWarps;
                wv[i] = c < nseg
                            ? __ldg(reinterpret_cast<const uint32_t *>(arow + static_cast<int64_t>(kb0 + c) * 128) + lane)
                            : 0u;
            }
            // lane i < 8 loads the scale of this warp's i-th chunk
            const int ci = c0 + lane * kWarps;
            if (lane < 8 && ci < nseg)
                s_s[ci] = __ldg(scale_a + static_cast<int64_t>(kb0 + ci) * ld_sa + row);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = c0 + i * kWarps;
                if (c < nseg)
                    s_p[c][lane] = e4m3x4_sum(wv[i]);
            }
        }
        __syncthreads();
        if (warp == 0)
            for (int c = 0; c < nseg; ++c)
                r = fmaf(s_p[c][lane], s_s[c], r);
        __syncthreads();
    }
    if (warp == 0) {
        r = lane_butterfly_sum(r);
        if (lane == 0)
            rowsum[row] = r;
    }
}

// BN      : output columns per tile (multiple of 32, <= 256; FP8 <= 128)
// FP8     : e4m3 operands with fp32 block scales (else bf16)
// GROUPED : MoE grouped layout (bf16 only)
// KC      : 128-byte K chunks per pipeline stage (group).  KC > 1 loads a group with one 3-D TMA
//           box per operand (chunk index as the third coordinate), so the producer and MMA
//           threads pay their per-stage handshakes once per KC chunks.  The MMA still walks the
//           chunks of a tile one by one in ascending K: KC changes no bit of the result.
// NSPLIT  : adjacent tiles of a plan, each BN/NSPLIT wide, that one CTA runs in lockstep on one
//           A operand (the wide forms: 2, or 4 for bf16 plans with K chains).  One BM x BN x K
//           instruction covers them at every K step, into adjacent TMEM columns.  tcgen05 forms
//           every element of D from its own row of A and column of B, accumulator and K step,
//           the same way whatever the instruction's N, so each output element gets the bits the
//           plan's (BN/NSPLIT)-wide instruction gives it, with the same K order (FP8: promoted in
//           the same ascending kb); the invariance tests compare the forms bit for bit, also on
//           inputs built to expose a different internal summation (wide exponent spreads,
//           cancellation).
// SPLIT   : the fixed-split-K research variant (bf16 dense only, not the batch-invariant product
//           path): a work unit is one K split of a tile and its epilogue writes fp32 partial
//           sums; bi_splitk_merge_kernel adds the splits in a fixed order.
// CH      : K chains of a dense bf16 tile, 1, 2 or 4.  Chain c accumulates, in ascending K, the
//           128-byte K chunks with chunk % CH == c into an accumulator of its own (each chain
//           issued by one thread), and the epilogue adds the chains once, in a fixed tree:
//           C = bf16_rne(chain0 + chain1) for 2, C = bf16_rne((chain0 + chain1) + (chain2 +
//           chain3)) for 4, leaving out the chains K leaves empty.  The order is fixed by K
//           alone -- the same for every M, row and scheduling form -- and stays inside one CTA:
//           no workspace, no atomics, no cross-CTA reduction.
// W4      : (with FP8, dense) B holds e2m1 weights with one power-of-two scale and one zero point
//           per output column ("DeepSeek V4的batch invariance：大模型确定性推理的工程基石"
//           (lshu.cn), section 4.3: W = W_fp4 * scale + zero, scale in {2^-j : j = 1..12}).  The
//           MMA takes the e2m1 codes as they are (kind::f8f6f4, B format e2m1) and the epilogue
//           promotes each K chunk with scale_a alone, acc = fma(partial, scale_a[m,kb], acc), kb
//           ascending; then C = fma(zero[n], rowsum[m], scale[n] * acc), or scale[n] * acc
//           without zero points.  A power-of-two scale multiplies exactly, so pulling it out of
//           the K sum changes no rounding.
// The ring depths follow from (BM, BN, KC) (see Rings).
template <int BM, int BN, int KC, bool FP8, bool GROUPED, int NSPLIT = 1, bool SPLIT = false,
          bool W4 = false, int CH = 1>
__global__ void __launch_bounds__(Issue<FP8, BN, NSPLIT, GROUPED, KC, CH>::kThreads, 1)
    bi_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_b,
                   const __grid_constant__ CUtensorMap tmap_a8, const GemmParams p)
{
    static_assert(BM == 64 || BM == 128, "MMA M is 64 or 128");
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN must be a multiple of 32 in [32,256]");
    static_assert(!FP8 || BN <= 128, "FP8 keeps BN fp32 accumulators per thread: BN <= 128");
    static_assert(!(FP8 && GROUPED), "grouped FP8 is not built");
    static_assert(KC >= 1 && KC <= 16, "1..16 chunks per group");
    static_assert(NSPLIT == 1 || (NSPLIT == 2 && !GROUPED && BN == (FP8 ? 128 : 64)) ||
                      (NSPLIT == 4 && CH >= 2 && BN == 128),
                  "lockstep tiles: dense bf16 64-wide and FP8 128-wide tiles hold two plan "
                  "tiles; bf16 128-wide tiles with K chains hold four");
    static_assert(!SPLIT || (!FP8 && !GROUPED && NSPLIT == 1), "split-K variant: bf16 dense");
    static_assert(!W4 || (FP8 && !GROUPED && !SPLIT), "e2m1 weights: the dense FP8 kernel");
    static_assert(CH == 1 || ((CH == 2 || CH == 4) && !FP8 && !GROUPED && !SPLIT),
                  "two or four K chains: dense bf16");
    constexpr int kMmaN = BN;                            // MMA instruction N (all NSPLIT tiles)
    using Iss = Issue<FP8, BN, NSPLIT, GROUPED, KC, CH>;
    constexpr int kIssuers = Iss::kIssuers;              // threads issuing MMAs
    using R = Rings<BM, BN, KC>;
    constexpr int kElemsPerRow = FP8 ? 128 : 64;         // K elements per 128-byte row
    constexpr int kMmaK = FP8 ? 32 : 16;                 // K per tcgen05.mma
    constexpr int kMmaPerStage = kElemsPerRow / kMmaK;   // 4
    constexpr int kBytesPerMmaK = kMmaK * (FP8 ? 1 : 2); // 32 bytes
    constexpr int kRowsPerWarp = BM / 4;                 // output rows owned by one epilogue warp
    // TMEM buffers: bf16 double-buffers the accumulator; FP8 rings kNumAcc partial products
    // (one per K chunk, at least two groups' worth so the promotion overlaps the next group).
    constexpr int kNumAcc = FP8 ? ((512 / BN) < 8 ? (512 / BN) : 8) : (2 * CH * BN <= 512 ? 2 : 1);
    constexpr int kAccCols = FP8 ? BN : CH * BN;         // columns of one buffer (bf16: CH chains)
    constexpr int kTmemColsNeeded = kNumAcc * kAccCols;
    constexpr uint32_t kTmemCols = kTmemColsNeeded <= 32    ? 32
                                   : kTmemColsNeeded <= 64  ? 64
                                   : kTmemColsNeeded <= 128 ? 128
                                   : kTmemColsNeeded <= 256 ? 256
                                                            : 512;
    static_assert(kTmemColsNeeded <= 512, "TMEM holds 512 columns");
    static_assert(!FP8 || kNumAcc >= 2 * KC, "FP8 needs two groups of partial buffers");
    // (the host keeps sb > kNumAcc / KC so the FP8 epilogue can track partials on the consumed ring)
    constexpr uint32_t kIdesc = W4    ? ptx::idesc_e4m3_e2m1(BM, kMmaN)
                                : FP8 ? ptx::idesc_e4m3(BM, kMmaN)
                                      : ptx::idesc_bf16(BM, kMmaN);
    // bytes a B group brings: e2m1 values travel packed (two per byte) and land in shared memory
    // in the 16-byte-aligned form, one byte of the tile per value
    constexpr uint32_t kBTxBytes = W4 ? R::kBBytes / 2 : R::kBBytes;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *smem_a = smem;
    uint8_t *smem_b = smem + p.b_offset;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + ring_bytes_1cta<GROUPED>());
    // full[j % sb]: both TMA loads of group j landed (two arrivals: the B load and, issued
    // later, the A load).  consumed[j % sb]: the MMAs of group j completed, which frees B slot
    // j % sb and A slot j % sa (one commit per group).  A group's two arrivals always land in
    // its own phase: slot j % sb is refilled only after group j was consumed.
    uint64_t *full = bars;
    uint64_t *consumed = full + kMaxSB;
    uint64_t *accf_bar = consumed + kMaxSB;    // accumulator (or partial) full
    uint64_t *acce_bar = accf_bar + kNumAcc;   // accumulator (or partial) empty
    uint64_t *drain_bar = acce_bar + kNumAcc;  // one per MMA issuer
    uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(drain_bar + 4);   // up to 4 issuers
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_smem + 1);
    int32_t *grp_prefix = reinterpret_cast<int32_t *>(tmem_base_smem + 4);   // [E+1]
    int32_t *grp_offs = grp_prefix + (GROUPED ? (kMaxExperts + 1) : 0);       // [E+1]

    const uint32_t warp = ptx::warp_id();
    const uint32_t lane = ptx::lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.sb; ++s) {   // only the ring slots this launch uses
            ptx::mbar_init(&full[s], 2);
            ptx::mbar_init(&consumed[s], kIssuers);   // one commit per issuer
        }
        for (int a = 0; a < kNumAcc; ++a) {
            ptx::mbar_init(&accf_bar[a], kIssuers);
            ptx::mbar_init(&acce_bar[a], Epi<FP8, BN>::kWarps * 32);
        }
        for (int i = 0; i < kIssuers; ++i)
            ptx::mbar_init(&drain_bar[i], 1);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
        ptx::prefetch_tmap(&tmap_a);
        ptx::prefetch_tmap(&tmap_b);
        if (GROUPED)
            ptx::prefetch_tmap(&tmap_a8);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_base_smem, kTmemCols);
        ptx::tmem_relinquish_alloc_permit();
    }

    const int nkb = p.num_k_blocks;              // 128-byte K chunks per tile
    const int nkg = (nkb + KC - 1) / KC;         // groups per tile
    const uint32_t a_chunk_pitch = static_cast<uint32_t>(p.a_box_rows) * kRowBytes;
    int num_tiles = 0;                           // set below (grouped: from the offsets)
    auto tile_at = [&](int t) -> TileCoord {
        if constexpr (GROUPED)
            return grouped_tile(p, BM, BN, t, grp_prefix, grp_offs);
        else if constexpr (SPLIT)
            return split_unit(p, BM, BN, t);
        else
            return dense_tile(p, BM, BN, t);
    };
    // groups of a work unit (a tile, or one K split of a tile)
    auto groups_of = [&](const TileCoord &tc) -> int {
        if constexpr (SPLIT)
            return (tc.nkb + KC - 1) / KC;
        else
            return nkg;
    };
    const int tile_units = SPLIT ? p.k_splits : 1;

    // TMA producer state (used by thread 0 only).  Two cursors walk this CTA's (tile, group)
    // sequence: the B loads run `lag` = sb - sa groups ahead of the A loads.
    struct Cursor {
        int t, kg;
        bool valid;
        TileCoord tc;
    };
    Cursor cb{}, ca{};
    int jb = 0, ja = 0;                 // groups issued so far
    int bs = 0, as = 0, cs = 0;         // B slot of jb, A slot of ja, consumed slot of ja - sa
    int fs = 0;                         // full-ring slot of group ja
    uint32_t bph = 0, cph = 0;
    bool skipped_b0 = false;
    const uint64_t pol = ptx::policy_evict_normal();
    auto advance = [&](Cursor &c) {
        if (++c.kg == groups_of(c.tc)) {
            c.kg = 0;
            c.t += gridDim.x;
            c.valid = c.t < num_tiles;
            if (c.valid)
                c.tc = tile_at(c.t);
        }
    };
    auto first_cursor = [&]() {
        Cursor c{static_cast<int>(blockIdx.x), 0, static_cast<int>(blockIdx.x) < num_tiles, {}};
        if (c.valid)
            c.tc = tile_at(c.t);
        return c;
    };
    // load group kg of a work unit whose first K chunk is kb0
    auto load = [&](void *dst, const CUtensorMap *map, uint64_t *bar, int kb0, int kg, int row) {
        if constexpr (KC == 1)
            ptx::tma_load_2d(dst, map, bar, (kb0 + kg) * kElemsPerRow, row, pol);
        else
            ptx::tma_load_3d(dst, map, bar, 0, row, kb0 + kg * KC, pol);
    };
    // B group jb into slot bs; its slot is free (the consumed wait, if any, is done)
    auto issue_b = [&]() {
        if (jb == 0 && (p.debug_flags & 1u)) {
            skipped_b0 = true;      // fault injection: this B group is never filled
        } else {
            ptx::mbar_arrive_expect_tx(&full[bs], kBTxBytes);
            load(smem_b + bs * R::kBBytes, &tmap_b, &full[bs], cb.tc.kb0, cb.kg, cb.tc.b_row0);
        }
        advance(cb);
        ++jb;
        if (++bs == p.sb) {
            bs = 0;
            bph ^= 1u;
        }
    };
    bool b_started = false;
    if constexpr (!GROUPED) {
        // Resident weights: B is not written by the previous kernel in the stream, so the first
        // sb groups of B (their slots are free in a fresh ring) are requested before that
        // kernel has completed.
        if (threadIdx.x == 0 && p.prefetch_b) {
            num_tiles = p.num_m_blocks * p.num_n_blocks * tile_units;
            cb = first_cursor();
            for (int i = 0; i < p.sb && cb.valid; ++i)
                issue_b();
            b_started = true;
        }
    }

    // Everything above touches only this CTA's shared and tensor memory, the kernel parameters
    // and (resident weights only) B, so it overlaps the tail of the previous kernel in the
    // stream when this one was launched as its programmatic dependent.  No thread reads A, the
    // scales or the offsets, or writes anything to global memory, before the previous grid has
    // completed.
    ptx::grid_dependency_wait();
    if (threadIdx.x == 0)
        ptx::launch_dependents();

    // Grouped: read and validate the expert offsets, build the tile prefix sum.
    __shared__ int32_t s_num_tiles;
    if constexpr (GROUPED) {
        __shared__ int s_bad;
        if (threadIdx.x == 0)
            s_bad = 0;
        __syncthreads();
        const int E = p.num_experts;
        for (int e = threadIdx.x; e <= E; e += blockDim.x)
            grp_offs[e] = p.offsets[e];
        __syncthreads();
        for (int e = threadIdx.x; e < E; e += blockDim.x)
            if (grp_offs[e + 1] < grp_offs[e])
                s_bad = 1;
        if (threadIdx.x == 0 && (grp_offs[0] != 0 || grp_offs[E] != p.rows))
            s_bad = 1;
        __syncthreads();
        if (threadIdx.x == 0) {
            int32_t acc = 0;
            if (!s_bad) {
                for (int e = 0; e < E; ++e) {
                    grp_prefix[e] = acc;
                    const int mb = (grp_offs[e + 1] - grp_offs[e] + BM - 1) / BM;
                    acc += mb * p.num_n_blocks;
                }
            } else if (blockIdx.x == 0) {
                atomicCAS(p.status, 0, kStatusBadOffsets);
            }
            grp_prefix[E] = acc;
            s_num_tiles = acc;
        }
    } else {
        if (threadIdx.x == 0)
            s_num_tiles = p.num_m_blocks * p.num_n_blocks * tile_units;
    }

    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_base_smem;
    num_tiles = s_num_tiles;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            if (!b_started)
                cb = first_cursor();
            ca = first_cursor();
            const int SA = p.sa, SB = p.sb, lag = SB - SA;   // B groups lead A groups by lag
            bool ok = true;
            while (ok && (cb.valid || ca.valid)) {
                if (ca.valid && (ja + lag < jb || !cb.valid)) {
                    // slot `as` is free once group ja - SA was consumed.  That group's consumed
                    // barrier cannot have moved on to group ja - SA + SB yet: that one needs A
                    // group ja + lag, which is not issued.
                    if (ja >= SA) {
                        if (!ptx::mbar_wait(&consumed[cs], cph, p.timeout_cycles, abort_flag)) {
                            record_failure(p, abort_flag, kStatusTimeout);
                            ok = false;
                            break;
                        }
                        if (++cs == SB) {
                            cs = 0;
                            cph ^= 1u;
                        }
                    }
                    int nsub = 0;
                    if constexpr (GROUPED)
                        nsub = short_segment_boxes(ca.tc, kShortSegmentRows);
                    if (nsub == 0) {
                        ptx::mbar_arrive_expect_tx(&full[fs], KC * a_chunk_pitch);
                        load(smem_a + as * p.a_stride, &tmap_a, &full[fs], ca.tc.kb0, ca.kg, ca.tc.m0);
                    } else {
                        // a short segment: its rows as 8-row boxes of all KC chunks
                        ptx::mbar_arrive_expect_tx(&full[fs], static_cast<uint32_t>(nsub) * KC * 1024u);
                        for (int i = 0; i < nsub; ++i)
                            load(smem_a + as * p.a_stride + i * KC * 1024, &tmap_a8, &full[fs],
                                 ca.tc.kb0, ca.kg, ca.tc.m0 + 8 * i);
                    }
                    advance(ca);
                    ++ja;
                    if (++as == SA)
                        as = 0;
                    if (++fs == SB)
                        fs = 0;
                    continue;
                }
                // A is `lag` groups behind B (or done): the next B group.  Slot bs is free once
                // group jb - SB was consumed, whose A load was issued above.
                if (!ptx::mbar_wait(&consumed[bs], bph ^ 1u, p.timeout_cycles, abort_flag)) {
                    record_failure(p, abort_flag, kStatusTimeout);
                    ok = false;
                    break;
                }
                issue_b();
            }
            // Drain: every load this thread issued must have landed before the CTA exits (on
            // the normal path they all have: the MMA warp consumed them).  Only the last SB
            // groups can still be in flight.  A group whose A load was never issued (the loop
            // stopped early) cannot complete its phase: its B bytes are waited for alone by
            // letting this thread stand in for the missing A arrival.
            for (int i = jb > SB ? jb - SB : 0; i < jb; ++i) {
                if (i == 0 && skipped_b0)
                    continue;
                if (i >= ja)
                    ptx::mbar_arrive(&full[i % SB]);
                ptx::mbar_wait(&full[i % SB], static_cast<uint32_t>(i / SB) & 1u, p.timeout_cycles,
                               nullptr);
            }
        }
    } else if (warp == 1 || (kIssuers > 1 && warp >= Iss::kSecondWarp &&
                             warp < Iss::kSecondWarp + kIssuers - 1)) {
        // ------------------------------------------------------------------ MMA issuers
        // Issuer `iss` issues the MMAs of the K chunks c with c % kIssuers == iss, each
        // accumulator's instructions in ascending K.  All issuers wait on the same barriers, and
        // each commits every group (the consumed and accumulator-full barriers count one commit
        // per issuer), so a slot or an accumulator is handed on when all are done.
        const int iss = warp == 1 ? 0 : 1 + static_cast<int>(warp) - Iss::kSecondWarp;
        const int chunk_iss = Iss::kByChunk ? iss : 0;
        if (lane == 0) {
            const int SA = p.sa, SB = p.sb;
            int sa = 0, sb = 0;      // ring slots of the next group
            uint32_t pb = 0;         // phase of full[sb] / consumed[sb]
            // Shared-memory descriptors are linear in the address (start address >> 4 in the low
            // bits), so every slot / chunk / K-step descriptor is a base plus an offset (a chunk
            // of fewer than 8 rows' pitch starts inside a swizzle atom: see a_box_rows).
            const uint64_t a_desc0 = ptx::sw128_kmajor_desc(ptx::smem_u32(smem_a));
            const uint64_t b_desc0 = ptx::sw128_kmajor_desc(ptx::smem_u32(smem_b));
            // A of a short grouped segment: 8-row groups KC * 1024 bytes apart, chunks 1024 apart
            const uint64_t a_desc0_short = ptx::sw128_kmajor_desc(ptx::smem_u32(smem_a), KC * 1024u);
            uint32_t acc_iter = 0;   // bf16: tiles done; FP8: K chunks done
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                uint64_t a_base = a_desc0;
                uint32_t a_cp = a_chunk_pitch;   // bytes between the K chunks of an A slot
                if constexpr (GROUPED) {
                    if (short_segment_boxes(tile_at(t), kShortSegmentRows) != 0) {
                        a_base = a_desc0_short;
                        a_cp = 1024u;
                    }
                }
                uint32_t d_tmem = 0;
                if (!FP8) {
                    const uint32_t a = acc_iter % kNumAcc;
                    const uint32_t par = (acc_iter / kNumAcc) & 1u;
                    if (!ptx::mbar_wait(&acce_bar[a], par ^ 1u, p.timeout_cycles, abort_flag)) {
                        record_failure(p, abort_flag, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after_sync();
                    d_tmem = tmem_base + a * kAccCols;
                }
                // chunks and groups of this work unit (the whole K of a tile, or one K split)
                int unit_nkb = nkb, unit_nkg = nkg;
                if constexpr (SPLIT) {
                    const TileCoord tu = tile_at(t);
                    unit_nkb = tu.nkb;
                    unit_nkg = groups_of(tu);
                }
                for (int kg = 0; kg < unit_nkg; ++kg) {
                    if (!ptx::mbar_wait(&full[sb], pb, p.timeout_cycles, abort_flag)) {
                        record_failure(p, abort_flag, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after_sync();
                    const uint64_t a_slot = a_base + ((sa * p.a_stride) >> 4);
                    const uint64_t b_slot = b_desc0 + ((sb * R::kBBytes) >> 4);
                    const int nc = unit_nkb - kg * KC;   // chunks in this group: KC, except at a unit's end
                    if constexpr (FP8) {
                        // Each K chunk's partial product goes to its own TMEM buffer.  Every
                        // epilogue thread hands the buffers back in chunk order, so the buffer of
                        // the group's last chunk being free means the others are free as well:
                        // one wait per group.
                        const uint32_t last = acc_iter + static_cast<uint32_t>((nc < KC ? nc : KC) - 1);
                        if (!ptx::mbar_wait(&acce_bar[last % kNumAcc], ((last / kNumAcc) & 1u) ^ 1u,
                                            p.timeout_cycles, abort_flag)) {
                            record_failure(p, abort_flag, kStatusTimeout);
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after_sync();
                    }
                    // the MMAs of chunk c of this group (K chunk number `chunk` of the tile)
                    auto issue_chunk = [&](int c, int chunk) -> bool {
                        uint32_t d = d_tmem;
                        if constexpr (FP8)   // chunk c of the group has partial buffer acc_iter + c
                            d = tmem_base + ((acc_iter + static_cast<uint32_t>(c)) % kNumAcc) * BN;
                        else if constexpr (CH > 1)   // the chain of the chunk: chunk % CH
                            d = d_tmem + static_cast<uint32_t>(chunk % CH) * BN;
                        const uint64_t a_desc = a_slot + ((c * a_cp) >> 4);
                        const uint64_t b_desc = b_slot + ((c * R::kBChunkBytes) >> 4);
#pragma unroll
                        for (int q = 0; q < kMmaPerStage; ++q) {
                            const uint64_t step = static_cast<uint64_t>((q * kBytesPerMmaK) >> 4);
                            // bf16: accumulate across the whole K of the tile (of the chunk's
                            // chain); FP8: one K chunk
                            const uint32_t accumulate = (q > 0) ? 1u : (FP8 ? 0u : (chunk >= CH ? 1u : 0u));
                            // all BN columns (every lockstep tile) in one instruction
                            if constexpr (FP8)
                                ptx::mma_e4m3_ss(d, a_desc + step, b_desc + step, kIdesc, accumulate);
                            else
                                ptx::mma_bf16_ss(d, a_desc + step, b_desc + step, kIdesc, accumulate);
                        }
                        return true;
                    };
                    // A full group issues its KC chunks as straight-line code: control flow
                    // between consecutive tcgen05.mma instructions slows their issue.  Only the
                    // last group of a tile can hold fewer chunks.
                    if (nc >= KC) {
                        if constexpr (Iss::kByChunk) {
#pragma unroll
                            for (int j = 0; j < KC / kIssuers; ++j)
                                issue_chunk(kIssuers * j + chunk_iss, kg * KC + kIssuers * j + chunk_iss);
                        } else {
#pragma unroll
                            for (int c = 0; c < KC; ++c)
                                issue_chunk(c, kg * KC + c);
                        }
                    } else {
#pragma unroll 1
                        for (int c = chunk_iss; c < nc; c += kIssuers)
                            issue_chunk(c, kg * KC + c);
                    }
                    if constexpr (FP8)
                        acc_iter += static_cast<uint32_t>(nc < KC ? nc : KC);
                    // one commit per group frees both smem slots and, for FP8, marks the group's
                    // partial products ready for the epilogue
                    ptx::mma_commit(&consumed[sb]);
                    if (++sa == SA)
                        sa = 0;
                    if (++sb == SB) {
                        sb = 0;
                        pb ^= 1u;
                    }
                }
                if (!ok)
                    break;
                if (!FP8) {
                    ptx::mma_commit(&accf_bar[acc_iter % kNumAcc]);   // tile accumulator ready
                    ++acc_iter;
                }
            }
            // Drain: wait for every MMA this thread issued before tensor memory is freed.
            ptx::mma_commit(&drain_bar[iss]);
            ptx::mbar_wait(&drain_bar[iss], 0, p.timeout_cycles, nullptr);
        }
    } else {
        // ------------------------------------------------------------------ epilogue warps
        const uint32_t q = warp & 3u;                 // TMEM lane quarter of this warp
        const uint32_t half = (warp - 2) / 4;         // FP8 column half (0 with 4 epilogue warps)
        const bool lane_holds_row = BM == 128 || lane < 16;
        const uint32_t row_in_tile = q * kRowsPerWarp + (BM == 128 ? lane : (lane & 15u));
        const uint32_t lane_addr = (q * 32u) << 16;
        uint32_t acc_iter = 0;   // bf16: tiles; FP8: K chunks
        int gs = 0;              // FP8: consumed-ring slot of the next group, and its phase
        uint32_t gph = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            const TileCoord tc = tile_at(t);
            const int row = tc.m0 + static_cast<int>(row_in_tile);
            const bool row_ok = lane_holds_row && row < tc.row_end;
            __nv_bfloat16 *crow = p.c + static_cast<int64_t>(row) * p.ldc;
            if constexpr (!FP8) {
                const uint32_t a = acc_iter % kNumAcc;
                const uint32_t par = (acc_iter / kNumAcc) & 1u;
                if (!ptx::mbar_wait(&accf_bar[a], par, p.timeout_cycles, abort_flag)) {
                    record_failure(p, abort_flag, kStatusTimeout);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32], r1[32];
                    const uint32_t col = tmem_base + lane_addr + a * kAccCols + c * 32;
                    float v[32];
                    ptx::tmem_ld_32x32b_x32(col, r);
                    if constexpr (CH >= 2)
                        ptx::tmem_ld_32x32b_x32(col + BN, r1);
                    ptx::tmem_wait_ld(r);
                    if constexpr (CH >= 2)
                        ptx::tmem_wait_ld(r1);
                    if constexpr (CH >= 2) {
                        // chain 0 + chain 1 (one chunk in K: chain 0 alone)
                        const bool two = nkb > 1;
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                            v[jj] = two ? __uint_as_float(r[jj]) + __uint_as_float(r1[jj])
                                        : __uint_as_float(r[jj]);
                    } else {
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                            v[jj] = __uint_as_float(r[jj]);
                    }
                    if constexpr (CH == 4) {
                        // C = (chain 0 + chain 1) + (chain 2 + chain 3), in this order; the
                        // chains that K leaves empty (fewer than four chunks) are left out
                        if (nkb > 2) {
                            ptx::tmem_ld_32x32b_x32(col + 2 * BN, r);
                            ptx::tmem_ld_32x32b_x32(col + 3 * BN, r1);
                            ptx::tmem_wait_ld(r);
                            ptx::tmem_wait_ld(r1);
                            const bool four = nkb > 3;
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj)
                                v[jj] += four ? __uint_as_float(r[jj]) + __uint_as_float(r1[jj])
                                              : __uint_as_float(r[jj]);
                        }
                    }
                    if (c == BN / 32 - 1) {
                        ptx::tc_fence_before_sync();
                        ptx::mbar_arrive(&acce_bar[a]);   // accumulator free for the next tile
                    }
                    if (row_ok) {
                        if constexpr (SPLIT)
                            store_row_chunk32_f32(p.ws + tc.split * p.ws_split_stride +
                                                      static_cast<int64_t>(row) * p.ld_ws,
                                                  tc.n0 + c * 32, p.n, v);
                        else
                            store_row_chunk32(crow, tc.n0 + c * 32, p.n, v);
                    }
                }
                ++acc_iter;
            } else {
                // this thread promotes columns [col0, col0 + kCols) of its row
                constexpr int kCols = Epi<FP8, BN>::kCols;
                constexpr int kLoads = kCols / 32;
                const int col0 = static_cast<int>(half) * kCols;
                float acc[kCols];
#pragma unroll
                for (int jj = 0; jj < kCols; ++jj)
                    acc[jj] = 0.0f;
                const float *sa_col = p.scale_a + (row_ok ? row : 0);
                // the scales of group kg + 1 are loaded while group kg is promoted, so their
                // global-memory latency stays off the per-chunk chain
                float sa_g[KC], sb_g[KC][kLoads];
                load_group_scales<KC, kLoads, !W4>(p, sa_col, row_ok, tc.n0 + col0, 0, nkb, sa_g, sb_g);
                // e2m1 weights: this tile's column constants, loaded before the K loop
                W4Consts<kLoads> w4c;
                if constexpr (W4)
                    w4c = w4_load_consts<kLoads>(p, row, row_ok, tc.n0 + col0, lane);
                for (int kg = 0; kg < nkg && ok; ++kg) {
                    float sa_n[KC], sb_n[KC][kLoads];
                    load_group_scales<KC, kLoads, !W4>(p, sa_col, row_ok, tc.n0 + col0, kg + 1, nkb, sa_n, sb_n);
                    // the group's partials are ready when its consumed barrier completes; the MMA
                    // warp runs at most kNumAcc chunks (< sb groups) ahead, so the barrier cannot
                    // have moved on to the group sb later
                    if (!ptx::mbar_wait(&consumed[gs], gph, p.timeout_cycles, abort_flag)) {
                        record_failure(p, abort_flag, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    if (++gs == p.sb) {
                        gs = 0;
                        gph ^= 1u;
                    }
                    ptx::tc_fence_after_sync();
#pragma unroll
                    for (int cc = 0; cc < KC; ++cc) {
                        const int kb = kg * KC + cc;
                        if (kb >= nkb)
                            break;
                        const uint32_t part = acc_iter % kNumAcc;
                        // issue every TMEM load of this chunk, then wait once
                        uint32_t r[kLoads][32];
#pragma unroll
                        for (int c = 0; c < kLoads; ++c)
                            ptx::tmem_ld_32x32b_x32(tmem_base + lane_addr + part * BN + col0 + c * 32, r[c]);
#pragma unroll
                        for (int c = 0; c < kLoads; ++c)
                            ptx::tmem_wait_ld(r[c]);
                        ptx::tc_fence_before_sync();
                        ptx::mbar_arrive(&acce_bar[part]);   // the partial buffer is free again
#pragma unroll
                        for (int c = 0; c < kLoads; ++c) {
                            const float s = W4 ? sa_g[cc] : sa_g[cc] * sb_g[cc][c];
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj)
                                acc[c * 32 + jj] = fmaf(__uint_as_float(r[c][jj]), s, acc[c * 32 + jj]);
                        }
                        ++acc_iter;
                    }
#pragma unroll
                    for (int cc = 0; cc < KC; ++cc) {
                        sa_g[cc] = sa_n[cc];
#pragma unroll
                        for (int c = 0; c < kLoads; ++c)
                            sb_g[cc][c] = sb_n[cc][c];
                    }
                }
                if (!ok)
                    break;
                if constexpr (W4)
                    w4_finish<kLoads>(p, w4c, acc);
                if (row_ok) {
#pragma unroll
                    for (int c = 0; c < kLoads; ++c) {
                        float v[32];
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                            v[jj] = acc[c * 32 + jj];
                        store_row_chunk32(crow, tc.n0 + col0 + c * 32, p.n, v);
                    }
                }
            }
        }
    }

    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// C = 0 for K == 0 (an empty contraction).
__global__ void bi_zero_kernel(__nv_bfloat16 *c, int64_t ldc, int64_t m, int64_t n)
{
    const int64_t total = m * n;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / n;
        const int64_t col = i - r * n;
        c[r * ldc + col] = __float2bfloat16_rn(0.0f);
    }
}

// Split-K variant: C = bf16_rne(sum of the S fp32 partials), added in a fixed pairwise tree,
// ((p0 + p1) + (p2 + p3)) + ..., the same for every M.  S is 2, 4 or 8.
__global__ void bi_splitk_merge_kernel(const float *ws, int64_t ld_ws, int64_t split_stride, int S,
                                       __nv_bfloat16 *c, int64_t ldc, int64_t m, int64_t n)
{
    const int64_t total = m * n;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / n;
        const int64_t col = i - r * n;
        float v[8];
#pragma unroll
        for (int s = 0; s < 8; ++s)
            v[s] = s < S ? ws[s * split_stride + r * ld_ws + col] : 0.0f;
#pragma unroll
        for (int w = 1; w < 8; w *= 2)
#pragma unroll
            for (int s = 0; s + w < 8; s += 2 * w)
                if (s + w < S)
                    v[s] = v[s] + v[s + w];
        c[r * ldc + col] = __float2bfloat16_rn(v[0]);
    }
}

template <int BM, int BN, int KC, bool FP8, bool GROUPED, int NSPLIT = 1, bool SPLIT = false,
          bool W4 = false, int CH = 1>
constexpr int smem_bytes_for()
{
    return 1024 + ring_bytes_1cta<GROUPED>() + 1024 + (GROUPED ? 2 * (kMaxExperts + 1) * 4 : 0);
}

} // namespace bi
