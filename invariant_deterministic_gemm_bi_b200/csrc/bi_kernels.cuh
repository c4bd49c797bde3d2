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
// are zero-filled by TMA and never stored.  When the whole problem has fewer than 128 rows,
// TMA brings only the first roundup(M, 8) rows of the A tile; the MMA still runs on all 128
// rows, and the rows never loaded feed only output rows that are never stored (every output
// element depends on its own A row alone).  The CTA <-> tile mapping does depend on M, which is
// harmless: it decides where a tile is computed, not how.
//
// Roles inside a CTA (6 warps = 192 threads):
//   warp 0, lane 0 : TMA producer -- A tile [128 x 128 B] and B tile [BN x 128 B] per stage
//                    into a STAGES-deep shared-memory ring (128-byte swizzle)
//   warp 1         : allocates tensor memory; lane 0 issues tcgen05.mma and commits
//   warps 2..5     : epilogue -- tcgen05.ld from TMEM, fp32 -> bf16 (RNE), masked stores
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

#include "ptx_sm100.cuh"

namespace bi {

constexpr int kBlockM = 128;        // output rows per tile = MMA M (cta_group::1)
constexpr int kRowBytes = 128;      // K bytes per stage per row: one 128-byte swizzle row
constexpr int kEpilogueWarps = 4;
constexpr int kThreads = (2 + kEpilogueWarps) * 32;
constexpr int kMaxExperts = 1024;

// Device status codes (the same values as bi_status_t).
constexpr int kStatusTimeout = 6;
constexpr int kStatusBadOffsets = 7;

struct GemmParams {
    int32_t rows;            // M (dense) or total_rows (grouped)
    int32_t n;               // N
    int32_t k;               // K (elements)
    int32_t num_k_blocks;    // ceil(K * elt / 128)
    int32_t num_n_blocks;    // ceil(N / BN)
    int32_t num_m_blocks;    // dense: ceil(M / 128)
    int32_t num_experts;     // grouped: E
    int32_t raster_m;        // dense raster band height in m-blocks
    int32_t a_box_rows;      // rows of A one TMA load brings (<= 128, a multiple of 8)
    __nv_bfloat16 *c;
    int64_t ldc;
    const float *scale_a;    // FP8: [kb][ld_sa]
    int64_t ld_sa;
    const float *scale_b;    // FP8: [ceil(N/128)][kb_scale]
    int32_t kb_scale;        // ceil(K / 128)
    const int32_t *offsets;  // grouped: [E+1] (device)
    int *status;             // device status word
    uint64_t timeout_ns;
    uint32_t debug_flags;    // bit 0: skip the first load (fault-injection tests)
};

struct TileCoord {
    int32_t m0;       // first output row of the tile
    int32_t row_end;  // one past the last row that belongs to this tile's problem
    int32_t n0;       // first output column
    int32_t b_row0;   // row of the tile's first B row in the (grouped: stacked) B tensor
};

template <int BN>
struct SmemLayout {
    static constexpr int kABytes = kBlockM * kRowBytes;
    static constexpr int kBBytes = BN * kRowBytes;
    static constexpr int kStageBytes = kABytes + kBBytes;
};

// Dense tile id -> coordinates.  Tiles are rastered in bands of `raster_m` m-blocks; inside a
// band the m-block varies fastest, so the CTAs running at the same time share B tiles in L2.
__device__ __forceinline__ TileCoord dense_tile(const GemmParams &p, int bn, int t)
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
    tc.m0 = m_blk * kBlockM;
    tc.row_end = p.rows;
    tc.n0 = n_blk * bn;
    tc.b_row0 = tc.n0;
    return tc;
}

// Grouped tile id -> coordinates.  prefix[e] = number of tiles of experts < e (E+1 entries,
// shared memory).  Inside an expert the m-block varies fastest (the segment's CTAs share B_e).
__device__ __forceinline__ TileCoord grouped_tile(const GemmParams &p, int bn, int t,
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
    const int mb = (seg1 - seg0 + kBlockM - 1) / kBlockM;
    const int m_blk = local % mb;
    const int n_blk = local / mb;
    TileCoord tc;
    tc.m0 = seg0 + m_blk * kBlockM;
    tc.row_end = seg1;
    tc.n0 = n_blk * bn;
    tc.b_row0 = e * p.n + tc.n0;
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

// ---------------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------------
//
// BN      : output columns per tile = MMA N (multiple of 32, <= 256; FP8 <= 128)
// STAGES  : shared-memory ring depth
// FP8     : e4m3 operands with fp32 block scales (else bf16)
// GROUPED : MoE grouped layout (bf16 only)
template <int BN, int STAGES, bool FP8, bool GROUPED>
__global__ void __launch_bounds__(kThreads, 1)
    bi_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_b, const GemmParams p)
{
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN must be a multiple of 32 in [32,256]");
    static_assert(!FP8 || BN <= 128, "FP8 keeps BN fp32 accumulators per thread: BN <= 128");
    static_assert(!(FP8 && GROUPED), "grouped FP8 is not built");
    using L = SmemLayout<BN>;
    constexpr int kElemsPerRow = FP8 ? 128 : 64;        // K elements per 128-byte row
    constexpr int kMmaK = FP8 ? 32 : 16;                 // K per tcgen05.mma
    constexpr int kMmaPerStage = kElemsPerRow / kMmaK;   // 4
    constexpr int kBytesPerMmaK = kMmaK * (FP8 ? 1 : 2); // 32 bytes
    // TMEM buffers: bf16 double-buffers the accumulator; FP8 rings NPART partial products.
    constexpr int kNumAcc = FP8 ? ((512 / BN) < 4 ? (512 / BN) : 4) : 2;
    constexpr int kTmemColsNeeded = kNumAcc * BN;
    constexpr uint32_t kTmemCols = kTmemColsNeeded <= 32    ? 32
                                   : kTmemColsNeeded <= 64  ? 64
                                   : kTmemColsNeeded <= 128 ? 128
                                   : kTmemColsNeeded <= 256 ? 256
                                                            : 512;
    static_assert(kTmemColsNeeded <= 512, "TMEM holds 512 columns");
    constexpr uint32_t kIdesc = FP8 ? ptx::idesc_e4m3(kBlockM, BN) : ptx::idesc_bf16(kBlockM, BN);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *smem_a = smem;
    uint8_t *smem_b = smem + STAGES * L::kABytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * L::kStageBytes);
    uint64_t *full_bar = bars;
    uint64_t *empty_bar = bars + STAGES;
    uint64_t *accf_bar = bars + 2 * STAGES;            // accumulator (or partial) full
    uint64_t *acce_bar = bars + 2 * STAGES + kNumAcc;  // accumulator (or partial) empty
    uint64_t *drain_bar = bars + 2 * STAGES + 2 * kNumAcc;
    uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_smem + 1);
    int32_t *grp_prefix = reinterpret_cast<int32_t *>(tmem_base_smem + 4);   // [E+1]
    int32_t *grp_offs = grp_prefix + (GROUPED ? (kMaxExperts + 1) : 0);       // [E+1]

    const uint32_t warp = ptx::warp_id();
    const uint32_t lane = ptx::lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&full_bar[s], 1);
            ptx::mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < kNumAcc; ++a) {
            ptx::mbar_init(&accf_bar[a], 1);
            ptx::mbar_init(&acce_bar[a], kEpilogueWarps * 32);
        }
        ptx::mbar_init(drain_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
        ptx::prefetch_tmap(&tmap_a);
        ptx::prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_base_smem, kTmemCols);
        ptx::tmem_relinquish_alloc_permit();
    }

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
                    const int mb = (grp_offs[e + 1] - grp_offs[e] + kBlockM - 1) / kBlockM;
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
            s_num_tiles = p.num_m_blocks * p.num_n_blocks;
    }

    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_base_smem;
    const int num_tiles = s_num_tiles;

    auto tile_at = [&](int t) -> TileCoord {
        if constexpr (GROUPED)
            return grouped_tile(p, BN, t, grp_prefix, grp_offs);
        else
            return dense_tile(p, BN, t);
    };

    const int nkb = p.num_k_blocks;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_a = ptx::policy_evict_normal();
            const uint64_t pol_b = ptx::policy_evict_normal();
            uint32_t issued = 0, issued_phase = 0;            // per-stage: a load in flight / its parity
            int stage = 0;
            uint32_t phase = 0;
            bool skip_next = (p.debug_flags & 1u) != 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                const TileCoord tc = tile_at(t);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!ptx::mbar_wait(&empty_bar[stage], phase ^ 1u, p.timeout_ns, abort_flag)) {
                        record_failure(p, abort_flag, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    if (skip_next) {
                        skip_next = false;   // fault injection: this stage is never filled
                    } else {
                        ptx::mbar_arrive_expect_tx(&full_bar[stage],
                                                   (p.a_box_rows + BN) * kRowBytes);
                        ptx::tma_load_2d(smem_a + stage * L::kABytes, &tmap_a, &full_bar[stage],
                                         kb * kElemsPerRow, tc.m0, pol_a);
                        ptx::tma_load_2d(smem_b + stage * L::kBBytes, &tmap_b, &full_bar[stage],
                                         kb * kElemsPerRow, tc.b_row0, pol_b);
                        issued |= 1u << stage;
                        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Drain: every load this thread issued must have landed before the CTA exits.
            // (On the normal path they all have: the MMA warp consumed them.)
            for (int s = 0; s < STAGES; ++s)
                if (issued & (1u << s))
                    ptx::mbar_wait(&full_bar[s], (issued_phase >> s) & 1u, p.timeout_ns, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t acc_iter = 0;   // bf16: tiles done; FP8: K blocks done
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                uint32_t d_tmem = 0;
                if (!FP8) {
                    const uint32_t a = acc_iter % kNumAcc;
                    const uint32_t par = (acc_iter / kNumAcc) & 1u;
                    if (!ptx::mbar_wait(&acce_bar[a], par ^ 1u, p.timeout_ns, abort_flag)) {
                        record_failure(p, abort_flag, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after_sync();
                    d_tmem = tmem_base + a * BN;
                }
                for (int kb = 0; kb < nkb; ++kb) {
                    uint32_t part = 0;
                    if (FP8) {
                        part = acc_iter % kNumAcc;
                        const uint32_t par = (acc_iter / kNumAcc) & 1u;
                        if (!ptx::mbar_wait(&acce_bar[part], par ^ 1u, p.timeout_ns, abort_flag)) {
                            record_failure(p, abort_flag, kStatusTimeout);
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after_sync();
                        d_tmem = tmem_base + part * BN;
                    }
                    if (!ptx::mbar_wait(&full_bar[stage], phase, p.timeout_ns, abort_flag)) {
                        record_failure(p, abort_flag, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after_sync();
                    const uint64_t a_desc = ptx::sw128_kmajor_desc(ptx::smem_u32(smem_a + stage * L::kABytes));
                    const uint64_t b_desc = ptx::sw128_kmajor_desc(ptx::smem_u32(smem_b + stage * L::kBBytes));
#pragma unroll
                    for (int j = 0; j < kMmaPerStage; ++j) {
                        const uint64_t step = static_cast<uint64_t>((j * kBytesPerMmaK) >> 4);
                        // bf16: accumulate across the whole K of the tile; FP8: one K block
                        const uint32_t accumulate = FP8 ? (j > 0) : ((kb > 0) || (j > 0));
                        if (FP8)
                            ptx::mma_e4m3_ss(d_tmem, a_desc + step, b_desc + step, kIdesc, accumulate);
                        else
                            ptx::mma_bf16_ss(d_tmem, a_desc + step, b_desc + step, kIdesc, accumulate);
                    }
                    ptx::mma_commit(&empty_bar[stage]);   // frees the smem stage when the MMAs are done
                    if (FP8) {
                        ptx::mma_commit(&accf_bar[part]); // partial product of this K block ready
                        ++acc_iter;
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
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
            ptx::mma_commit(drain_bar);
            ptx::mbar_wait(drain_bar, 0, p.timeout_ns, nullptr);
        }
    } else {
        // ------------------------------------------------------------------ epilogue warps
        const uint32_t q = warp & 3u;                 // TMEM lane quarter of this warp
        const uint32_t row_in_tile = q * 32 + lane;
        const uint32_t lane_addr = (q * 32u) << 16;
        uint32_t acc_iter = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            const TileCoord tc = tile_at(t);
            const int row = tc.m0 + static_cast<int>(row_in_tile);
            const bool row_ok = row < tc.row_end;
            __nv_bfloat16 *crow = p.c + static_cast<int64_t>(row) * p.ldc;
            if constexpr (!FP8) {
                const uint32_t a = acc_iter % kNumAcc;
                const uint32_t par = (acc_iter / kNumAcc) & 1u;
                if (!ptx::mbar_wait(&accf_bar[a], par, p.timeout_ns, abort_flag)) {
                    record_failure(p, abort_flag, kStatusTimeout);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    ptx::tmem_ld_32x32b_x32(tmem_base + lane_addr + a * BN + c * 32, r);
                    ptx::tmem_wait_ld(r);
                    if (c == BN / 32 - 1) {
                        ptx::tc_fence_before_sync();
                        ptx::mbar_arrive(&acce_bar[a]);   // accumulator free for the next tile
                    }
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        v[j] = __uint_as_float(r[j]);
                    if (row_ok)
                        store_row_chunk32(crow, tc.n0 + c * 32, p.n, v);
                }
                ++acc_iter;
            } else {
                float acc[BN];
#pragma unroll
                for (int j = 0; j < BN; ++j)
                    acc[j] = 0.0f;
                const float *sa_col = p.scale_a + (row_ok ? row : 0);
                for (int kb = 0; kb < nkb; ++kb) {
                    const uint32_t part = acc_iter % kNumAcc;
                    const uint32_t par = (acc_iter / kNumAcc) & 1u;
                    const float sa = row_ok ? __ldg(sa_col + static_cast<int64_t>(kb) * p.ld_sa) : 0.0f;
                    if (!ptx::mbar_wait(&accf_bar[part], par, p.timeout_ns, abort_flag)) {
                        record_failure(p, abort_flag, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after_sync();
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c) {
                        uint32_t r[32];
                        ptx::tmem_ld_32x32b_x32(tmem_base + lane_addr + part * BN + c * 32, r);
                        ptx::tmem_wait_ld(r);
                        // 32 columns never straddle a 128-column scale block (n0 and c*32 are
                        // multiples of 32)
                        const int col = tc.n0 + c * 32;
                        const float sb = col < p.n
                                             ? __ldg(p.scale_b + static_cast<int64_t>(col >> 7) * p.kb_scale + kb)
                                             : 0.0f;
                        const float s = sa * sb;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            acc[c * 32 + j] = fmaf(__uint_as_float(r[j]), s, acc[c * 32 + j]);
                    }
                    ptx::tc_fence_before_sync();
                    ptx::mbar_arrive(&acce_bar[part]);
                    ++acc_iter;
                }
                if (!ok)
                    break;
                if (row_ok) {
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c) {
                        float v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            v[j] = acc[c * 32 + j];
                        store_row_chunk32(crow, tc.n0 + c * 32, p.n, v);
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

template <int BN, int STAGES, bool FP8, bool GROUPED>
constexpr int smem_bytes_for()
{
    return 1024 + STAGES * SmemLayout<BN>::kStageBytes + 512 +
           (GROUPED ? 2 * (kMaxExperts + 1) * 4 : 0);
}

} // namespace bi
