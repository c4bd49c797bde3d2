// bi_kernels_pair.cuh -- the GEMM on a CTA pair (tcgen05 cta_group::2) for wide tiles.
//
// A cluster of two CTAs computes a 256 x BN output tile with one MMA stream: CTA r of the pair
// holds rows [128 r, 128 r + 128) of the tile's A rows and rows [r BN/2, (r+1) BN/2) of its B
// rows in its own shared memory; one thread of the leader CTA (rank 0) issues
// tcgen05.mma.cta_group::2 with M = 256, N = BN, and each CTA's tensor memory receives its own
// 128 output rows.  Each SM therefore reads only half of B per MMA, which halves the
// shared-memory traffic per FLOP of a one-CTA 128 x BN tile.
//
// The batch-invariance argument is the one of bi_kernels.cuh: the pair owns the whole K range of
// its tile, the K chunks are walked in ascending order, and the MMA instruction shape, the tile
// and the K order are fixed by the plan from (N, K, dtype).  Which CTA of the pair (and which
// half of the 256 rows) a row lands in depends on M; the arithmetic per row does not.
//
// Barriers (every CTA has the same layout):
//   full[s]      leader only: the four TMA loads of group s (A and B of both CTAs) landed.  The
//                leader arms it with both CTAs' bytes; the peer's loads complete on it remotely.
//   consumed[s]  per CTA: the MMAs of group s completed (the leader commits to both CTAs).
//   accf[a]      per CTA: tile accumulator a is ready (bf16), committed to both CTAs.
//   acce[a]      leader only: both CTAs' epilogues are done with accumulator / partial a
//                (8 arrivals: one per epilogue warp of each CTA).
// No TMA load uses cluster multicast: every CTA loads its own boxes.
#pragma once

#include "bi_kernels.cuh"

namespace bi {

template <int BN, int KC>
struct PairRings {
    static constexpr int kAChunkBytes = 128 * kRowBytes;        // one CTA's 128 A rows
    static constexpr int kBChunkBytes = (BN / 2) * kRowBytes;   // one CTA's half of the B rows
    static constexpr int kABytes = KC * kAChunkBytes;
    static constexpr int kBBytes = KC * kBChunkBytes;
    static constexpr int kStages0 = kRingBytes / (kABytes + kBBytes);
    static constexpr int kStages = kStages0 > kMaxSB ? kMaxSB : kStages0;
    static_assert(kStages >= 2, "pair ring depth");
};

// BN      : output columns per pair tile = MMA N (128 or 256; FP8 128)
// KC      : 128-byte K chunks per pipeline stage (1 or 2)
template <int BN, int KC, bool FP8, bool GROUPED>
__global__ void __launch_bounds__(Epi<FP8, BN>::kThreads, 1)
    bi_gemm_kernel_pair(const __grid_constant__ CUtensorMap tmap_a,
                        const __grid_constant__ CUtensorMap tmap_b,
                        const __grid_constant__ CUtensorMap tmap_a8, const GemmParams p)
{
    static_assert(BN == 128 || BN == 256, "pair tiles are 128 or 256 wide");
    static_assert(!FP8 || BN == 128, "FP8 keeps BN fp32 accumulators per thread");
    static_assert(!(FP8 && GROUPED), "grouped FP8 is not built");
    static_assert(KC == 1 || KC == 2, "1 or 2 chunks per stage");
    using R = PairRings<BN, KC>;
    constexpr int S = R::kStages;
    constexpr int kPairRows = 256;                       // tile height = MMA M
    constexpr int kElemsPerRow = FP8 ? 128 : 64;
    constexpr int kMmaK = FP8 ? 32 : 16;
    constexpr int kMmaPerChunk = kElemsPerRow / kMmaK;   // 4
    constexpr int kBytesPerMmaK = kMmaK * (FP8 ? 1 : 2); // 32
    constexpr int kNumAcc = FP8 ? ((512 / BN) < 8 ? (512 / BN) : 8) : 2;
    constexpr uint32_t kTmemCols = kNumAcc * BN <= 128 ? 128 : kNumAcc * BN <= 256 ? 256 : 512;
    static_assert(kNumAcc * BN <= 512, "TMEM holds 512 columns");
    static_assert(!FP8 || kNumAcc >= 2 * KC, "FP8 needs two groups of partial buffers");
    static_assert(!FP8 || kNumAcc / KC < S, "the FP8 epilogue tracks partials on the consumed ring");
    constexpr uint32_t kIdesc = FP8 ? ptx::idesc_e4m3(kPairRows, BN) : ptx::idesc_bf16(kPairRows, BN);
    constexpr int kEpiWarps = Epi<FP8, BN>::kWarps;
    // Bytes of one group over both CTAs: B halves always, A rows as the launch boxes them (fewer
    // than 128 rows when the whole problem is smaller than a CTA's share; the peer loads no A
    // at all when the problem has at most 128 rows).
    const uint32_t a_chunk_pitch = static_cast<uint32_t>(p.a_box_rows) * kRowBytes;
    // How a tile's A rows are loaded.  Dense: each CTA loads its 128 rows (boxed to the problem's
    // rows when it has fewer), the peer nothing when the problem has at most 128 rows.  Grouped:
    // the segment's rows from the tile's first row decide -- at most kShortSegmentRows come in as 8-row boxes
    // (layout [8-row group][chunk][8 rows]) to the leader, at most 128 as the leader's full box,
    // more as both CTAs' full boxes.
    struct ALoad {
        int nsub;          // 8-row boxes of the leader (0: one full box)
        bool peer;         // the peer CTA loads its 128 rows
        uint32_t bytes;    // A bytes of one group over both CTAs
    };
    auto a_load = [&](const TileCoord &tc) -> ALoad {
        ALoad al{0, p.pair_a1 != 0, 0};
        if constexpr (GROUPED) {
            const int rows = tc.row_end - tc.m0;
            al.nsub = rows <= kShortSegmentRows ? (rows + 7) >> 3 : 0;
            al.peer = rows > 128;
        }
        al.bytes = (al.nsub ? static_cast<uint32_t>(al.nsub) * 1024u : a_chunk_pitch) * KC +
                   (al.peer ? KC * a_chunk_pitch : 0u);
        return al;
    };

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *smem_a = smem;
    uint8_t *smem_b = smem + S * R::kABytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kRingBytes);
    uint64_t *full = bars;
    uint64_t *consumed = full + kMaxSB;
    uint64_t *accf_bar = consumed + kMaxSB;
    uint64_t *acce_bar = accf_bar + 8;
    uint64_t *drain_bar = acce_bar + 8;
    uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_smem + 1);
    int32_t *grp_prefix = reinterpret_cast<int32_t *>(tmem_base_smem + 4);
    int32_t *grp_offs = grp_prefix + (GROUPED ? (kMaxExperts + 1) : 0);

    const uint32_t warp = ptx::warp_id();
    const uint32_t lane = ptx::lane_id();
    const uint32_t rank = ptx::cluster_ctarank();        // 0 = leader, 1 = peer
    const int pair = static_cast<int>(ptx::cluster_id_x());
    const int npairs = static_cast<int>(ptx::num_clusters_x());

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxSB; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&consumed[s], 1);
        }
        for (int a = 0; a < 8; ++a) {
            ptx::mbar_init(&accf_bar[a], 1);
            ptx::mbar_init(&acce_bar[a], 2 * kEpiWarps);
        }
        ptx::mbar_init(drain_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
        ptx::prefetch_tmap(&tmap_a);
        ptx::prefetch_tmap(&tmap_b);
        if constexpr (GROUPED)
            ptx::prefetch_tmap(&tmap_a8);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(tmem_base_smem, kTmemCols);
        ptx::tmem_relinquish_alloc_permit_pair();
    }
    // No global memory is touched before the previous grid in the stream has completed (see
    // bi_gemm_kernel); the set-up above overlaps its tail.
    ptx::grid_dependency_wait();
    if (threadIdx.x == 0)
        ptx::launch_dependents();

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
                    const int mb = (grp_offs[e + 1] - grp_offs[e] + kPairRows - 1) / kPairRows;
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

    // Both CTAs' barriers are initialised and the pair's tensor memory is allocated before any
    // CTA touches the other's shared memory.
    ptx::tc_fence_before_sync();
    __syncwarp();
    ptx::cluster_sync();
    ptx::tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_base_smem;
    const int num_tiles = s_num_tiles;

    auto tile_at = [&](int t) -> TileCoord {
        if constexpr (GROUPED)
            return grouped_tile(p, kPairRows, BN, t, grp_prefix, grp_offs);
        else
            return dense_tile(p, kPairRows, BN, t);
    };

    const int nkb = p.num_k_blocks;
    const int nkg = (nkb + KC - 1) / KC;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer (both)
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_normal();
            const uint32_t full0_leader = ptx::mapa_shared(ptx::smem_u32(&full[0]), 0);
            int s = 0, j = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs) {
                const TileCoord tc = tile_at(t);
                const int a_row = tc.m0 + 128 * static_cast<int>(rank);
                const int b_row = tc.b_row0 + (BN / 2) * static_cast<int>(rank);
                const ALoad al = a_load(tc);
                for (int kg = 0; kg < nkg; ++kg, ++j) {
                    if (!ptx::mbar_wait(&consumed[s], ph ^ 1u, p.timeout_cycles, abort_flag)) {
                        record_failure(p, abort_flag, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    const uint32_t bar = full0_leader + s * 8;
                    if (!(j == 0 && (p.debug_flags & 1u) && rank == 0)) {   // fault injection skips
                        if (rank == 0)                                        // the leader's first group
                            ptx::mbar_arrive_expect_tx(&full[s], 2u * R::kBBytes + al.bytes);
                        const bool load_a = rank == 0 || al.peer;
                        const int nbox = (rank == 0 && al.nsub) ? al.nsub : (load_a ? 1 : 0);
                        const CUtensorMap *amap = (rank == 0 && al.nsub) ? &tmap_a8 : &tmap_a;
                        // 8-row boxes go KC * 1024 bytes apart (each holds all KC chunks)
                        for (int i = 0; i < nbox; ++i) {
                            uint8_t *dst = smem_a + s * R::kABytes + i * KC * 1024;
                            if constexpr (KC == 1)
                                ptx::tma_load_2d_pair(dst, amap, bar, kg * kElemsPerRow, a_row + 8 * i, pol);
                            else
                                ptx::tma_load_3d_pair(dst, amap, bar, 0, a_row + 8 * i, kg * KC, pol);
                        }
                        if constexpr (KC == 1)
                            ptx::tma_load_2d_pair(smem_b + s * R::kBBytes, &tmap_b, bar,
                                                  kg * kElemsPerRow, b_row, pol);
                        else
                            ptx::tma_load_3d_pair(smem_b + s * R::kBBytes, &tmap_b, bar, 0, b_row,
                                                  kg * KC, pol);
                    }
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // Drain (leader): the loads of the last S groups of both CTAs land on its barriers.
            // On the normal path they were all consumed; after a timeout the wait is bounded.
            if (rank == 0) {
                const bool skipped = (p.debug_flags & 1u) != 0;
                for (int i = j > S ? j - S : 0; i < j; ++i)
                    if (!(i == 0 && skipped))
                        ptx::mbar_wait(&full[i % S], static_cast<uint32_t>(i / S) & 1u,
                                       p.timeout_cycles, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && rank == 0) {
            const uint32_t consumed_peer0 = ptx::mapa_shared(ptx::smem_u32(&consumed[0]), 1);
            const uint32_t accf_peer0 = ptx::mapa_shared(ptx::smem_u32(&accf_bar[0]), 1);
            const uint64_t a_desc0 = ptx::sw128_kmajor_desc(ptx::smem_u32(smem_a));
            const uint64_t b_desc0 = ptx::sw128_kmajor_desc(ptx::smem_u32(smem_b));
            int s = 0;
            uint32_t ph = 0;
            uint32_t acc_iter = 0;   // bf16: tiles; FP8: K chunks
            bool ok = true;
            const uint64_t a_desc0_short = ptx::sw128_kmajor_desc(ptx::smem_u32(smem_a), KC * 1024u);
            for (int t = pair; t < num_tiles && ok; t += npairs) {
                uint64_t a_base = a_desc0;
                uint32_t a_cp = a_chunk_pitch;   // bytes between the K chunks of an A slot
                if constexpr (GROUPED) {
                    if (a_load(tile_at(t)).nsub != 0) {
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
                    d_tmem = tmem_base + a * BN;
                }
                for (int kg = 0; kg < nkg; ++kg) {
                    if (!ptx::mbar_wait(&full[s], ph, p.timeout_cycles, abort_flag)) {
                        record_failure(p, abort_flag, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after_sync();
                    const uint64_t a_slot = a_base + ((s * R::kABytes) >> 4);
                    const uint64_t b_slot = b_desc0 + ((s * R::kBBytes) >> 4);
                    const int nc = nkb - kg * KC;   // chunks in this group: KC, except at a tile's end
                    if constexpr (FP8) {
                        // every epilogue warp of both CTAs releases the partial buffers in chunk
                        // order: the group's last buffer being free frees them all
                        const uint32_t last = acc_iter + static_cast<uint32_t>((nc < KC ? nc : KC) - 1);
                        if (!ptx::mbar_wait(&acce_bar[last % kNumAcc], ((last / kNumAcc) & 1u) ^ 1u,
                                            p.timeout_cycles, abort_flag)) {
                            record_failure(p, abort_flag, kStatusTimeout);
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after_sync();
                    }
                    auto issue_chunk = [&](int c, int chunk) -> bool {
                        uint32_t d = d_tmem;
                        if constexpr (FP8) {
                            d = tmem_base + (acc_iter % kNumAcc) * BN;
                            ++acc_iter;
                        }
                        const uint64_t a_desc = a_slot + ((c * a_cp) >> 4);
                        const uint64_t b_desc = b_slot + ((c * R::kBChunkBytes) >> 4);
#pragma unroll
                        for (int q = 0; q < kMmaPerChunk; ++q) {
                            const uint64_t step = static_cast<uint64_t>((q * kBytesPerMmaK) >> 4);
                            const uint32_t accumulate = (q > 0) ? 1u : (FP8 ? 0u : (chunk > 0 ? 1u : 0u));
                            if constexpr (FP8)
                                ptx::mma_e4m3_ss_pair(d, a_desc + step, b_desc + step, kIdesc, accumulate);
                            else
                                ptx::mma_bf16_ss_pair(d, a_desc + step, b_desc + step, kIdesc, accumulate);
                        }
                        return true;
                    };
                    // straight-line MMAs for a full group; only a tile's last group can be short
                    if (nc >= KC) {
#pragma unroll
                        for (int c = 0; c < KC; ++c)
                            if (!issue_chunk(c, kg * KC + c)) {
                                ok = false;
                                break;
                            }
                    } else {
#pragma unroll 1
                        for (int c = 0; c < nc; ++c)
                            if (!issue_chunk(c, kg * KC + c)) {
                                ok = false;
                                break;
                            }
                    }
                    if (!ok)
                        break;
                    // frees slot s in both CTAs (and marks FP8 partials ready in both)
                    ptx::mma_commit_pair(ptx::smem_u32(&consumed[s]));
                    ptx::mma_commit_pair(consumed_peer0 + s * 8);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok)
                    break;
                if (!FP8) {
                    const uint32_t a = acc_iter % kNumAcc;
                    ptx::mma_commit_pair(ptx::smem_u32(&accf_bar[a]));
                    ptx::mma_commit_pair(accf_peer0 + a * 8);
                    ++acc_iter;
                }
            }
            ptx::mma_commit_pair(ptx::smem_u32(drain_bar));
            ptx::mbar_wait(drain_bar, 0, p.timeout_cycles, nullptr);
        }
    } else {
        // ------------------------------------------------------------------ epilogue (both)
        const uint32_t q = warp & 3u;
        const uint32_t half = (warp - 2) / 4;   // FP8 column half (0 with 4 epilogue warps)
        const uint32_t row_in_tile = 128 * rank + q * 32 + lane;
        const uint32_t lane_addr = (q * 32u) << 16;
        const uint32_t acce_leader0 = ptx::mapa_shared(ptx::smem_u32(&acce_bar[0]), 0);
        auto release = [&](uint32_t idx) {   // this warp is done with TMEM buffer idx
            ptx::tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0)
                    ptx::mbar_arrive(&acce_bar[idx]);
                else
                    ptx::mbar_arrive_cluster(acce_leader0 + idx * 8);
            }
        };
        uint32_t acc_iter = 0;
        int gs = 0;
        uint32_t gph = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += npairs) {
            const TileCoord tc = tile_at(t);
            const int row = tc.m0 + static_cast<int>(row_in_tile);
            const bool row_ok = row < tc.row_end;
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
                    uint32_t r[32];
                    ptx::tmem_ld_32x32b_x32(tmem_base + lane_addr + a * BN + c * 32, r);
                    ptx::tmem_wait_ld(r);
                    if (c == BN / 32 - 1)
                        release(a);
                    float v[32];
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        v[jj] = __uint_as_float(r[jj]);
                    if (row_ok)
                        store_row_chunk32(crow, tc.n0 + c * 32, p.n, v);
                }
                ++acc_iter;
            } else {
                constexpr int kCols = Epi<FP8, BN>::kCols;
                constexpr int kLoads = kCols / 32;
                const int col0 = static_cast<int>(half) * kCols;
                float acc[kCols];
#pragma unroll
                for (int jj = 0; jj < kCols; ++jj)
                    acc[jj] = 0.0f;
                const float *sa_col = p.scale_a + (row_ok ? row : 0);
                float sa_g[KC], sb_g[KC][kLoads];   // scales of group kg, loaded one group ahead
                load_group_scales<KC, kLoads>(p, sa_col, row_ok, tc.n0 + col0, 0, nkb, sa_g, sb_g);
                for (int kg = 0; kg < nkg && ok; ++kg) {
                    float sa_n[KC], sb_n[KC][kLoads];
                    load_group_scales<KC, kLoads>(p, sa_col, row_ok, tc.n0 + col0, kg + 1, nkb, sa_n, sb_n);
                    if (!ptx::mbar_wait(&consumed[gs], gph, p.timeout_cycles, abort_flag)) {
                        record_failure(p, abort_flag, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    if (++gs == S) {
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
                        uint32_t r[kLoads][32];
#pragma unroll
                        for (int c = 0; c < kLoads; ++c)
                            ptx::tmem_ld_32x32b_x32(tmem_base + lane_addr + part * BN + col0 + c * 32, r[c]);
#pragma unroll
                        for (int c = 0; c < kLoads; ++c)
                            ptx::tmem_wait_ld(r[c]);
                        release(part);
#pragma unroll
                        for (int c = 0; c < kLoads; ++c) {
                            const float sc = sa_g[cc] * sb_g[cc][c];
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj)
                                acc[c * 32 + jj] = fmaf(__uint_as_float(r[c][jj]), sc, acc[c * 32 + jj]);
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

    // Nobody leaves while its pair may still touch its shared or tensor memory.
    ptx::tc_fence_before_sync();
    __syncwarp();
    ptx::cluster_sync();
    if (warp == 1) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

template <int BN, int KC, bool FP8, bool GROUPED>
constexpr int smem_bytes_for_pair()
{
    return 1024 + kRingBytes + 1024 + (GROUPED ? 2 * (kMaxExperts + 1) * 4 : 0);
}

} // namespace bi
