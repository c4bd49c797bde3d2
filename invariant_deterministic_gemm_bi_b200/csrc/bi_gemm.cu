// bi_gemm.cu -- host side of libbigemm: plans, argument checks, TMA tensor maps, launches and
// the extern "C" ABI declared in include/bi_gemm.h.
//
// The plan is a pure function of (N, K, dtype, num_experts): it picks one tile configuration
// (tile shape, MMA instruction shape, pipeline depth) and never looks at M, at the device's
// occupancy or at anything measured at run time.  This is the "fixed kernel path instead of
// run-time heuristics" of "DeepSeek V4的batch invariance：大模型确定性推理的工程基石" (lshu.cn),
// sections 3.1-3.2, with the split-K of the heuristic libraries removed altogether.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <deque>
#include <mutex>
#include <new>
#include <vector>

#include "bi_gemm.h"
#include "bi_kernels.cuh"
#include "bi_kernels_pair.cuh"

namespace {

using bi::GemmParams;

// ---------------------------------------------------------------------------------------------
// Kernel registry: every instantiated configuration
// ---------------------------------------------------------------------------------------------

// (A map, B map, 8-row A map for short grouped segments, parameters)
typedef void (*KernelFn)(const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,
                         const __grid_constant__ CUtensorMap, const GemmParams);

struct KernelEntry {
    int threads;   // threads per CTA
    int bm;        // tile height = MMA M (256 for a CTA pair)
    int bn;
    int kc;
    bool fp8;
    bool grouped;
    bool pair;     // cta_group::2 on a cluster of two CTAs
    KernelFn fn;
    int smem;
    int nsplit;    // MMAs per K step (MMA N = bn / nsplit)
    bool ksplit;   // fixed-split-K research variant (fp32 partials + merge)
    bool w4;       // e2m1 weights with per-column scale and zero point (with fp8)
    int chains;    // K chains of a dense bf16 tile (2: chunks of each parity summed apart, then added)
};

#define BI_ENTRY(BM, BN, KC, F8, GR)                                                               \
    KernelEntry{bi::Issue<F8, BN, 1, GR, KC>::kThreads, BM, BN, KC, F8, GR, false,                              \
                &bi::bi_gemm_kernel<BM, BN, KC, F8, GR>,                                           \
                bi::smem_bytes_for<BM, BN, KC, F8, GR>(), 1, false, false, 1}
#define BI_ENTRY_W4(BM, BN, KC)                                                                    \
    KernelEntry{bi::Issue<true, BN, 1, false, KC>::kThreads, BM, BN, KC, true, false, false,                       \
                &bi::bi_gemm_kernel<BM, BN, KC, true, false, 1, false, true>,                      \
                bi::smem_bytes_for<BM, BN, KC, true, false, 1, false, true>(), 1, false, true, 1}
#define BI_ENTRY_W4_SPLIT2(BM, BN, KC)                                                             \
    KernelEntry{bi::Issue<true, BN, 2, false, KC>::kThreads, BM, BN, KC, true, false, false,                       \
                &bi::bi_gemm_kernel<BM, BN, KC, true, false, 2, false, true>,                      \
                bi::smem_bytes_for<BM, BN, KC, true, false, 2, false, true>(), 2, false, true, 1}
#define BI_ENTRY_KSPLIT(BM, BN, KC)                                                                \
    KernelEntry{bi::Issue<false, BN, 1, false, KC>::kThreads, BM, BN, KC, false, false, false,                     \
                &bi::bi_gemm_kernel<BM, BN, KC, false, false, 1, true>,                            \
                bi::smem_bytes_for<BM, BN, KC, false, false, 1, true>(), 1, true, false, 1}
#define BI_ENTRY_SPLIT2(BM, BN, KC, F8)                                                            \
    KernelEntry{bi::Issue<F8, BN, 2, false, KC>::kThreads, BM, BN, KC, F8, false, false,                           \
                &bi::bi_gemm_kernel<BM, BN, KC, F8, false, 2>,                                     \
                bi::smem_bytes_for<BM, BN, KC, F8, false, 2>(), 2, false, false, 1}
#define BI_PAIR(BN, KC, F8, GR)                                                                    \
    KernelEntry{bi::Epi<F8, BN>::kThreads, 256, BN, KC, F8, GR, true,                              \
                &bi::bi_gemm_kernel_pair<BN, KC, F8, GR>,                                          \
                bi::smem_bytes_for_pair<BN, KC, F8, GR>(), 1, false, false, 1}

#define BI_ENTRY_CHAINS(BM, BN, KC, CHN)                                                           \
    KernelEntry{bi::Issue<false, BN, 1, false, KC, CHN>::kThreads, BM, BN, KC, false, false, false, \
                &bi::bi_gemm_kernel<BM, BN, KC, false, false, 1, false, false, CHN>,               \
                bi::smem_bytes_for<BM, BN, KC, false, false, 1, false, false, CHN>(), 1, false,    \
                false, CHN}
#define BI_ENTRY_CHAINS_SPLITN(BM, BN, KC, NS, CHN)                                                \
    KernelEntry{bi::Issue<false, BN, NS, false, KC, CHN>::kThreads, BM, BN, KC, false, false,      \
                false, &bi::bi_gemm_kernel<BM, BN, KC, false, false, NS, false, false, CHN>,       \
                bi::smem_bytes_for<BM, BN, KC, false, false, NS, false, false, CHN>(), NS, false,  \
                false, CHN}

// Narrow tiles (BN <= 64) run on one CTA; wide ones (BN >= 128) on a CTA pair.  Every tile comes
// in two forms: its preferred number of 128-byte K chunks per pipeline stage (3-D TMA boxes;
// needs K to be a multiple of the chunk), and one chunk per stage for any other K.  The bf16
// 64 x 32 and the FP8 128 x 64 tiles have a third, small-batch form with twice the preferred
// chunks per stage (the bf16 tile a fourth, tiny-batch form with 16), and wide forms that run
// two (bf16: or four) adjacent tiles in lockstep on one A operand (see dense_kernel_for).
const KernelEntry kKernels[] = {
    // bf16 32-column tiles: 64-row MMA, four K chains on up to four issuing threads (the plan
    // form, the small- and tiny-batch forms, one chunk per stage for K not a multiple of 64, and
    // the wide lockstep forms of two and four tiles)
    BI_ENTRY_CHAINS(64, 32, 1, 4),            BI_ENTRY_CHAINS(64, 32, 4, 4),
    BI_ENTRY_CHAINS(64, 32, 8, 4),            BI_ENTRY_CHAINS(64, 32, 16, 4),
    BI_ENTRY_CHAINS_SPLITN(64, 64, 4, 2, 4),  BI_ENTRY_CHAINS_SPLITN(64, 128, 2, 4, 4),
    BI_ENTRY(128, 64, 1, false, false), BI_ENTRY(128, 64, 2, false, false),
    BI_ENTRY(128, 32, 1, true, false),  BI_ENTRY(128, 32, 4, true, false),
    BI_ENTRY(128, 64, 1, true, false),  BI_ENTRY(128, 64, 2, true, false),
    BI_ENTRY(128, 64, 4, true, false),  BI_ENTRY_SPLIT2(128, 128, 2, true),
    BI_ENTRY(128, 32, 1, false, true),  BI_ENTRY(128, 32, 4, false, true),
    BI_ENTRY(128, 64, 1, false, true),  BI_ENTRY(128, 64, 2, false, true),
    BI_ENTRY(128, 128, 1, false, true), BI_ENTRY(128, 128, 2, false, true),
    // grouped wide form: 2 x 2 tiles of the 128 x 128 MoE plan on a CTA pair
    BI_PAIR(256, 1, false, true),
    BI_PAIR(128, 1, false, false),      BI_PAIR(128, 2, false, false),
    BI_PAIR(256, 1, false, false),      BI_PAIR(256, 2, false, false),
    BI_PAIR(128, 1, true, false),       BI_PAIR(128, 2, true, false),
    // e2m1 weights x e4m3 activations (the FP8 tiles; K is a multiple of 128)
    BI_ENTRY_W4(128, 32, 4),            BI_ENTRY_W4(128, 64, 2),
    BI_ENTRY_W4(128, 64, 4),            BI_ENTRY_W4_SPLIT2(128, 128, 2),
    // fixed-split-K research variant (bi_gemm_plan_splitk), not the product path
    BI_ENTRY_KSPLIT(128, 32, 1),        BI_ENTRY_KSPLIT(128, 32, 4),
    BI_ENTRY_KSPLIT(128, 64, 1),        BI_ENTRY_KSPLIT(128, 64, 2),
    BI_ENTRY_KSPLIT(128, 128, 1),       BI_ENTRY_KSPLIT(128, 128, 2),
};
constexpr int kNumKernels = sizeof(kKernels) / sizeof(kKernels[0]);

int preferred_chunks(int bn) { return bn <= 32 ? 4 : 2; }

const KernelEntry *find_kernel(int bm, int bn, int kc, bool fp8, bool grouped, bool w4 = false,
                               int chains = 1)
{
    for (int i = 0; i < kNumKernels; ++i)
        if (kKernels[i].bm == bm && kKernels[i].bn == bn && kKernels[i].kc == kc &&
            kKernels[i].fp8 == fp8 && kKernels[i].grouped == grouped && kKernels[i].nsplit == 1 &&
            !kKernels[i].ksplit && kKernels[i].w4 == w4 && kKernels[i].chains == chains)
            return &kKernels[i];
    return nullptr;
}

// Ring geometry of one launch (see bi::Rings): A slots hold the a_rows rows TMA brings; wide
// tiles give A and B the same depth, narrow ones keep up to ~96 KB for A and the rest for B.
struct RingGeom {
    int sa, sb;
    uint32_t a_stride, b_offset;
};

RingGeom ring_geometry(const KernelEntry *k, int a_rows)
{
    const int chunk = bi::kRowBytes;
    if (k->pair) {   // fixed at compile time (bi::PairRings): 128 A rows and BN/2 B rows per CTA
        const int a_bytes = k->kc * 128 * chunk;
        const int b_bytes = k->kc * (k->bn / 2) * chunk;
        int st = bi::kRingBytes / (a_bytes + b_bytes);
        if (st > bi::kMaxSB)
            st = bi::kMaxSB;
        return RingGeom{st, st, static_cast<uint32_t>(a_bytes), static_cast<uint32_t>(st * a_bytes)};
    }
    const int ring = k->grouped ? bi::kRingBytesGrouped : bi::kRingBytes1;
    const int a_stride = (k->kc * a_rows * chunk + 1023) / 1024 * 1024;   // slots start on swizzle atoms
    // The MMA reads BM rows from every A chunk: past the last loaded row of the last A slot it
    // reads on into the B ring, which lies right after the A region and must reach that far.
    const int over = (k->bm - a_rows) * chunk;
    const int b_stride = k->kc * k->bn * chunk;
    auto a_region_of = [&](int s) { return (s * a_stride + 1023) / 1024 * 1024; };
    int sa, sb, a_region;
    if (k->bn >= 128) {
        sa = ring / (a_stride + b_stride);
        if (sa > bi::kMaxSA)
            sa = bi::kMaxSA;
        sb = sa;
        a_region = a_region_of(sa);
        if (a_region + sb * b_stride > ring)
            --sa, --sb, a_region = a_region_of(sa);
    } else {
        sa = (96 * 1024) / a_stride;
        sa = sa < 2 ? 2 : sa > bi::kMaxSA ? bi::kMaxSA : sa;
        for (;; --sa) {   // deepest A ring that still leaves B at least as deep
            a_region = a_region_of(sa);
            sb = (ring - a_region) / b_stride;
            if (sb > bi::kMaxSB)
                sb = bi::kMaxSB;
            if (sb >= sa || sa == 2)
                break;
        }
    }
    if (a_region + sb * b_stride < sa * a_stride + over)
        sb = 0;   // the MMA's reads would leave the ring: reported as an invalid geometry
    // The kernel relies on 2 <= sa <= sb (the A-slot reuse test reads the consumed ring) and, for
    // FP8, on sb groups outlasting the partial-product ring.  Every tile in kKernels satisfies
    // this for every a_rows in [8, BM], except the bf16 tiny-batch form (16 chunks per group),
    // valid up to 24 rows and used up to 8; set_rows reports a violation and the launch is
    // refused.  tests/test_abi.py checks the reported depths.
    return RingGeom{sa, sb, static_cast<uint32_t>(a_stride), static_cast<uint32_t>(a_region)};
}

// ---------------------------------------------------------------------------------------------
// Plan table
// ---------------------------------------------------------------------------------------------

// The tile (BM x BN) for (N, K, dtype, experts).  Known projection shapes get the tile tuned for
// them; any other shape takes the widest tile that still gives enough tiles for a small batch,
// since without split-K the N tiles are the only parallelism such a batch has.  Tiles 256 rows
// high run on a CTA pair.  Grouped (MoE) plans use one-CTA tiles: an expert's segment is often
// only a few rows long, and a taller tile would only load more rows that are never stored.
struct TileChoice {
    int bm, bn;
};

TileChoice choose_tile(int64_t N, int64_t K, bi_dtype_t dtype, int experts)
{
    struct Row {
        int64_t n, k;
        int dtype, experts, bm, bn;
    };
    static const Row table[] = {
        {4096, 7168, BI_DTYPE_BF16, 1, 64, 32},               // decode-shaped projection
        {7168, 2048, BI_DTYPE_BF16, 1, 256, 256},             // prefill-shaped, wide N (CTA pair)
        {2048, 7168, BI_DTYPE_BF16, 1, 256, 256},             // prefill-shaped, long K (CTA pair)
        {256, 512, BI_DTYPE_BF16, 1, 64, 32},                 // small correctness shape
        {7168, 7168, BI_DTYPE_E4M3_BLOCKSCALED, 1, 128, 64},  // FP8 projection
        {7168, 7168, BI_DTYPE_E2M1_W4A8, 1, 128, 64},         // the same projection, e2m1 weights
        {2048, 7168, BI_DTYPE_BF16, 64, 128, 128},            // MoE experts
    };
    for (const Row &r : table)
        if (r.n == N && r.k == K && r.dtype == dtype && r.experts == (experts > 1 ? 64 : 1) &&
            (experts == 1 || experts == 64))
            return {r.bm, r.bn};
    if (experts > 1) {
        for (int bn = 128; bn > 32; bn /= 2)
            if ((N + bn - 1) / bn >= 100)
                return {128, bn};
        return {128, 32};
    }
    if (dtype == BI_DTYPE_E2M1_W4A8)   // one-CTA tiles only
        return {128, (N + 63) / 64 >= 100 ? 64 : 32};
    // wide dense fallback tiles run on a CTA pair (256 rows)
    const int max_bn = dtype == BI_DTYPE_E4M3_BLOCKSCALED ? 128 : 256;
    for (int bn = max_bn; bn >= 128; bn /= 2)
        if ((N + bn - 1) / bn >= 100)
            return {256, bn};
    if ((N + 63) / 64 >= 100)
        return {128, 64};
    return {dtype == BI_DTYPE_BF16 ? 64 : 128, 32};
}

// ---------------------------------------------------------------------------------------------
// Per-device state
// ---------------------------------------------------------------------------------------------

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool probed = false;
    bool ok = false;       // sm_100 family
    int num_sms = 0;
    bool attr_set[kNumKernels] = {};
    int max_pairs[kNumKernels] = {};   // co-resident CTA pairs of a pair kernel
};

std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

bi_status_t current_device(int *dev_out, DeviceInfo **info_out)
{
    int count = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess || count <= 0) {
        cudaGetLastError();
        return BI_ERR_NO_DEVICE;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return BI_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.probed) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess)
            return BI_ERR_CUDA;
        d.ok = prop.major == 10;
        d.num_sms = prop.multiProcessorCount;
        d.probed = true;
    }
    if (!d.ok)
        return BI_ERR_NO_DEVICE;
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    if (!g_encode)
        return BI_ERR_CUDA;
    *dev_out = dev;
    *info_out = &d;
    return BI_OK;
}

} // namespace

// ---------------------------------------------------------------------------------------------
// The plan object
// ---------------------------------------------------------------------------------------------

// Staging regions of bi_gemm_run_host_batch: one per batch in flight, as many as the caller's
// staging holds, 2 to kMaxHostSlots.  A region is refilled once its previous batch's copy-outs
// have completed, so the copy-in stream runs up to (regions - 1) batches ahead of the kernels.
constexpr int kMaxHostSlots = 32;
constexpr int kMaxHostCalls = 1024;   // GEMMs in one batch

// A batch's copy-outs are enqueued this many batches later (or by a flush): by then the kernels
// they wait for have long finished, so they never hold up the copy-ins queued behind them.
constexpr int kHostDefer = 2;

// A copy-out of bi_gemm_run_host_batch that waits for a later batch (or a flush) to be issued.
struct PendingOut {
    void *c_host;
    const void *c_dev;
    size_t bytes;
};

struct HostPipe {
    cudaEvent_t in_done[kMaxHostSlots] = {};
    cudaEvent_t gemm_done[kMaxHostSlots] = {};
    cudaEvent_t out_done[kMaxHostSlots] = {};
    uint64_t next = 0;                  // batches issued so far (region = next % slots)
    const void *staging = nullptr;      // layout of the last batch
    size_t slot_bytes = 0;              // bytes of one region
    int slots = 0;                      // regions
    // copy-outs of the last kHostDefer batches, not yet enqueued, oldest first, each with its
    // region (whose gemm_done was recorded after that batch's kernels)
    std::deque<std::pair<std::vector<PendingOut>, int>> pending;
    // stream capture: the capture the batches belong to, and its own region order
    unsigned long long cap_id = 0;
    uint64_t cap_next = 0;
    uint32_t cap_used = 0;              // regions filled inside the capture
};

struct bi_plan_s {
    int64_t n = 0, k = 0;
    bi_dtype_t dtype = BI_DTYPE_BF16;
    int experts = 1;
    const KernelEntry *kernel = nullptr;
    // The same tile with more K chunks per pipeline group, for launches whose A rows are few
    // (dense plans only; may be null).  It issues the same MMAs in the same K order, so a row's
    // result does not depend on which of the two a launch takes.
    const KernelEntry *kernel_small = nullptr;
    // The bf16 small-batch tile with twice its chunks again (16 per group), for launches of
    // fewer than 8 rows (dense bf16 64 x 32 plans only; may be null).  Same MMAs, same K order.
    const KernelEntry *kernel_tiny = nullptr;
    // Dense: two adjacent tiles in lockstep on one A operand, for launches with more tiles than
    // SMs.  Grouped: 2 x 2 tiles of the plan on a CTA pair (one 256 x 256 cta_group::2
    // instruction per K step), for launches with at least a tile's worth of rows per expert on
    // average.  Either way one instruction covers the tiles, in the plan's K order, and gives
    // every element the plan's bits.  May be null.
    const KernelEntry *kernel_wide = nullptr;
    // Four adjacent tiles in lockstep (bf16 plans with K chains), for dense launches whose lockstep pairs
    // still outnumber the SMs.  May be null.
    const KernelEntry *kernel_wide4 = nullptr;
    // CTA-pair plans 256 columns wide: the same tile cut in two 128-column halves, each run by
    // its own pair with a 256 x 128 instruction in the same K order, for launches with fewer
    // tiles than co-resident pairs.  May be null.
    const KernelEntry *kernel_half = nullptr;
    int small_rows = 64;     // kernel_small serves launches whose A boxes hold at most this many rows
    uint64_t timeout_ns = 2000000000ull;
    uint32_t debug_flags = 0;
    uint32_t flags = 0;      // BI_PLAN_* flags
    int k_splits = 1;        // > 1: fixed-split-K research plan (bi_gemm_plan_splitk)
    std::mutex mu;
    int *status[kMaxDevices] = {};
    // bi_gemm_run_host_batch, per device: the events that order the reuse of each staging slot
    // (copy-in done, GEMM done, copy-out done), the next slot, and the staging layout last used
    HostPipe *pipe[kMaxDevices] = {};
    std::mutex pipe_mu;      // one host batch of this plan at a time (the slot order is shared)
};

namespace {

bi_status_t plan_status_word(bi_plan_s *plan, int dev, int **out)
{
    std::lock_guard<std::mutex> lock(plan->mu);
    if (!plan->status[dev]) {
        int *p = nullptr;
        if (cudaMalloc(&p, sizeof(int)) != cudaSuccess)
            return BI_ERR_CUDA;
        if (cudaMemset(p, 0, sizeof(int)) != cudaSuccess) {
            cudaFree(p);
            return BI_ERR_CUDA;
        }
        plan->status[dev] = p;
    }
    *out = plan->status[dev];
    return BI_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// TMA map of a K-major operand [rows][ld] with 128-byte rows per box, 128-byte swizzle.
// kc == 1: 2-D, box {128 B of K, box_rows}.  kc > 1: 3-D view [K/chunk][rows][chunk] (the chunk
// index has a 128-byte stride), box {chunk, box_rows, kc}, which lands in shared memory as kc
// consecutive [box_rows x 128 B] tiles; it needs K to be a multiple of the chunk.
bi_status_t encode_operand(CUtensorMap *map, const void *base, bool fp8, int64_t K, int64_t rows,
                           int64_t ld_elems, int box_rows, int kc)
{
    const int elt = fp8 ? 1 : 2;
    const int chunk = bi::kRowBytes / elt;
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r;
    if (kc == 1) {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_elems * elt)};
        cuuint32_t box[2] = {static_cast<cuuint32_t>(chunk), static_cast<cuuint32_t>(box_rows)};
        r = g_encode(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(chunk), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(K / chunk)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld_elems * elt),
                                 static_cast<cuuint64_t>(bi::kRowBytes)};
        cuuint32_t box[3] = {static_cast<cuuint32_t>(chunk), static_cast<cuuint32_t>(box_rows),
                             static_cast<cuuint32_t>(kc)};
        r = g_encode(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                     const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    return r == CUDA_SUCCESS ? BI_OK : BI_ERR_CUDA;
}

// TMA map of packed e2m1 weights [rows][ld_elems / 2 bytes] (value k of a row in byte k / 2, the
// even value in the low four bits).  The boxes are those of an 8-bit operand -- 128 values of K
// per row, kc chunks per 3-D box -- and land in shared memory in the 16-byte-aligned form the
// MMA reads (each 8 bytes of values followed by 8 unused bytes, so 128 bytes per box row).  The
// format needs a 32-byte aligned base, row pitches of 32 bytes and K a multiple of 128.
bi_status_t encode_e2m1(CUtensorMap *map, const void *base, int64_t K, int64_t rows, int64_t ld_elems,
                        int box_rows, int kc)
{
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r;
    if (kc == 1) {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_elems / 2)};
        cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
        r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        // [K / 128][rows][128 values]; a chunk of 128 values is 64 bytes of global memory
        cuuint64_t dims[3] = {128u, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(K / 128)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld_elems / 2), 64u};
        cuuint32_t box[3] = {128u, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(kc)};
        r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    return r == CUDA_SUCCESS ? BI_OK : BI_ERR_CUDA;
}

bi_status_t ensure_kernel_attr(const KernelEntry *k, DeviceInfo *d)
{
    std::lock_guard<std::mutex> lock(g_dev_mu);
    const int ki = static_cast<int>(k - kKernels);
    if (!d->attr_set[ki]) {
        if (cudaFuncSetAttribute(reinterpret_cast<const void *>(k->fn),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, k->smem) != cudaSuccess)
            return BI_ERR_CUDA;
        if (k->pair) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(2 * (d->num_sms / 2));
            cfg.blockDim = dim3(k->threads);
            cfg.dynamicSmemBytes = k->smem;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, reinterpret_cast<const void *>(k->fn),
                                               &cfg) != cudaSuccess ||
                clusters < 1) {
                cudaGetLastError();
                clusters = d->num_sms / 2;
            }
            d->max_pairs[ki] = clusters;
        }
        d->attr_set[ki] = true;
    }
    return BI_OK;
}

int pair_grid_limit(const KernelEntry *k, const DeviceInfo *d)
{
    const int ki = static_cast<int>(k - kKernels);
    return d->max_pairs[ki] > 0 ? d->max_pairs[ki] : d->num_sms / 2;
}

bi_status_t launch_zero(void *C, int64_t ldc, int64_t rows, int64_t n, cudaStream_t stream)
{
    const int64_t total = rows * n;
    int blocks = static_cast<int>((total + 255) / 256);
    if (blocks > 4096)
        blocks = 4096;
    if (blocks < 1)
        blocks = 1;
    bi::bi_zero_kernel<<<blocks, 256, 0, stream>>>(static_cast<__nv_bfloat16 *>(C), ldc, rows, n);
    return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

// Checks shared by the dense and grouped runs (pointers, strides, alignment, 32-bit limits).
bi_status_t check_common(const bi_plan_s *plan, int64_t rows, const void *A, int64_t lda,
                         const void *B, int64_t ldb, const void *C, int64_t ldc)
{
    if (rows < 0)
        return BI_ERR_INVALID_ARG;
    if (rows == 0 || plan->n == 0)
        return BI_OK;
    if (!C)
        return BI_ERR_INVALID_ARG;
    if (ldc < plan->n)
        return BI_ERR_INVALID_ARG;
    if (!aligned16(C) || (ldc * 2) % 16 != 0)
        return BI_ERR_ALIGNMENT;
    if (plan->k == 0)
        return BI_OK;
    if (!A || !B)
        return BI_ERR_INVALID_ARG;
    if (lda < plan->k || ldb < plan->k)
        return BI_ERR_INVALID_ARG;
    const int elt = plan->dtype == BI_DTYPE_BF16 ? 2 : 1;   // bytes per A element
    if (!aligned16(A) || (lda * elt) % 16 != 0)
        return BI_ERR_ALIGNMENT;
    if (plan->dtype == BI_DTYPE_E2M1_W4A8) {
        // packed e2m1 rows (two values per byte): 32-byte aligned base and row pitch
        if ((reinterpret_cast<uintptr_t>(B) & 31u) != 0 || ldb % 64 != 0)
            return BI_ERR_ALIGNMENT;
    } else if (!aligned16(B) || (ldb * elt) % 16 != 0) {
        return BI_ERR_ALIGNMENT;
    }
    if (rows > INT32_MAX - 256 || plan->n * plan->experts > INT32_MAX - 512 ||
        plan->k > INT32_MAX - 256)
        return BI_ERR_UNSUPPORTED_SHAPE;
    return BI_OK;
}

// FP8 scale arguments of a dense run with M > 0, N > 0 and K > 0: both scales present, the
// K-block-major pitch of scale_a at least M, and 4-byte alignment of every scale pointer the
// kernel reads (scale_a only when it is a device pointer the kernel reads directly).
bi_status_t check_fp8_scales(int64_t M, const float *scale_a, int64_t ld_sa, const float *scale_b,
                             bool scale_a_read_by_kernel)
{
    if (!scale_a || !scale_b)
        return BI_ERR_DTYPE_MISMATCH;
    if (ld_sa < M)
        return BI_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(scale_b) & 3u)
        return BI_ERR_ALIGNMENT;
    if (scale_a_read_by_kernel && (reinterpret_cast<uintptr_t>(scale_a) & 3u))
        return BI_ERR_ALIGNMENT;
    return BI_OK;
}

// Dense bf16 plans of 32-column tiles use the 64-row MMA with four K chains on four issuing
// threads: one thread issues a tcgen05.mma every ~57 cycles whatever the shape, two on
// independent accumulators every ~29 and four every ~25 cycles, close to the 24 shared-memory
// wavefronts one 64 x 32 x 16 instruction reads (half the A rows of the 128-row instruction).
int chains_for(const TileChoice &tile, bool fp8, int experts)
{
    return (!fp8 && experts == 1 && tile.bm == 64 && tile.bn == 32) ? 4 : 1;
}

// Rows of A one TMA load brings for a dense problem of M rows: the tile's 128 rows, or, when the
// problem is smaller than one tile, only the rows that exist (rounded up to the 8-row swizzle
// atom).  This changes which shared-memory rows are written, not the MMA or its K order.
int dense_a_box_rows(int64_t M, int bm)
{
    return M >= bm ? bm : static_cast<int>((M + 7) / 8 * 8);
}

bool set_rows(GemmParams *p, const KernelEntry *k, int a_rows)
{
    const RingGeom g = ring_geometry(k, a_rows);
    // FP8: the epilogue tracks partial products on the consumed ring, which must outlast them
    const int nacc = k->fp8 ? ((512 / k->bn) < 8 ? (512 / k->bn) : 8) : 0;
    p->a_box_rows = a_rows;
    // the peer CTA of a pair has A rows to load unless the whole problem fits in 128 rows
    p->pair_a1 = (k->grouped || p->rows > 128) ? 1 : 0;
    p->sa = g.sa;
    p->sb = g.sb;
    p->a_stride = g.a_stride;
    p->b_offset = g.b_offset;
    return g.sa >= 2 && g.sa <= g.sb && g.sa <= bi::kMaxSA && g.sb <= bi::kMaxSB &&
           (!k->fp8 || k->pair || g.sb > nacc / k->kc);
}

GemmParams base_params(const bi_plan_s *plan, const KernelEntry *k, int64_t rows, void *C, int64_t ldc,
                       int *status)
{
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    const int elt = plan->dtype == BI_DTYPE_BF16 ? 2 : 1;   // bytes per A element
    p.rows = static_cast<int32_t>(rows);
    p.n = static_cast<int32_t>(plan->n);
    p.k = static_cast<int32_t>(plan->k);
    p.num_k_blocks = static_cast<int32_t>((plan->k * elt + bi::kRowBytes - 1) / bi::kRowBytes);
    p.num_n_blocks = static_cast<int32_t>((plan->n + k->bn - 1) / k->bn);
    p.num_m_blocks = static_cast<int32_t>((rows + k->bm - 1) / k->bm);
    p.num_experts = plan->experts;
    p.raster_m = 16;
    (void)set_rows(&p, k, k->bm);
    p.c = static_cast<__nv_bfloat16 *>(C);
    p.ldc = ldc;
    p.kb_scale = static_cast<int32_t>((plan->k + 127) / 128);
    p.status = status;
    // the wait limit is counted in SM cycles; 2 cycles per ns is at or above the B200's highest
    // SM clock (1965 MHz), so a wait lasts at least timeout_ns
    p.timeout_cycles = plan->timeout_ns * 2;
    p.debug_flags = plan->debug_flags;
    p.prefetch_b = (plan->flags & BI_PLAN_RESIDENT_WEIGHTS) && !k->grouped ? 1 : 0;
    return p;
}

// Launch kernel entry k.  `units` is the number of work tiles; a one-CTA kernel gets
// min(units, #SMs) CTAs, a pair kernel min(units, co-resident pairs) clusters of two CTAs.  Every
// launch is a programmatic dependent of the previous kernel in the stream: it may start (and set
// up its shared and tensor memory) while that kernel finishes, and waits for it to complete
// before touching global memory (bi::ptx::grid_dependency_wait).
bi_status_t launch_main(const KernelEntry *k, const DeviceInfo *d, const CUtensorMap &ta,
                        const CUtensorMap &tb, const CUtensorMap &ta8, const GemmParams &p,
                        int64_t units, cudaStream_t stream)
{
    if (units < 1)
        units = 1;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (!k->pair) {
        cfg.gridDim = dim3(static_cast<unsigned>(units < d->num_sms ? units : d->num_sms));
    } else {
        const int lim = pair_grid_limit(k, d);
        const int pairs = static_cast<int>(units < lim ? units : lim);
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 2;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
        cfg.gridDim = dim3(2 * pairs);
    }
    cfg.blockDim = dim3(k->threads);
    cfg.dynamicSmemBytes = k->smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = na;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, k->fn, ta, tb, ta8, p);
    return e == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

// Rows of A one TMA box covers and rows of B one box covers, for this plan and M.  One-CTA
// kernels load exactly the problem's rows when it has fewer than a tile's (see
// bi::GemmParams::a_box_rows).  A pair CTA owns 128 rows of a tile; a dense problem smaller than
// that boxes its roundup(M, 8) rows.
int a_box_rows_for(const KernelEntry *k, int64_t M)
{
    if (k->pair)
        return dense_a_box_rows(M, 128);
    return M >= k->bm ? k->bm : static_cast<int>(M);
}

int b_box_rows_for(const KernelEntry *k)
{
    return k->pair ? k->bn / 2 : k->bn;
}

// A dense launch of M rows whose A boxes hold at most bi_plan_s::small_rows rows takes the plan's
// small-batch kernel form (when it has one): with few A rows, groups of twice the chunks halve
// the per-group wait and commit overhead of the MMA threads, and the ring still holds two groups
// of A and of B (and, for FP8, more groups than partial-product buffers).  At most this many
// rows take the tiny-batch form (16 chunks per group): its 16 KB groups of A rows cost little
// shared memory only while the batch stays below 8 rows.
constexpr int kTinyBatchRows = 7;

// A dense launch with more tiles than the device has SMs takes the plan's wide form (when it has
// one): a CTA runs two adjacent column tiles in lockstep, so each A chunk is loaded once for both
// and the launch needs half the CTAs, i.e. fewer waves.
const KernelEntry *dense_kernel_for(const bi_plan_s *plan, const DeviceInfo *d, int64_t M)
{
    if (plan->kernel_half) {
        const int64_t m_blocks = (M + plan->kernel->bm - 1) / plan->kernel->bm;
        const int64_t n_blocks = (plan->n + plan->kernel->bn - 1) / plan->kernel->bn;
        if (m_blocks * n_blocks < pair_grid_limit(plan->kernel, d))
            return plan->kernel_half;
    }
    if (plan->kernel_tiny && M <= kTinyBatchRows)
        return plan->kernel_tiny;
    if (plan->kernel_small && a_box_rows_for(plan->kernel_small, M) <= plan->small_rows)
        return plan->kernel_small;
    if (plan->kernel_wide) {
        const int64_t m_blocks = (M + plan->kernel->bm - 1) / plan->kernel->bm;
        const int64_t n_blocks = (plan->n + plan->kernel->bn - 1) / plan->kernel->bn;
        if (m_blocks * n_blocks > d->num_sms) {
            if (plan->kernel_wide4 && m_blocks * ((n_blocks + 1) / 2) > d->num_sms)
                return plan->kernel_wide4;
            return plan->kernel_wide;
        }
    }
    return plan->kernel;
}

} // namespace

// ---------------------------------------------------------------------------------------------
// Static device scratch for bi_gemm_run_host_noalloc: status word + staging copies of A,
// scale_a and C.  Host code must not use the symbol as an address: it looks the device address
// up once per device with cudaGetSymbolAddress (the device current) and passes that pointer.
// ---------------------------------------------------------------------------------------------

static __device__ __align__(256) unsigned char bi_noalloc_scratch[BI_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mu;
unsigned char *g_noalloc_ptr[kMaxDevices] = {};

bi_status_t noalloc_scratch_for(int dev, unsigned char **out)
{
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, bi_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return BI_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = static_cast<unsigned char *>(p);
    }
    *out = g_noalloc_ptr[dev];
    return BI_OK;
}

constexpr int64_t round256(int64_t x) { return (x + 255) / 256 * 256; }

} // namespace

// ---------------------------------------------------------------------------------------------
// extern "C" ABI
// ---------------------------------------------------------------------------------------------

extern "C" {

int bi_gemm_abi_version(void) { return BI_GEMM_ABI_VERSION; }

const char *bi_status_string(bi_status_t s)
{
    switch (s) {
    case BI_OK: return "BI_OK";
    case BI_ERR_INVALID_ARG: return "BI_ERR_INVALID_ARG: invalid argument";
    case BI_ERR_ALIGNMENT: return "BI_ERR_ALIGNMENT: pointer or stride not 16-byte aligned";
    case BI_ERR_UNSUPPORTED_SHAPE: return "BI_ERR_UNSUPPORTED_SHAPE: shape not supported";
    case BI_ERR_DTYPE_MISMATCH: return "BI_ERR_DTYPE_MISMATCH: arguments do not match the plan's dtype";
    case BI_ERR_CUDA: return "BI_ERR_CUDA: a CUDA call failed";
    case BI_ERR_DEVICE_TIMEOUT: return "BI_ERR_DEVICE_TIMEOUT: a device pipeline wait ran out of time";
    case BI_ERR_BAD_OFFSETS: return "BI_ERR_BAD_OFFSETS: malformed grouped expert offsets";
    case BI_ERR_NO_DEVICE: return "BI_ERR_NO_DEVICE: no sm_100 CUDA device";
    }
    return "BI_ERR_UNKNOWN";
}

bi_status_t bi_gemm_plan(bi_plan_t *out, int64_t N, int64_t K, bi_dtype_t dtype, int num_experts)
{
    if (!out)
        return BI_ERR_INVALID_ARG;
    *out = nullptr;
    if (N < 0 || K < 0 || num_experts < 1)
        return BI_ERR_INVALID_ARG;
    if (dtype != BI_DTYPE_BF16 && dtype != BI_DTYPE_E4M3_BLOCKSCALED && dtype != BI_DTYPE_E2M1_W4A8)
        return BI_ERR_INVALID_ARG;
    if (num_experts > bi::kMaxExperts)
        return BI_ERR_UNSUPPORTED_SHAPE;
    if (num_experts > 1 && dtype != BI_DTYPE_BF16)
        return BI_ERR_UNSUPPORTED_SHAPE;
    if (N > INT32_MAX / 2 || K > INT32_MAX / 2 || N * num_experts > INT32_MAX / 2)
        return BI_ERR_UNSUPPORTED_SHAPE;
    const bool w4 = dtype == BI_DTYPE_E2M1_W4A8;
    if (w4 && K % 128 != 0)   // the packed e2m1 tensor format counts K in 128-value units
        return BI_ERR_UNSUPPORTED_SHAPE;
    const bool fp8 = dtype != BI_DTYPE_BF16;
    const TileChoice tile = choose_tile(N, K, dtype, num_experts);
    const int chunk_elems = fp8 ? 128 : 64;
    const int kc = ((K > 0 && K % chunk_elems == 0) || w4) ? preferred_chunks(tile.bn) : 1;
    const int chains = chains_for(tile, fp8, num_experts);
    const KernelEntry *k = find_kernel(tile.bm, tile.bn, kc, fp8, num_experts > 1, w4, chains);
    if (!k)
        return BI_ERR_UNSUPPORTED_SHAPE;
    bi_plan_s *p = new (std::nothrow) bi_plan_s();
    if (!p)
        return BI_ERR_INVALID_ARG;
    p->n = N;
    p->k = K;
    p->dtype = dtype;
    p->experts = num_experts;
    p->kernel = k;
    if (num_experts == 1 && !k->pair && (k->bm == 128 || k->chains > 1) &&
        k->kc == preferred_chunks(k->bn) && k->bn == (fp8 ? 64 : 32))
        p->kernel_small = find_kernel(k->bm, k->bn, 2 * k->kc, fp8, false, w4, chains);
    if (p->kernel_small && !fp8 && p->kernel_small->kc == 8)
        p->kernel_tiny = find_kernel(k->bm, k->bn, 16, false, false, false, chains);
    // plans with K chains take the 8-chunk form up to 32 rows: their 64-row A boxes would leave
    // a 96 KB B ring at 8 chunks, while 4 chunks keep eight B groups in flight
    p->small_rows = chains > 1 ? 32 : 64;
    if (num_experts == 1 && k->pair && k->bn == 256)
        p->kernel_half = find_kernel(256, 128, k->kc, fp8, false, w4, chains);
    if (num_experts > 1 && !k->pair && k->bm == 128 && k->bn == 128) {
        for (int i = 0; i < kNumKernels; ++i)
            if (kKernels[i].pair && kKernels[i].grouped && kKernels[i].bn == 256)
                p->kernel_wide = &kKernels[i];
    }
    if (num_experts == 1 && !k->pair && (k->bm == 128 || k->chains > 1) &&
        k->bn == (fp8 ? 64 : 32) && K % chunk_elems == 0 && K > 0) {
        for (int i = 0; i < kNumKernels; ++i)
            if (kKernels[i].bm == k->bm && kKernels[i].fp8 == fp8 && kKernels[i].w4 == w4 &&
                !kKernels[i].grouped && kKernels[i].chains == chains && !kKernels[i].ksplit) {
                if (kKernels[i].nsplit == 2 && kKernels[i].bn == 2 * k->bn)
                    p->kernel_wide = &kKernels[i];
                if (kKernels[i].nsplit == 4 && kKernels[i].bn == 4 * k->bn)
                    p->kernel_wide4 = &kKernels[i];
            }
    }
    *out = p;
    return BI_OK;
}

bi_status_t bi_gemm_plan_column_shard(bi_plan_t *out, bi_plan_t full, int64_t n_begin, int64_t n_end)
{
    if (!out)
        return BI_ERR_INVALID_ARG;
    *out = nullptr;
    if (!full || full->experts != 1 || full->k_splits > 1)
        return BI_ERR_INVALID_ARG;
    if (n_begin < 0 || n_end < n_begin || n_end > full->n)
        return BI_ERR_INVALID_ARG;
    // FP8 weights carry one scale per 128 x 128 block: a shard must start on a block boundary so
    // that its columns keep their scale blocks (the caller passes scale_b from row n_begin / 128)
    if (full->dtype == BI_DTYPE_E4M3_BLOCKSCALED && n_begin % 128 != 0)
        return BI_ERR_UNSUPPORTED_SHAPE;
    bi_plan_s *p = new (std::nothrow) bi_plan_s();
    if (!p)
        return BI_ERR_INVALID_ARG;
    p->n = n_end - n_begin;
    p->k = full->k;
    p->dtype = full->dtype;
    p->experts = 1;
    p->kernel = full->kernel;
    p->kernel_small = full->kernel_small;
    p->kernel_tiny = full->kernel_tiny;
    p->kernel_wide = full->kernel_wide;
    p->kernel_wide4 = full->kernel_wide4;
    p->kernel_half = full->kernel_half;
    p->small_rows = full->small_rows;
    p->timeout_ns = full->timeout_ns;
    p->flags = full->flags;
    *out = p;
    return BI_OK;
}

bi_status_t bi_gemm_plan_destroy(bi_plan_t plan)
{
    if (!plan)
        return BI_OK;
    int cur = -1;
    const bool have_dev = cudaGetDevice(&cur) == cudaSuccess;
    for (int d = 0; d < kMaxDevices; ++d) {
        if (plan->status[d]) {
            cudaSetDevice(d);
            cudaFree(plan->status[d]);
        }
        if (plan->pipe[d]) {
            cudaSetDevice(d);
            for (int i = 0; i < kMaxHostSlots; ++i) {
                cudaEventDestroy(plan->pipe[d]->in_done[i]);
                cudaEventDestroy(plan->pipe[d]->gemm_done[i]);
                cudaEventDestroy(plan->pipe[d]->out_done[i]);
            }
            delete plan->pipe[d];
        }
    }
    if (have_dev)
        cudaSetDevice(cur);
    cudaGetLastError();
    delete plan;
    return BI_OK;
}

bi_status_t bi_gemm_plan_describe(bi_plan_t plan, bi_plan_info_t *info)
{
    if (!plan || !info)
        return BI_ERR_INVALID_ARG;
    const bool fp8 = plan->dtype != BI_DTYPE_BF16;
    std::memset(info, 0, sizeof(*info));
    info->n = plan->n;
    info->k = plan->k;
    info->dtype = plan->dtype;
    info->num_experts = plan->experts;
    info->block_m = plan->kernel->bm;
    info->block_n = plan->kernel->bn;
    info->block_k = (fp8 ? 128 : 64) * plan->kernel->kc;
    info->cta_group = plan->kernel->pair ? 2 : 1;
    info->mma_m = plan->kernel->bm;
    info->mma_n = plan->kernel->bn;
    info->mma_k = fp8 ? 32 : 16;
    const RingGeom g = ring_geometry(plan->kernel, plan->kernel->bm);
    info->stages = g.sb;
    info->stages_a = g.sa;
    info->k_order_id = plan->k_splits > 1 ? 1 : plan->kernel->chains == 4 ? 3 : plan->kernel->chains == 2 ? 2 : 0;
    info->k_splits = plan->k_splits;
    info->threads_per_cta = plan->kernel->threads;
    info->smem_bytes = plan->kernel->smem;
    const int nacc = fp8 ? ((512 / plan->kernel->bn) < 8 ? (512 / plan->kernel->bn) : 8) : 2;
    int cols = 32;
    while (cols < nacc * plan->kernel->bn * plan->kernel->chains)
        cols *= 2;
    info->tmem_columns = cols;
    return BI_OK;
}

bi_status_t bi_gemm_set_wait_timeout(bi_plan_t plan, uint64_t timeout_ns)
{
    if (!plan)
        return BI_ERR_INVALID_ARG;
    plan->timeout_ns = timeout_ns ? timeout_ns : 2000000000ull;
    return BI_OK;
}

bi_status_t bi_gemm_plan_set_flags(bi_plan_t plan, uint32_t flags)
{
    if (!plan || (flags & ~(BI_PLAN_RESIDENT_WEIGHTS | BI_PLAN_HOST_ROW_BLOCKS)))
        return BI_ERR_INVALID_ARG;
    plan->flags = flags;
    return BI_OK;
}

bi_status_t bi_gemm_debug_set_flags(bi_plan_t plan, uint32_t flags)
{
    if (!plan)
        return BI_ERR_INVALID_ARG;
    plan->debug_flags = flags;
    return BI_OK;
}

bi_status_t bi_gemm_run(bi_plan_t plan, int64_t M, const void *A, int64_t lda, const void *B,
                        int64_t ldb, void *C, int64_t ldc, const float *scale_a, int64_t ld_sa,
                        const float *scale_b, cudaStream_t stream)
{
    if (!plan)
        return BI_ERR_INVALID_ARG;
    if (plan->experts != 1 || plan->k_splits > 1)
        return BI_ERR_INVALID_ARG;
    if (plan->dtype == BI_DTYPE_E2M1_W4A8)
        return BI_ERR_DTYPE_MISMATCH;   // bi_gemm_run_w4a8
    const bool fp8 = plan->dtype == BI_DTYPE_E4M3_BLOCKSCALED;
    if (fp8) {
        if (M > 0 && plan->n > 0 && plan->k > 0) {
            const bi_status_t sst = check_fp8_scales(M, scale_a, ld_sa, scale_b, true);
            if (sst != BI_OK)
                return sst;
        }
    } else if (scale_a || scale_b) {
        return BI_ERR_DTYPE_MISMATCH;
    }
    bi_status_t st = check_common(plan, M, A, lda, B, ldb, C, ldc);
    if (st != BI_OK || M == 0 || plan->n == 0)
        return st;
    int dev = 0;
    DeviceInfo *d = nullptr;
    if ((st = current_device(&dev, &d)) != BI_OK)
        return st;
    if (plan->k == 0)
        return launch_zero(C, ldc, M, plan->n, stream);
    int *status = nullptr;
    if ((st = plan_status_word(plan, dev, &status)) != BI_OK)
        return st;
    const KernelEntry *k = dense_kernel_for(plan, d, M);
    if ((st = ensure_kernel_attr(k, d)) != BI_OK)
        return st;
    CUtensorMap ta, tb;
    const int a_rows = a_box_rows_for(k, M);
    if ((st = encode_operand(&ta, A, fp8, plan->k, M, lda, a_rows, k->kc)) != BI_OK)
        return st;
    if ((st = encode_operand(&tb, B, fp8, plan->k, plan->n, ldb, b_box_rows_for(k), k->kc)) != BI_OK)
        return st;
    GemmParams p = base_params(plan, k, M, C, ldc, status);
    if (!set_rows(&p, k, a_rows))
        return BI_ERR_UNSUPPORTED_SHAPE;
    p.scale_a = scale_a;
    p.ld_sa = ld_sa;
    p.scale_b = scale_b;
    const int64_t tiles = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks;
    return launch_main(k, d, ta, tb, ta, p, tiles, stream);
}

bi_status_t bi_grouped_gemm_run(bi_plan_t plan, int64_t total_rows, const void *A, int64_t lda,
                                const void *B, int64_t ldb, void *C, int64_t ldc,
                                const int32_t *expert_offsets, cudaStream_t stream)
{
    if (!plan)
        return BI_ERR_INVALID_ARG;
    if (plan->experts <= 1)
        return BI_ERR_INVALID_ARG;
    bi_status_t st = check_common(plan, total_rows, A, lda, B, ldb, C, ldc);
    if (st != BI_OK || total_rows == 0 || plan->n == 0)
        return st;
    if (!expert_offsets)
        return BI_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(expert_offsets) & 3u)
        return BI_ERR_ALIGNMENT;
    int dev = 0;
    DeviceInfo *d = nullptr;
    if ((st = current_device(&dev, &d)) != BI_OK)
        return st;
    if (plan->k == 0)
        return launch_zero(C, ldc, total_rows, plan->n, stream);
    int *status = nullptr;
    if ((st = plan_status_word(plan, dev, &status)) != BI_OK)
        return st;
    // With at least a tile's worth of rows per expert on average, 2 x 2 plan tiles run on a CTA
    // pair (the wide form: one wider instruction, same K order, same bits).
    const KernelEntry *k = plan->kernel;
    if (plan->kernel_wide && total_rows >= static_cast<int64_t>(plan->kernel->bm) * plan->experts)
        k = plan->kernel_wide;
    if ((st = ensure_kernel_attr(k, d)) != BI_OK)
        return st;
    CUtensorMap ta, tb, ta8;
    const int a_rows = k->pair ? 128 : k->bm;
    if ((st = encode_operand(&ta, A, false, plan->k, total_rows, lda, a_rows, k->kc)) != BI_OK)
        return st;
    // short segments load their rows as 8-row boxes
    if ((st = encode_operand(&ta8, A, false, plan->k, total_rows, lda, 8, k->kc)) != BI_OK)
        return st;
    if ((st = encode_operand(&tb, B, false, plan->k, plan->n * plan->experts, ldb, b_box_rows_for(k),
                             k->kc)) != BI_OK)
        return st;
    GemmParams p = base_params(plan, k, total_rows, C, ldc, status);
    (void)set_rows(&p, k, a_rows);
    p.offsets = expert_offsets;
    // Upper bound on the tile count without reading the offsets: sum_e ceil(len_e/BM) is at
    // most total_rows/BM + E.
    const int64_t max_tiles = (total_rows / k->bm + plan->experts) * p.num_n_blocks;
    return launch_main(k, d, ta, tb, ta8, p, max_tiles, stream);
}

bi_status_t bi_gemm_run_host(bi_plan_t plan, int64_t M, const void *A_host, int64_t lda,
                             const void *B, int64_t ldb, void *C_host, int64_t ldc,
                             const float *scale_a_host, int64_t ld_sa, const float *scale_b,
                             void *A_dev, void *C_dev, float *scale_a_dev, cudaStream_t stream)
{
    if (!plan)
        return BI_ERR_INVALID_ARG;
    if (M < 0)
        return BI_ERR_INVALID_ARG;
    if (plan->dtype == BI_DTYPE_E2M1_W4A8)
        return BI_ERR_DTYPE_MISMATCH;
    if (M == 0 || plan->n == 0)
        return BI_OK;
    const bool fp8 = plan->dtype == BI_DTYPE_E4M3_BLOCKSCALED;
    if (!C_host || !C_dev || (plan->k > 0 && (!A_host || !A_dev)))
        return BI_ERR_INVALID_ARG;
    if (fp8 && plan->k > 0 && (!scale_a_host || !scale_a_dev))
        return BI_ERR_DTYPE_MISMATCH;
    const int elt = fp8 ? 1 : 2;
    // Validate before enqueueing any copy.
    bi_status_t st = check_common(plan, M, A_dev, lda, B, ldb, C_dev, ldc);
    if (st != BI_OK)
        return st;
    if (fp8 && plan->k > 0 && (st = check_fp8_scales(M, scale_a_dev, ld_sa, scale_b, true)) != BI_OK)
        return st;
    if (!fp8 && (scale_a_host || scale_b))
        return BI_ERR_DTYPE_MISMATCH;
    if (plan->k > 0) {
        if (cudaMemcpyAsync(A_dev, A_host, static_cast<size_t>(M * lda * elt),
                            cudaMemcpyHostToDevice, stream) != cudaSuccess)
            return BI_ERR_CUDA;
        if (fp8 && cudaMemcpyAsync(scale_a_dev, scale_a_host,
                                   static_cast<size_t>(((plan->k + 127) / 128) * ld_sa * 4),
                                   cudaMemcpyHostToDevice, stream) != cudaSuccess)
            return BI_ERR_CUDA;
    }
    st = bi_gemm_run(plan, M, A_dev, lda, B, ldb, C_dev, ldc, fp8 ? scale_a_dev : nullptr, ld_sa,
                     fp8 ? scale_b : nullptr, stream);
    if (st != BI_OK)
        return st;
    if (cudaMemcpyAsync(C_host, C_dev, static_cast<size_t>(M * ldc * 2), cudaMemcpyDeviceToHost,
                        stream) != cudaSuccess)
        return BI_ERR_CUDA;
    return BI_OK;
}

// The plan's host-batch state on this device, created with its events on first use.
static bi_status_t host_pipe_for(bi_plan_s *plan, int dev, HostPipe **out)
{
    HostPipe *hp = plan->pipe[dev];
    if (!hp) {
        hp = new (std::nothrow) HostPipe();
        if (!hp)
            return BI_ERR_INVALID_ARG;
        for (int i = 0; i < kMaxHostSlots; ++i)
            if (cudaEventCreateWithFlags(&hp->in_done[i], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&hp->gemm_done[i], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&hp->out_done[i], cudaEventDisableTiming) != cudaSuccess) {
                cudaGetLastError();
                for (int j = 0; j < kMaxHostSlots; ++j) {
                    if (hp->in_done[j]) cudaEventDestroy(hp->in_done[j]);
                    if (hp->gemm_done[j]) cudaEventDestroy(hp->gemm_done[j]);
                    if (hp->out_done[j]) cudaEventDestroy(hp->out_done[j]);
                }
                delete hp;
                return BI_ERR_CUDA;
            }
        plan->pipe[dev] = hp;
    }
    *out = hp;
    return BI_OK;
}

// Enqueue on copy_out, after each batch's kernels, the copy-outs pending from all but the newest
// `keep` batches (oldest first).
static bi_status_t host_batch_flush(HostPipe *hp, cudaStream_t copy_out, size_t keep = 0)
{
    while (hp->pending.size() > keep) {
        const auto &b = hp->pending.front();
        if (cudaStreamWaitEvent(copy_out, hp->gemm_done[b.second], 0) != cudaSuccess)
            return BI_ERR_CUDA;
        for (const PendingOut &o : b.first)
            if (cudaMemcpyAsync(o.c_host, o.c_dev, o.bytes, cudaMemcpyDeviceToHost, copy_out) != cudaSuccess)
                return BI_ERR_CUDA;
        if (cudaEventRecord(hp->out_done[b.second], copy_out) != cudaSuccess)
            return BI_ERR_CUDA;
        hp->pending.pop_front();
    }
    return BI_OK;
}

// Where the calls of one host batch live in its staging region: the A rows of every call, then
// the C rows, then (FP8) the scale_a blocks.  With BI_PLAN_HOST_ROW_BLOCKS a call whose host A
// rows begin where the previous call's end shares that call's copy (one run), and likewise for
// C, so a batch laid out back to back in one host allocation moves with one copy each way
// instead of one per call (without the flag nothing says two touching buffers are one
// allocation, and a copy may not span two).  Every run starts on a 256-byte boundary; a call
// inside a run sits at its host offset from the run's start.
struct HostRun {
    const void *host;   // first byte in host memory
    int64_t off;        // offset in the region's A (or C) part
    int64_t bytes;
};

struct BatchLayout {
    std::vector<int64_t> a_off, c_off, s_off;   // per call, within their parts (-1: M == 0)
    std::vector<HostRun> a_runs, c_runs;
    int64_t a_part = 0, c_part = 0, s_part = 0;
    int64_t bytes() const { return a_part + c_part + s_part; }
};

// Returns false for arguments no call may have (negative or huge sizes).
static bool host_batch_layout(const bi_plan_s *plan, int n, const bi_host_gemm_t *calls, BatchLayout *L)
{
    const bool fp8 = plan->dtype == BI_DTYPE_E4M3_BLOCKSCALED;
    const int elt = fp8 ? 1 : 2;
    const int64_t kb = (plan->k + 127) / 128;
    const int64_t cap = int64_t(1) << 40;   // bounds every factor, so no product below can wrap
    L->a_off.assign(static_cast<size_t>(n), -1);
    L->c_off.assign(static_cast<size_t>(n), -1);
    L->s_off.assign(static_cast<size_t>(n), -1);
    int64_t a = 0, c = 0, sa = 0;
    const bool merge = (plan->flags & BI_PLAN_HOST_ROW_BLOCKS) != 0;
    auto place = [merge](std::vector<HostRun> &runs, int64_t &end, const void *host, int64_t bytes) {
        const unsigned char *h = static_cast<const unsigned char *>(host);
        if (merge && !runs.empty()) {
            HostRun &r = runs.back();
            if (static_cast<const unsigned char *>(r.host) + r.bytes == h) {
                const int64_t off = r.off + r.bytes;
                r.bytes += bytes;
                end = r.off + r.bytes;
                return off;
            }
        }
        const int64_t off = round256(end);
        runs.push_back(HostRun{host, off, bytes});
        end = off + bytes;
        return off;
    };
    for (int i = 0; i < n; ++i) {
        const bi_host_gemm_t &g = calls[i];
        if (g.M < 0 || g.M > cap || g.lda < 0 || g.lda > cap || g.ldc < 0 || g.ldc > cap ||
            g.ld_sa < 0 || g.ld_sa > cap)
            return false;
        if (g.M == 0)
            continue;
        if (plan->k > 0)
            L->a_off[i] = place(L->a_runs, a, g.A_host, g.M * g.lda * elt);
        L->c_off[i] = place(L->c_runs, c, g.C_host, g.M * g.ldc * 2);
        if (fp8 && plan->k > 0) {
            L->s_off[i] = sa;
            sa += round256(kb * g.ld_sa * 4);
        }
    }
    L->a_part = round256(a);
    L->c_part = round256(c);
    L->s_part = sa;
    return true;
}

size_t bi_gemm_host_batch_staging_bytes(bi_plan_t plan, int n, const bi_host_gemm_t *calls, int regions)
{
    if (!plan || n < 0 || n > kMaxHostCalls || (n > 0 && !calls) || regions < 2 || regions > kMaxHostSlots)
        return 0;
    BatchLayout L;
    if (!host_batch_layout(plan, n, calls, &L))
        return 0;
    return static_cast<size_t>(L.bytes()) * static_cast<size_t>(regions);
}

bi_status_t bi_gemm_run_host_batch(bi_plan_t plan, int n, const bi_host_gemm_t *calls, void *staging,
                                   size_t staging_bytes, cudaStream_t copy_in, cudaStream_t compute,
                                   cudaStream_t copy_out)
{
    if (!plan || n < 0 || n > kMaxHostCalls || (n > 0 && !calls))
        return BI_ERR_INVALID_ARG;
    if (plan->experts != 1 || plan->k_splits > 1)
        return BI_ERR_INVALID_ARG;
    if (plan->dtype == BI_DTYPE_E2M1_W4A8)
        return BI_ERR_DTYPE_MISMATCH;
    if (n == 0 || plan->n == 0)
        return BI_OK;
    const bool fp8 = plan->dtype == BI_DTYPE_E4M3_BLOCKSCALED;
    const int64_t kb = (plan->k + 127) / 128;
    BatchLayout L;
    if (!host_batch_layout(plan, n, calls, &L))
        return BI_ERR_INVALID_ARG;
    const int64_t region_bytes = L.bytes();
    if (region_bytes == 0)
        return BI_OK;   // every call has M == 0
    if (!staging || staging_bytes < static_cast<size_t>(region_bytes) * 2)
        return BI_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(staging) & 255u)
        return BI_ERR_ALIGNMENT;
    const size_t fit = staging_bytes / static_cast<size_t>(region_bytes);
    const int slots = fit > static_cast<size_t>(kMaxHostSlots) ? kMaxHostSlots : static_cast<int>(fit);
    unsigned char *base = static_cast<unsigned char *>(staging);
    // Validate every call before enqueueing anything, at its addresses in region 0 (every region
    // has the same alignment).
    for (int i = 0; i < n; ++i) {
        const bi_host_gemm_t &g = calls[i];
        if (g.M == 0)
            continue;
        if (!g.C_host || (plan->k > 0 && !g.A_host))
            return BI_ERR_INVALID_ARG;
        unsigned char *A_dev = plan->k > 0 ? base + L.a_off[i] : base;
        bi_status_t st = check_common(plan, g.M, A_dev, g.lda, g.B, g.ldb, base + L.a_part + L.c_off[i], g.ldc);
        if (st != BI_OK)
            return st;
        if (fp8 && plan->k > 0) {
            if ((st = check_fp8_scales(g.M, g.scale_a_host, g.ld_sa, g.scale_b, false)) != BI_OK)
                return st;
        } else if (!fp8 && (g.scale_a_host || g.scale_b)) {
            return BI_ERR_DTYPE_MISMATCH;
        }
    }
    int dev = 0;
    DeviceInfo *d = nullptr;
    bi_status_t st = current_device(&dev, &d);
    if (st != BI_OK)
        return st;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    unsigned long long cap_id = 0;
    if (cudaStreamGetCaptureInfo(compute, &cap, &cap_id) != cudaSuccess)
        return BI_ERR_CUDA;
    const bool captured = cap == cudaStreamCaptureStatusActive;
    std::lock_guard<std::mutex> lock(plan->pipe_mu);
    HostPipe *hp = nullptr;
    if ((st = host_pipe_for(plan, dev, &hp)) != BI_OK)
        return st;
    if (captured) {
        if (hp->cap_id != cap_id) {
            // the first batch of this capture: copy-outs pending from outside it would run at
            // replay instead of now, so they must have been flushed; the copy streams join the
            // capture by waiting on the compute stream once
            if (!hp->pending.empty())
                return BI_ERR_INVALID_ARG;
            if (cudaEventRecord(hp->gemm_done[0], compute) != cudaSuccess ||
                cudaStreamWaitEvent(copy_in, hp->gemm_done[0], 0) != cudaSuccess ||
                cudaStreamWaitEvent(copy_out, hp->gemm_done[0], 0) != cudaSuccess)
                return BI_ERR_CUDA;
            hp->cap_id = cap_id;
            hp->cap_next = 0;
            hp->cap_used = 0;
        }
    } else {
        // A different staging buffer or layout than the last batch: the regions may overlap the
        // old ones, so the copy-ins wait for every copy-out issued so far.
        const bool relayout = hp->staging != staging || hp->slot_bytes != static_cast<size_t>(region_bytes) ||
                              hp->slots != slots;
        if (relayout) {
            if ((st = host_batch_flush(hp, copy_out)) != BI_OK)
                return st;
            if (hp->next > 0)
                for (int i = 0; i < hp->slots; ++i)
                    if (cudaStreamWaitEvent(copy_in, hp->out_done[i], 0) != cudaSuccess)
                        return BI_ERR_CUDA;
            hp->next = 0;
        }
        hp->staging = staging;
        hp->slot_bytes = static_cast<size_t>(region_bytes);
        hp->slots = slots;
    }
    // This batch's copy-ins into its region (refilled once the region's previous copy-outs have
    // completed); then the copy-outs of the batch kHostDefer batches back, queued after these
    // copy-ins, behind kernels that have long finished; then this batch's kernels after one wait
    // for its copy-ins.  A copy-out queued while its kernel is still running would hold up the
    // copies queued after it.
    uint64_t &next = captured ? hp->cap_next : hp->next;
    const int r = static_cast<int>(next % static_cast<uint64_t>(slots));
    ++next;
    unsigned char *R = base + r * region_bytes;
    const bool reused = captured ? ((hp->cap_used >> r) & 1u) != 0 : true;
    if (reused && cudaStreamWaitEvent(copy_in, hp->out_done[r], 0) != cudaSuccess)
        return BI_ERR_CUDA;
    if (captured)
        hp->cap_used |= 1u << r;
    for (const HostRun &run : L.a_runs)
        if (cudaMemcpyAsync(R + run.off, run.host, static_cast<size_t>(run.bytes), cudaMemcpyHostToDevice,
                            copy_in) != cudaSuccess)
            return BI_ERR_CUDA;
    if (fp8)
        for (int i = 0; i < n; ++i)
            if (L.s_off[i] >= 0 &&
                cudaMemcpyAsync(R + L.a_part + L.c_part + L.s_off[i], calls[i].scale_a_host,
                                static_cast<size_t>(kb * calls[i].ld_sa * 4), cudaMemcpyHostToDevice,
                                copy_in) != cudaSuccess)
                return BI_ERR_CUDA;
    std::vector<PendingOut> outs;
    outs.reserve(L.c_runs.size());
    for (const HostRun &run : L.c_runs)
        outs.push_back(PendingOut{const_cast<void *>(run.host), R + L.a_part + run.off,
                                  static_cast<size_t>(run.bytes)});
    if ((st = host_batch_flush(hp, copy_out, kHostDefer - 1)) != BI_OK)
        return st;
    if (cudaEventRecord(hp->in_done[r], copy_in) != cudaSuccess ||
        cudaStreamWaitEvent(compute, hp->in_done[r], 0) != cudaSuccess)
        return BI_ERR_CUDA;
    for (int i = 0; i < n; ++i) {
        const bi_host_gemm_t &g = calls[i];
        if (g.M == 0)
            continue;
        unsigned char *A_dev = plan->k > 0 ? R + L.a_off[i] : R;
        float *sa_dev = fp8 && plan->k > 0 ? reinterpret_cast<float *>(R + L.a_part + L.c_part + L.s_off[i]) : nullptr;
        if ((st = bi_gemm_run(plan, g.M, A_dev, g.lda, g.B, g.ldb, R + L.a_part + L.c_off[i], g.ldc,
                              sa_dev, g.ld_sa, fp8 ? g.scale_b : nullptr, compute)) != BI_OK)
            return st;
    }
    if (cudaEventRecord(hp->gemm_done[r], compute) != cudaSuccess)
        return BI_ERR_CUDA;
    hp->pending.emplace_back(std::move(outs), r);
    return BI_OK;
}

bi_status_t bi_gemm_host_batch_flush(bi_plan_t plan, cudaStream_t copy_in, cudaStream_t compute,
                                     cudaStream_t copy_out)
{
    if (!plan)
        return BI_ERR_INVALID_ARG;
    int dev = 0;
    DeviceInfo *d = nullptr;
    bi_status_t st = current_device(&dev, &d);
    if (st != BI_OK)
        return st;
    std::lock_guard<std::mutex> lock(plan->pipe_mu);
    HostPipe *hp = plan->pipe[dev];
    if (!hp)
        return BI_OK;
    if ((st = host_batch_flush(hp, copy_out)) != BI_OK)
        return st;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    unsigned long long cap_id = 0;
    if (cudaStreamGetCaptureInfo(compute, &cap, &cap_id) != cudaSuccess)
        return BI_ERR_CUDA;
    if (cap == cudaStreamCaptureStatusActive && cap_id == hp->cap_id) {
        // join both copy streams back into the compute stream so the capture can end
        if (cudaEventRecord(hp->in_done[0], copy_in) != cudaSuccess ||
            cudaEventRecord(hp->out_done[0], copy_out) != cudaSuccess ||
            cudaStreamWaitEvent(compute, hp->in_done[0], 0) != cudaSuccess ||
            cudaStreamWaitEvent(compute, hp->out_done[0], 0) != cudaSuccess)
            return BI_ERR_CUDA;
        hp->cap_id = 0;
    }
    return BI_OK;
}

bi_status_t bi_gemm_run_host_noalloc(bi_plan_t plan, int64_t M, const void *A_host, int64_t lda,
                                     const void *B, int64_t ldb, void *C_host, int64_t ldc,
                                     const float *scale_a_host, int64_t ld_sa,
                                     const float *scale_b, cudaStream_t stream)
{
    if (!plan)
        return BI_ERR_INVALID_ARG;
    if (plan->experts != 1 || plan->k_splits > 1 || M < 0)
        return BI_ERR_INVALID_ARG;
    if (plan->dtype == BI_DTYPE_E2M1_W4A8)
        return BI_ERR_DTYPE_MISMATCH;
    if (M == 0 || plan->n == 0)
        return BI_OK;
    const bool fp8 = plan->dtype == BI_DTYPE_E4M3_BLOCKSCALED;
    const int elt = fp8 ? 1 : 2;
    if (!C_host || (plan->k > 0 && !A_host))
        return BI_ERR_INVALID_ARG;
    if (fp8 && plan->k > 0) {
        // scale_a_host is only copied (any alignment); scale_b is read by the kernel
        const bi_status_t sst = check_fp8_scales(M, scale_a_host, ld_sa, scale_b, false);
        if (sst != BI_OK)
            return sst;
    } else if (!fp8 && (scale_a_host || scale_b)) {
        return BI_ERR_DTYPE_MISMATCH;
    }
    if (lda < plan->k || ldc < plan->n || (fp8 && ld_sa < 0))
        return BI_ERR_INVALID_ARG;
    // Bound every factor of the scratch offsets before multiplying: no row count, pitch or
    // scale pitch can exceed the scratch size, so each product below stays far inside int64.
    const int64_t cap = static_cast<int64_t>(BI_NOALLOC_SCRATCH_BYTES);
    if (M > cap || lda > cap || ldc > cap || (fp8 && ld_sa > cap))
        return BI_ERR_UNSUPPORTED_SHAPE;
    // Scratch layout: [status word | A | C | scale_a], each part 256-byte aligned.
    const int64_t kb = (plan->k + 127) / 128;
    const int64_t a_off = 256;
    const int64_t c_off = a_off + round256(M * lda * elt);
    const int64_t s_off = c_off + round256(M * ldc * 2);
    const int64_t need = s_off + (fp8 ? round256(kb * ld_sa * 4) : 0);
    if (need > static_cast<int64_t>(BI_NOALLOC_SCRATCH_BYTES))
        return BI_ERR_UNSUPPORTED_SHAPE;
    int dev = 0;
    DeviceInfo *d = nullptr;
    bi_status_t st = current_device(&dev, &d);
    if (st != BI_OK)
        return st;
    unsigned char *base = nullptr;
    if ((st = noalloc_scratch_for(dev, &base)) != BI_OK)
        return st;
    int *status = reinterpret_cast<int *>(base);
    void *A_dev = base + a_off;
    void *C_dev = base + c_off;
    float *sa_dev = reinterpret_cast<float *>(base + s_off);
    if ((st = check_common(plan, M, A_dev, lda, B, ldb, C_dev, ldc)) != BI_OK)
        return st;
    if (cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess)
        return BI_ERR_CUDA;
    if (plan->k == 0) {
        if ((st = launch_zero(C_dev, ldc, M, plan->n, stream)) != BI_OK)
            return st;
    } else {
        if (cudaMemcpyAsync(A_dev, A_host, static_cast<size_t>(M * lda * elt),
                            cudaMemcpyHostToDevice, stream) != cudaSuccess)
            return BI_ERR_CUDA;
        if (fp8 && cudaMemcpyAsync(sa_dev, scale_a_host, static_cast<size_t>(kb * ld_sa * 4),
                                   cudaMemcpyHostToDevice, stream) != cudaSuccess)
            return BI_ERR_CUDA;
        const KernelEntry *k = dense_kernel_for(plan, d, M);
        if ((st = ensure_kernel_attr(k, d)) != BI_OK)
            return st;
        CUtensorMap ta, tb;
        const int a_rows = a_box_rows_for(k, M);
        if ((st = encode_operand(&ta, A_dev, fp8, plan->k, M, lda, a_rows, k->kc)) != BI_OK)
            return st;
        if ((st = encode_operand(&tb, B, fp8, plan->k, plan->n, ldb, b_box_rows_for(k), k->kc)) != BI_OK)
            return st;
        GemmParams p = base_params(plan, k, M, C_dev, ldc, status);
        if (!set_rows(&p, k, a_rows))
            return BI_ERR_UNSUPPORTED_SHAPE;
        p.scale_a = fp8 ? sa_dev : nullptr;
        p.ld_sa = fp8 ? ld_sa : 0;
        p.scale_b = fp8 ? scale_b : nullptr;
        const int64_t tiles = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks;
        if ((st = launch_main(k, d, ta, tb, ta, p, tiles, stream)) != BI_OK)
            return st;
    }
    if (cudaMemcpyAsync(C_host, C_dev, static_cast<size_t>(M * ldc * 2), cudaMemcpyDeviceToHost,
                        stream) != cudaSuccess)
        return BI_ERR_CUDA;
    // the status word comes back on the same stream, so one synchronisation covers C and it
    int host = 0;
    if (cudaMemcpyAsync(&host, status, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return BI_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return BI_ERR_CUDA;
    return host == 0 ? BI_OK : static_cast<bi_status_t>(host);
}

// ---------------------------------------------------------------------------------------------
// e2m1 weights x e4m3 activations
// ---------------------------------------------------------------------------------------------

size_t bi_gemm_w4a8_workspace_bytes(int64_t M)
{
    return M > 0 ? static_cast<size_t>(round256(M * 4)) : 0;
}

bi_status_t bi_gemm_run_w4a8(bi_plan_t plan, int64_t M, const void *A, int64_t lda,
                             const float *scale_a, int64_t ld_sa, const void *W, int64_t ldw,
                             const float *w_scale, const float *w_zero, float *workspace,
                             size_t workspace_bytes, void *C, int64_t ldc, cudaStream_t stream)
{
    if (!plan)
        return BI_ERR_INVALID_ARG;
    if (plan->dtype != BI_DTYPE_E2M1_W4A8)
        return BI_ERR_DTYPE_MISMATCH;
    if (plan->experts != 1 || plan->k_splits > 1)
        return BI_ERR_INVALID_ARG;
    bi_status_t st = check_common(plan, M, A, lda, W, ldw, C, ldc);
    if (st != BI_OK || M == 0 || plan->n == 0)
        return st;
    if (plan->k > 0) {
        if (!scale_a || !w_scale)
            return BI_ERR_INVALID_ARG;
        if (ld_sa < M)
            return BI_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(scale_a) & 3u) || (reinterpret_cast<uintptr_t>(w_scale) & 3u) ||
            (reinterpret_cast<uintptr_t>(w_zero) & 3u))
            return BI_ERR_ALIGNMENT;
        if (w_zero) {
            if (!workspace || workspace_bytes < bi_gemm_w4a8_workspace_bytes(M))
                return BI_ERR_INVALID_ARG;
            if (reinterpret_cast<uintptr_t>(workspace) & 15u)
                return BI_ERR_ALIGNMENT;
        }
    }
    int dev = 0;
    DeviceInfo *d = nullptr;
    if ((st = current_device(&dev, &d)) != BI_OK)
        return st;
    if (plan->k == 0)
        return launch_zero(C, ldc, M, plan->n, stream);
    int *status = nullptr;
    if ((st = plan_status_word(plan, dev, &status)) != BI_OK)
        return st;
    const KernelEntry *k = dense_kernel_for(plan, d, M);
    if ((st = ensure_kernel_attr(k, d)) != BI_OK)
        return st;
    CUtensorMap ta, tb;
    const int a_rows = a_box_rows_for(k, M);
    if ((st = encode_operand(&ta, A, true, plan->k, M, lda, a_rows, k->kc)) != BI_OK)
        return st;
    if ((st = encode_e2m1(&tb, W, plan->k, plan->n, ldw, b_box_rows_for(k), k->kc)) != BI_OK)
        return st;
    GemmParams p = base_params(plan, k, M, C, ldc, status);
    if (!set_rows(&p, k, a_rows))
        return BI_ERR_UNSUPPORTED_SHAPE;
    p.scale_a = scale_a;
    p.ld_sa = ld_sa;
    p.w_scale = w_scale;
    p.w_zero = w_zero;
    p.w_rowsum = w_zero ? workspace : nullptr;
    if (w_zero) {
        // the row sums of the dequantised A, for the zero-point term: one CTA per row for a few
        // rows, one warp per row once there are enough rows to fill the device (the two compute
        // the same bits).  The GEMM reads them after this grid has completed: it is this
        // kernel's programmatic dependent and waits for it before touching global memory.
        const bool warp_per_row = M > 1024;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.gridDim = dim3(static_cast<unsigned>(warp_per_row ? (M + 7) / 8 : M));
        cfg.blockDim = dim3(256);
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, warp_per_row ? bi::bi_w4_rowsum_warp_kernel : bi::bi_w4_rowsum_kernel,
                               static_cast<const uint8_t *>(A), lda, scale_a, ld_sa,
                               static_cast<int32_t>(M), static_cast<int32_t>(plan->k),
                               workspace) != cudaSuccess)
            return BI_ERR_CUDA;
    }
    const int64_t tiles = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks;
    return launch_main(k, d, ta, tb, ta, p, tiles, stream);
}

// ---------------------------------------------------------------------------------------------
// Fixed-split-K research variant (not the batch-invariant product path)
// ---------------------------------------------------------------------------------------------

bi_status_t bi_gemm_plan_splitk(bi_plan_t *out, int64_t N, int64_t K, int splits)
{
    if (!out)
        return BI_ERR_INVALID_ARG;
    *out = nullptr;
    if (N < 0 || K < 0 || (splits != 2 && splits != 4 && splits != 8))
        return BI_ERR_INVALID_ARG;
    if (N > INT32_MAX / 2 || K > INT32_MAX / 2)
        return BI_ERR_UNSUPPORTED_SHAPE;
    const int64_t nkb = (K * 2 + bi::kRowBytes - 1) / bi::kRowBytes;
    if (nkb < splits)
        return BI_ERR_UNSUPPORTED_SHAPE;   // every split must own at least one K chunk
    // the widest tile that still gives >= 100 work units (tiles x splits) for one row tile
    int bn = 32;
    for (int cand = 128; cand >= 32; cand /= 2)
        if ((N + cand - 1) / cand * splits >= 100) {
            bn = cand;
            break;
        }
    const int kc = (K > 0 && K % 64 == 0) ? preferred_chunks(bn) : 1;
    const KernelEntry *k = nullptr;
    for (int i = 0; i < kNumKernels; ++i)
        if (kKernels[i].ksplit && kKernels[i].bn == bn && kKernels[i].kc == kc)
            k = &kKernels[i];
    if (!k)
        return BI_ERR_UNSUPPORTED_SHAPE;
    bi_plan_s *p = new (std::nothrow) bi_plan_s();
    if (!p)
        return BI_ERR_INVALID_ARG;
    p->n = N;
    p->k = K;
    p->dtype = BI_DTYPE_BF16;
    p->experts = 1;
    p->kernel = k;
    p->k_splits = splits;
    *out = p;
    return BI_OK;
}

size_t bi_gemm_splitk_workspace_bytes(bi_plan_t plan, int64_t M)
{
    if (!plan || plan->k_splits <= 1 || M <= 0)
        return 0;
    const int64_t ld_ws = (plan->n + 3) / 4 * 4;
    return static_cast<size_t>(plan->k_splits) * static_cast<size_t>(M) * static_cast<size_t>(ld_ws) * 4u;
}

bi_status_t bi_gemm_run_splitk(bi_plan_t plan, int64_t M, const void *A, int64_t lda, const void *B,
                               int64_t ldb, void *C, int64_t ldc, void *workspace,
                               size_t workspace_bytes, cudaStream_t stream)
{
    if (!plan || plan->k_splits <= 1)
        return BI_ERR_INVALID_ARG;
    bi_status_t st = check_common(plan, M, A, lda, B, ldb, C, ldc);
    if (st != BI_OK || M == 0 || plan->n == 0)
        return st;
    if (!workspace || workspace_bytes < bi_gemm_splitk_workspace_bytes(plan, M))
        return BI_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u)
        return BI_ERR_ALIGNMENT;
    int dev = 0;
    DeviceInfo *d = nullptr;
    if ((st = current_device(&dev, &d)) != BI_OK)
        return st;
    if (plan->k == 0)
        return launch_zero(C, ldc, M, plan->n, stream);
    int *status = nullptr;
    if ((st = plan_status_word(plan, dev, &status)) != BI_OK)
        return st;
    const KernelEntry *k = plan->kernel;
    if ((st = ensure_kernel_attr(k, d)) != BI_OK)
        return st;
    CUtensorMap ta, tb;
    const int a_rows = a_box_rows_for(k, M);
    if ((st = encode_operand(&ta, A, false, plan->k, M, lda, a_rows, k->kc)) != BI_OK)
        return st;
    if ((st = encode_operand(&tb, B, false, plan->k, plan->n, ldb, b_box_rows_for(k), k->kc)) != BI_OK)
        return st;
    GemmParams p = base_params(plan, k, M, C, ldc, status);
    if (!set_rows(&p, k, a_rows))
        return BI_ERR_UNSUPPORTED_SHAPE;
    p.prefetch_b = 0;
    p.k_splits = plan->k_splits;
    p.ws = static_cast<float *>(workspace);
    p.ld_ws = (plan->n + 3) / 4 * 4;
    p.ws_split_stride = M * p.ld_ws;
    const int64_t units = static_cast<int64_t>(p.num_m_blocks) * p.num_n_blocks * plan->k_splits;
    if ((st = launch_main(k, d, ta, tb, ta, p, units, stream)) != BI_OK)
        return st;
    const int64_t total = M * plan->n;
    const int64_t blocks = (total + 255) / 256;
    const int grid = static_cast<int>(blocks < d->num_sms * 8 ? blocks : d->num_sms * 8);
    bi::bi_splitk_merge_kernel<<<grid, 256, 0, stream>>>(p.ws, p.ld_ws, p.ws_split_stride,
                                                          plan->k_splits,
                                                          static_cast<__nv_bfloat16 *>(C), ldc, M,
                                                          plan->n);
    return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status_t bi_gemm_sync_status(bi_plan_t plan, cudaStream_t stream)
{
    if (!plan)
        return BI_ERR_INVALID_ARG;
    int dev = 0;
    DeviceInfo *d = nullptr;
    bi_status_t st = current_device(&dev, &d);
    if (st != BI_OK)
        return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return BI_ERR_CUDA;
    int *word = nullptr;
    {
        std::lock_guard<std::mutex> lock(plan->mu);
        word = plan->status[dev];
    }
    if (!word)
        return BI_OK;
    int host = 0;
    if (cudaMemcpy(&host, word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return BI_ERR_CUDA;
    if (host != 0 && cudaMemset(word, 0, sizeof(int)) != cudaSuccess)
        return BI_ERR_CUDA;
    return host == 0 ? BI_OK : static_cast<bi_status_t>(host);
}

} // extern "C"
