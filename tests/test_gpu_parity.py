"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element.

Small and ragged shapes are compared in full; the full-size workloads, in the launch
configuration the benchmark times, on sampled rows that the oracle computes one by one.  Inputs
come from the seeded generators in ``invariant_deterministic_gemm_bi_b200.inputs`` and reach both
sides as the same bits.  Floating-point inputs are held to the tolerance in ``tests/parity.py``;
small-integer and power-of-two-scale inputs must match the oracle's bf16 bits exactly.
"""
import numpy as np
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
import oracle
from invariant_deterministic_gemm_bi_b200 import inputs
from tests import routing as routing_mod
from tests import parity
from tests.gpu_util import GuardedC, kblock_major_scales, strided_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_dense(A, B, M=None, scale_a=None, scale_b=None, dtype=bg.BI_DTYPE_BF16):
    N, K = B.shape
    M = A.shape[0] if M is None else M
    plan = bg.bi_gemm_plan(N, K, dtype, 1)
    out = GuardedC(M, N)
    bg.bi_gemm_run(plan, A, B, out.c, scale_a=scale_a, scale_b=scale_b)
    bg.bi_gemm_sync_status(plan)
    out.check()
    return out.c, plan


def oracle_bf16(A, B):
    return oracle.gemm_bf16(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B))


# ---------------------------------------------------------------------------------------------
# dense bf16, small and ragged
# ---------------------------------------------------------------------------------------------

SMALL_M = [1, 3, 8, 17, 64]


@pytest.mark.parametrize("M", SMALL_M)
def test_small_gaussian_within_tolerance(M):
    A = inputs.bf16_gaussian((M, 512), seed=1000 + M)
    B = inputs.bf16_gaussian((256, 512), seed=1001)
    C, _ = run_dense(A.to(DEV), B.to(DEV))
    cref, _ = oracle_bf16(A, B)
    parity.assert_within_tolerance(parity.bits(C), cref, 512, parity.rms(A.float().numpy()),
                                   parity.rms(B.float().numpy()), f"small M={M}")


@pytest.mark.parametrize("M", SMALL_M)
def test_small_integers_bit_exact(M):
    A = inputs.bf16_integers((M, 512), seed=1100 + M)
    B = inputs.bf16_integers((256, 512), seed=1101)
    C, _ = run_dense(A.to(DEV), B.to(DEV))
    _, cbits = oracle_bf16(A, B)
    parity.assert_bits_equal_values(parity.bits(C), cbits, f"integer M={M}")


RAGGED = [
    # (M, N, K, lda, ldb): tails in every dimension, strided operands, several tiles per CTA
    (300, 200, 200, 208, 200),
    (129, 33, 72, 72, 80),
    (5, 7, 3, 8, 8),
    (1, 1, 8, 8, 8),
    (257, 1000, 100, 104, 112),
    (2048, 2048, 128, 128, 128),
    (130, 6400, 136, 136, 136),     # BN 64
    (129, 12800, 72, 72, 72),       # BN 128
    (200, 25600, 64, 64, 64),       # BN 256
]


@pytest.mark.parametrize("M,N,K,lda,ldb", RAGGED)
def test_ragged_shapes(M, N, K, lda, ldb):
    A = inputs.bf16_gaussian((M, K), seed=7 * M + K)
    B = inputs.bf16_gaussian((N, K), seed=11 * N + K)
    Ad = strided_rows(A.to(DEV), lda)
    Bd = strided_rows(B.to(DEV), ldb)
    C, plan = run_dense(Ad, Bd)
    cref, _ = oracle_bf16(A, B)
    parity.assert_within_tolerance(parity.bits(C), cref, K, parity.rms(A.float().numpy()),
                                   parity.rms(B.float().numpy()), f"ragged {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(300, 200, 200), (129, 12800, 72), (200, 25600, 64)])
def test_ragged_integers_bit_exact(M, N, K):
    A = inputs.bf16_integers((M, K), seed=3 * M)
    B = inputs.bf16_integers((N, K), seed=5 * N)
    C, _ = run_dense(A.to(DEV), B.to(DEV))
    _, cbits = oracle_bf16(A, B)
    parity.assert_bits_equal_values(parity.bits(C), cbits, f"ragged integer {M}x{N}x{K}")


@pytest.mark.parametrize("K", [64, 128, 192, 256, 320, 448, 136, 200])
@pytest.mark.parametrize("M", [1, 8, 40])
def test_four_chain_plans_with_few_chunks(M, K):
    # The 32-column bf16 plans reduce K in four chains (chunk c to chain c % 4) and add them as
    # (c0 + c1) + (c2 + c3); K of 1..7 chunks leaves chains empty or short, including ragged K
    # (136, 200: the one-chunk-per-stage form).
    N = 256
    plan = bg.bi_gemm_plan(N, K)
    assert bg.bi_gemm_plan_describe(plan)["k_order_id"] == 3
    A = inputs.bf16_integers((M, K), seed=2300 + M + K)
    B = inputs.bf16_integers((N, K), seed=2301 + K)
    C, _ = run_dense(A.to(DEV), B.to(DEV))
    _, cbits = oracle_bf16(A, B)
    parity.assert_bits_equal_values(parity.bits(C), cbits, f"integers M={M} K={K}")
    A = inputs.bf16_gaussian((M, K), seed=2310 + M + K)
    B = inputs.bf16_gaussian((N, K), seed=2311 + K)
    C, _ = run_dense(A.to(DEV), B.to(DEV))
    cref, _ = oracle_bf16(A, B)
    parity.assert_within_tolerance(parity.bits(C), cref, K, parity.rms(A.float().numpy()),
                                   parity.rms(B.float().numpy()), f"gaussian M={M} K={K}")


def test_wide_lockstep_form_ragged_integers_bit_exact():
    # 64x32 four-chain plan at M = 300: 645 tiles > 148 SMs, so four adjacent tiles run in
    # lockstep on one A operand; N = 4128 leaves the last group of tiles partly outside N,
    # K = 7232 (113 chunks) gives the chains unequal lengths and a short last group.
    M, N, K = 300, 4128, 7232
    A = inputs.bf16_integers((M, K), seed=2201, device=DEV)
    B = inputs.bf16_integers((N, K), seed=2202, device=DEV)
    C, plan = run_dense(A, B)
    info = bg.bi_gemm_plan_describe(plan)
    assert (info["block_m"], info["block_n"]) == (64, 32)
    rows = [0, 1, 63, 64, 127, 128, 200, 255, 256, 299]
    _, cbits = oracle.gemm_bf16_rows(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B), rows)
    parity.assert_bits_equal_values(parity.bits(C)[rows], cbits, f"wide form {M}x{N}x{K}")


def test_k_zero_writes_zeros_and_m_zero_is_a_noop():
    plan = bg.bi_gemm_plan(40, 0)
    out = GuardedC(3, 40)
    A = torch.zeros((3, 8), dtype=torch.bfloat16, device=DEV)
    B = torch.zeros((40, 8), dtype=torch.bfloat16, device=DEV)
    bg.bi_gemm_run(plan, A, B, out.c)
    bg.bi_gemm_sync_status(plan)
    out.check()
    assert torch.all(out.c.float() == 0)
    plan2 = bg.bi_gemm_plan(40, 8)
    out2 = GuardedC(1, 40)
    bg.bi_gemm_run(plan2, A, B, out2.c, M=0)
    torch.cuda.synchronize()
    assert torch.all(out2.buf == 0x7FC1)


# ---------------------------------------------------------------------------------------------
# dense bf16, full-size workloads, sampled rows
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,M", [(4096, 7168, 1), (4096, 7168, 16), (4096, 7168, 64),
                                   (4096, 7168, 256), (7168, 2048, 1024), (7168, 2048, 4096),
                                   (7168, 2048, 16384), (2048, 7168, 1024), (2048, 7168, 4096),
                                   (2048, 7168, 16384)])
def test_full_size_sampled_rows(N, K, M):
    A = inputs.bf16_gaussian((M, K), seed=2000 + M, device=DEV)
    B = inputs.bf16_gaussian((N, K), seed=2001, std=K ** -0.5, device=DEV)
    C, _ = run_dense(A, B)
    rows = sorted({0, M - 1, M // 2, min(127, M - 1), min(128, M - 1), (M * 7) // 11})
    cref, _ = oracle.gemm_bf16_rows(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B), rows)
    parity.assert_within_tolerance(parity.bits(C)[rows], cref, K, parity.rms_t(A),
                                   parity.rms_t(B), f"{N}x{K} M={M}")


# ---------------------------------------------------------------------------------------------
# FP8 e4m3 block-scaled
# ---------------------------------------------------------------------------------------------

def fp8_case(M, N, K, seed, integer=False):
    KB, NB = (K + 127) // 128, (N + 127) // 128
    if integer:
        qa = inputs.e4m3_integers((M, K), seed)
        qb = inputs.e4m3_integers((N, K), seed + 1)
        sa = inputs.scales_pow2((M, KB), seed + 2)
        sb = inputs.scales_pow2((NB, KB), seed + 3)
    else:
        qa = inputs.e4m3_gaussian((M, K), seed)
        qb = inputs.e4m3_gaussian((N, K), seed + 1)
        sa = inputs.scales_log_uniform((M, KB), seed + 2)
        sb = inputs.scales_log_uniform((NB, KB), seed + 3)
    return qa, qb, sa, sb


def run_fp8(qa, qb, sa, sb):
    M, K = qa.shape
    N = qb.shape[0]
    sa_d = kblock_major_scales(sa.to(DEV))
    ld = ((K + 15) // 16) * 16          # 16-byte row pitch for TMA
    C, _ = run_dense(strided_rows(qa.to(DEV), ld), strided_rows(qb.to(DEV), ld), scale_a=sa_d,
                     scale_b=sb.to(DEV).contiguous(), dtype=bg.BI_DTYPE_E4M3_BLOCKSCALED)
    return C


def fp8_rms(q, scales, block_rows):
    v = parity.e4m3_bits_to_f64(inputs.to_numpy_bits(q))
    s = scales.numpy().astype(np.float64)
    s_full = np.repeat(np.repeat(s, block_rows, axis=0)[: v.shape[0]], 128, axis=1)[:, : v.shape[1]]
    return parity.rms(v * s_full)


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (8, 256, 512), (64, 256, 512), (200, 300, 384),
                                   (130, 6400, 256), (129, 12800, 256), (3, 40, 200)])
def test_fp8_within_tolerance(M, N, K):
    qa, qb, sa, sb = fp8_case(M, N, K, seed=4000 + M + N)
    C = run_fp8(qa, qb, sa, sb)
    cref, _ = oracle.gemm_fp8_blockscaled(inputs.to_numpy_bits(qa), inputs.to_numpy_bits(qb),
                                          sa.numpy(), sb.numpy())
    parity.assert_within_tolerance(parity.bits(C), cref, K, fp8_rms(qa, sa, 1), fp8_rms(qb, sb, 128),
                                   f"fp8 {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(8, 256, 512), (130, 6400, 256), (129, 12800, 256)])
def test_fp8_pow2_scales_integers_bit_exact(M, N, K):
    qa, qb, sa, sb = fp8_case(M, N, K, seed=4100 + M, integer=True)
    C = run_fp8(qa, qb, sa, sb)
    _, cbits = oracle.gemm_fp8_blockscaled(inputs.to_numpy_bits(qa), inputs.to_numpy_bits(qb),
                                           sa.numpy(), sb.numpy())
    parity.assert_bits_equal_values(parity.bits(C), cbits, f"fp8 integer {M}x{N}x{K}")


# A problem with fewer rows than a tile loads exactly its rows: chunk c of an A slot then starts
# c * M * 128 bytes in, inside a 1024-byte swizzle atom whenever M is not a multiple of 8.
EXACT_HEIGHT_M = [1, 2, 3, 5, 6, 7, 9, 15, 17, 23, 33, 63]


@pytest.mark.parametrize("M", EXACT_HEIGHT_M)
def test_exact_height_a_rows_bf16_bit_exact(M):
    N, K = 512, 2048      # the 64 x 32 plan: every form below 64 rows
    A = inputs.bf16_integers((M, K), seed=2400 + M)
    B = inputs.bf16_integers((N, K), seed=2401)
    C, _ = run_dense(A.to(DEV), B.to(DEV))
    _, cbits = oracle_bf16(A, B)
    parity.assert_bits_equal_values(parity.bits(C), cbits, f"bf16 integers M={M}")


@pytest.mark.parametrize("M", EXACT_HEIGHT_M + [100, 127])
def test_exact_height_a_rows_fp8_bit_exact(M):
    qa, qb, sa, sb = fp8_case(M, 256, 1024, seed=4300 + M, integer=True)
    C = run_fp8(qa, qb, sa, sb)
    _, cbits = oracle.gemm_fp8_blockscaled(inputs.to_numpy_bits(qa), inputs.to_numpy_bits(qb),
                                           sa.numpy(), sb.numpy())
    parity.assert_bits_equal_values(parity.bits(C), cbits, f"fp8 integer M={M}")


@pytest.mark.parametrize("M", [1, 64, 4096])
def test_fp8_full_size_sampled_rows(M):
    N = K = 7168
    qa, qb, sa, sb = fp8_case(M, N, K, seed=4200 + M)
    C = run_fp8(qa, qb, sa, sb)
    rows = sorted({0, M - 1, M // 2, min(127, M - 1), min(128, M - 1)})
    cref, _ = oracle.gemm_fp8_rows(inputs.to_numpy_bits(qa), inputs.to_numpy_bits(qb),
                                   sa.numpy(), sb.numpy(), rows)
    parity.assert_within_tolerance(parity.bits(C)[rows], cref, K, fp8_rms(qa, sa, 1),
                                   fp8_rms(qb, sb, 128), f"fp8 full M={M}")


# ---------------------------------------------------------------------------------------------
# grouped (MoE)
# ---------------------------------------------------------------------------------------------

def run_grouped(A, B, offsets):
    E, N, K = B.shape
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_BF16, E)
    out = GuardedC(A.shape[0], N)
    bg.bi_grouped_gemm_run(plan, A, B, out.c, offsets.to(DEV))
    bg.bi_gemm_sync_status(plan)
    out.check()
    return out.c


@pytest.mark.parametrize("offsets", [
    [0, 0, 1, 130, 130, 257, 300],        # empty experts, segments of 1, 129, 127
    [0, 300, 300, 300, 300, 300, 300],    # everything on expert 0
    [0, 128, 256, 384, 385, 512, 600],    # segments aligned to the tile and one off
])
def test_grouped_small_within_tolerance(offsets):
    E = len(offsets) - 1
    R, N, K = offsets[-1], 96, 200
    A = inputs.bf16_gaussian((R, K), seed=5000 + R)
    B = inputs.bf16_gaussian((E, N, K), seed=5001)
    C = run_grouped(A.to(DEV), B.to(DEV), torch.tensor(offsets, dtype=torch.int32))
    cref, _ = oracle.grouped_gemm_bf16(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B),
                                       np.array(offsets, np.int32))
    parity.assert_within_tolerance(parity.bits(C), cref, K, parity.rms(A.float().numpy()),
                                   parity.rms(B.float().numpy()), f"grouped {offsets}")


def test_grouped_integers_bit_exact_wide_tile():
    offsets = [0, 5, 140, 140, 400]
    E, R, N, K = 4, 400, 12800, 64        # BN 128 through the fallback rule
    A = inputs.bf16_integers((R, K), seed=5100)
    B = inputs.bf16_integers((E, N, K), seed=5101)
    C = run_grouped(A.to(DEV), B.to(DEV), torch.tensor(offsets, dtype=torch.int32))
    _, cbits = oracle.grouped_gemm_bf16(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B),
                                        np.array(offsets, np.int32))
    parity.assert_bits_equal_values(parity.bits(C), cbits, "grouped integer")


@pytest.mark.parametrize("T", [1, 64, 1024, 8192])
def test_grouped_full_size_sampled_rows(T):
    E, N, K = 64, 2048, 7168
    routing = routing_mod.softmax_top8_routing(T, E, seed=5200 + T)
    tokens = inputs.bf16_gaussian((T, K), seed=5201 + T, device=DEV)
    B = inputs.bf16_gaussian((E, N, K), seed=5202, std=K ** -0.5, device=DEV)
    A = tokens[routing.token_of_row.to(DEV)].contiguous()
    C = run_grouped(A, B, routing.offsets)
    off = routing.offsets.numpy()
    Cb = parity.bits(C)
    rng = np.random.default_rng(T)
    experts = [e for e in range(E) if off[e + 1] > off[e]]
    rms_a, rms_b = parity.rms_t(A), parity.rms_t(B)
    for e in rng.choice(experts, size=min(3, len(experts)), replace=False):
        rows = sorted({int(off[e]), int(off[e + 1] - 1)})
        cref, _ = oracle.gemm_bf16(inputs.to_numpy_bits(A[rows]), inputs.to_numpy_bits(B[e]))
        parity.assert_within_tolerance(Cb[rows], cref, K, rms_a, rms_b, f"moe T={T} e={e}")


def test_run_host_matches_device_run():
    M, N, K = 100, 256, 512
    plan = bg.bi_gemm_plan(N, K)
    A = inputs.bf16_integers((M, K), seed=6001).pin_memory()
    B = inputs.bf16_integers((N, K), seed=6002, device=DEV)
    C_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    A_dev = torch.empty((M, K), dtype=torch.bfloat16, device=DEV)
    C_dev = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    bg.bi_gemm_run_host(plan, A, B, C_host, A_dev, C_dev)
    bg.bi_gemm_sync_status(plan)
    _, want = oracle.gemm_bf16(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B))
    parity.assert_bits_equal_values(parity.bits(C_host), want, "run_host")
