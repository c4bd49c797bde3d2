"""bi_gemm_run_host_noalloc: the host-buffer GEMM for callers that cannot allocate device memory
(their GPU memory belongs to another allocator, such as a framework's caching allocator or an
inference server's arena, or allocating after start-up is not allowed).  It stages A, scale_a
and C in the library's static device scratch instead of caller or cudaMalloc buffers.

Each case runs the entry point twice in a row through the C ABI and compares both results with
the existing device entry point bi_gemm_run on the same inputs.  Batch invariance makes the
expected agreement bitwise; the tolerance of the other parity tests is checked as well.  This
file is collected last so that a stop at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
from invariant_deterministic_gemm_bi_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"


def device_reference(plan, A, B, scale_a_kb=None, scale_b=None):
    C = torch.empty((A.shape[0], B.shape[0]), dtype=torch.bfloat16, device=DEV)
    bg.bi_gemm_run(plan, A.to(DEV), B, C, scale_a=None if scale_a_kb is None else scale_a_kb.to(DEV),
                   scale_b=scale_b)
    bg.bi_gemm_sync_status(plan)
    return C.cpu()


@pytest.mark.parametrize("M,N,K", [(64, 4096, 7168), (300, 256, 512), (1, 40, 72)])
def test_noalloc_bf16_matches_device_entry_point_twice(M, N, K):
    plan = bg.bi_gemm_plan(N, K)
    A = inputs.bf16_gaussian((M, K), seed=9000 + M).pin_memory()
    B = inputs.bf16_gaussian((N, K), seed=9001, std=K ** -0.5, device=DEV)
    want = device_reference(plan, A, B)
    for call in range(2):
        C = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
        bg.bi_gemm_run_host_noalloc(plan, A, B, C)
        assert torch.equal(C.view(torch.int16), want.view(torch.int16)), f"call {call}"
        parity.assert_within_tolerance(parity.bits(C), parity.bf16_bits_to_f64(parity.bits(want)),
                                       K, 1.0, K ** -0.5, f"noalloc call {call}")


def test_noalloc_fp8_matches_device_entry_point_twice():
    M, N, K = 96, 512, 1024
    KB = K // 128
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    qa = inputs.e4m3_gaussian((M, K), seed=9100)
    qb = inputs.e4m3_gaussian((N, K), seed=9101, device=DEV)
    sa = inputs.scales_log_uniform((KB, M), seed=9102)          # K-block-major, ld_sa = M
    sb = inputs.scales_log_uniform((N // 128, KB), seed=9103, device=DEV)
    want = device_reference(plan, qa, qb, sa, sb)
    qa_h, sa_h = qa.pin_memory(), sa.pin_memory()
    for call in range(2):
        C = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
        bg.bi_gemm_run_host_noalloc(plan, qa_h, qb, C, scale_a_host=sa_h, scale_b=sb)
        assert torch.equal(C.view(torch.int16), want.view(torch.int16)), f"call {call}"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    N, K = 4096, 7168
    plan = bg.bi_gemm_plan(N, K)
    B = torch.zeros((N, K), dtype=torch.bfloat16, device=DEV)
    A = torch.zeros((373, K), dtype=torch.bfloat16)            # 373 rows need > 8 MiB
    C = torch.zeros((373, N), dtype=torch.bfloat16)
    with pytest.raises(bg.BiGemmError) as e:
        bg.bi_gemm_run_host_noalloc(plan, A, B, C)
    assert e.value.name == "BI_ERR_UNSUPPORTED_SHAPE"
    # the largest size that fits still runs
    A = inputs.bf16_integers((372, K), seed=1).pin_memory()
    C = torch.empty((372, N), dtype=torch.bfloat16).pin_memory()
    Bi = inputs.bf16_integers((N, K), seed=2, device=DEV)
    bg.bi_gemm_run_host_noalloc(plan, A, Bi, C)
    want = device_reference(plan, A, Bi)
    assert torch.equal(C.view(torch.int16), want.view(torch.int16))


def test_noalloc_allocates_no_device_memory():
    """After a warmed-up call, further calls leave the device's free memory unchanged: the staging
    copies live in the library's static scratch, never in a new allocation."""
    M, N, K = 64, 4096, 7168
    plan = bg.bi_gemm_plan(N, K)
    A = inputs.bf16_gaussian((M, K), seed=9200).pin_memory()
    B = inputs.bf16_gaussian((N, K), seed=9201, std=K ** -0.5, device=DEV)
    C = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    bg.bi_gemm_run_host_noalloc(plan, A, B, C)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        bg.bi_gemm_run_host_noalloc(plan, A, B, C)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_empty_contraction_writes_zeros_twice():
    M, N = 5, 256
    plan = bg.bi_gemm_plan(N, 0)
    A = torch.empty((M, 0), dtype=torch.bfloat16)
    B = torch.empty((N, 0), dtype=torch.bfloat16, device=DEV)
    want = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    bg.bi_gemm_run(plan, A.to(DEV), B, want)
    bg.bi_gemm_sync_status(plan)
    for call in range(2):
        C = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
        bg.bi_gemm_run_host_noalloc(plan, A, B, C)
        assert torch.equal(C.view(torch.int16), want.cpu().view(torch.int16)), f"call {call}"
        assert not C.float().abs().sum().item()


def test_noalloc_padded_pitches_match_device_entry_point():
    """lda > K for bf16, and an FP8 scale_a whose K-block pitch ld_sa exceeds M."""
    M, N, K = 40, 512, 1024
    plan = bg.bi_gemm_plan(N, K)
    Apad = inputs.bf16_gaussian((M, K + 64), seed=9300)
    A = Apad[:, :K]                                              # lda = K + 64
    B = inputs.bf16_gaussian((N, K), seed=9301, std=K ** -0.5, device=DEV)
    want = device_reference(plan, A.contiguous(), B)
    for call in range(2):
        C = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
        bg.bi_gemm_run_host_noalloc(plan, A, B, C)
        assert torch.equal(C.view(torch.int16), want.view(torch.int16)), f"bf16 call {call}"

    KB = K // 128
    p8 = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    qa = inputs.e4m3_gaussian((M, K), seed=9310)
    qb = inputs.e4m3_gaussian((N, K), seed=9311, device=DEV)
    sa_wide = inputs.scales_log_uniform((KB, M + 24), seed=9312)   # ld_sa = M + 24
    sb = inputs.scales_log_uniform((N // 128, KB), seed=9313, device=DEV)
    want8 = device_reference(p8, qa, qb, sa_wide[:, :M].contiguous(), sb)
    sa_view = sa_wide.pin_memory()[:, :M]
    for call in range(2):
        C = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
        bg.bi_gemm_run_host_noalloc(p8, qa.pin_memory(), qb, C, scale_a_host=sa_view, scale_b=sb)
        assert torch.equal(C.view(torch.int16), want8.view(torch.int16)), f"fp8 call {call}"
