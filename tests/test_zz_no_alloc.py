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
