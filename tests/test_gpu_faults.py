"""GPU failure paths that fault nothing: bounded waits that run out, malformed offsets, bad args.

The timeout test sets a test-only flag that makes every CTA's producer skip its first operand
load, so the MMA warp's first wait can never complete.  The wait's 20 ms limit runs out, the
kernel records BI_ERR_DEVICE_TIMEOUT, drains its own copies, frees its tensor memory and
returns; the context stays usable and the next call is correct.
"""
import numpy as np
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
import oracle
from invariant_deterministic_gemm_bi_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"


# (256, 512, FP8): two warps issue alternate K chunks; (4096, 512, bf16) at M = 256: 256 tiles run
# in the wide lockstep form, two warps issuing one column half each
@pytest.mark.parametrize("M,N,K,dtype", [(64, 256, 512, bg.BI_DTYPE_BF16),
                                         (64, 256, 512, bg.BI_DTYPE_E4M3_BLOCKSCALED),
                                         (256, 4096, 512, bg.BI_DTYPE_BF16)])
def test_wait_timeout_is_reported_and_context_survives(M, N, K, dtype):
    plan = bg.bi_gemm_plan(N, K, dtype, 1)
    if dtype == bg.BI_DTYPE_BF16:
        A = inputs.bf16_integers((M, K), seed=1, device=DEV)
        B = inputs.bf16_integers((N, K), seed=2, device=DEV)
        sa = sb = None
    else:
        A = inputs.e4m3_integers((M, K), seed=1, device=DEV)
        B = inputs.e4m3_integers((N, K), seed=2, device=DEV)
        sa = torch.ones((K // 128, M), dtype=torch.float32, device=DEV)
        sb = torch.ones((N // 128, K // 128), dtype=torch.float32, device=DEV)
    C = torch.zeros((M, N), dtype=torch.bfloat16, device=DEV)
    bg.bi_gemm_set_wait_timeout(plan, 20_000_000)          # 20 ms
    bg.bi_gemm_debug_set_flags(plan, bg.BI_DEBUG_SKIP_FIRST_LOAD)
    bg.bi_gemm_run(plan, A, B, C, scale_a=sa, scale_b=sb)
    st = bg.bi_gemm_sync_status(plan, raise_on_error=False)
    assert bg.binding.STATUS_NAMES[st] == "BI_ERR_DEVICE_TIMEOUT"
    # the status word was cleared and the same plan now computes correctly
    bg.bi_gemm_debug_set_flags(plan, 0)
    bg.bi_gemm_set_wait_timeout(plan, 0)
    bg.bi_gemm_run(plan, A, B, C, scale_a=sa, scale_b=sb)
    assert bg.bi_gemm_sync_status(plan) == 0
    if dtype == bg.BI_DTYPE_BF16:
        _, want = oracle.gemm_bf16(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B))
    else:
        _, want = oracle.gemm_fp8_blockscaled(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B),
                                              np.ones((M, K // 128), np.float32),
                                              np.ones((N // 128, K // 128), np.float32))
    parity.assert_bits_equal_values(parity.bits(C), want, "after timeout")


@pytest.mark.parametrize("offsets", [[0, 5, 3, 8], [1, 2, 3, 8], [0, 2, 3, 7]])
def test_malformed_offsets_are_rejected_on_device(offsets):
    E, N, K, R = 3, 64, 64, 8
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_BF16, E)
    A = inputs.bf16_gaussian((R, K), seed=3, device=DEV)
    B = inputs.bf16_gaussian((E, N, K), seed=4, device=DEV)
    C = torch.full((R, N), 7.0, dtype=torch.bfloat16, device=DEV)
    bg.bi_grouped_gemm_run(plan, A, B, C, torch.tensor(offsets, dtype=torch.int32, device=DEV))
    st = bg.bi_gemm_sync_status(plan, raise_on_error=False)
    assert bg.binding.STATUS_NAMES[st] == "BI_ERR_BAD_OFFSETS"
    assert torch.all(C.float() == 7.0), "nothing may be computed on malformed offsets"


def test_misaligned_and_mismatched_arguments_are_rejected_before_launch():
    plan = bg.bi_gemm_plan(64, 64)
    A = torch.zeros((4, 72), dtype=torch.bfloat16, device=DEV)
    B = torch.zeros((64, 64), dtype=torch.bfloat16, device=DEV)
    C = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(bg.BiGemmError) as e:
        bg.bi_gemm_run(plan, A[:, 1:65], B, C)              # A not 16-byte aligned
    assert e.value.name == "BI_ERR_ALIGNMENT"
    with pytest.raises(bg.BiGemmError) as e:
        bg.bi_gemm_run(plan, A[:, :64], B, C, scale_b=torch.ones(1, device=DEV))
    assert e.value.name == "BI_ERR_DTYPE_MISMATCH"
    fp8 = bg.bi_gemm_plan(64, 128, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    qa = torch.zeros((4, 128), dtype=torch.uint8, device=DEV)
    qb = torch.zeros((64, 128), dtype=torch.uint8, device=DEV)
    with pytest.raises(bg.BiGemmError) as e:
        bg.bi_gemm_run(fp8, qa, qb, C)                      # FP8 without scales
    assert e.value.name == "BI_ERR_DTYPE_MISMATCH"
    grouped = bg.bi_gemm_plan(64, 64, bg.BI_DTYPE_BF16, 4)
    with pytest.raises(bg.BiGemmError) as e:
        bg.bi_gemm_run(grouped, A[:, :64], B, C)            # grouped plan on the dense entry
    assert e.value.name == "BI_ERR_INVALID_ARG"
    torch.cuda.synchronize()
