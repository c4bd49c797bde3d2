"""The fixed-split-K research variant (bi_gemm_plan_splitk): parity with the oracle, and bitwise
M-invariance, because its split points and merge order are fixed by (N, K, splits).  It is not
the product path; its rows differ from the product plan's rows within the tolerance."""
import numpy as np
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
import oracle
from invariant_deterministic_gemm_bi_b200 import inputs
from tests import parity
from tests.gpu_util import GuardedC

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_splitk(plan, A, N):
    M = A.shape[0]
    out = GuardedC(M, N)
    ws = torch.empty(max(1, bg.bi_gemm_splitk_workspace_bytes(plan, M) // 4), dtype=torch.float32, device=DEV)
    return out, ws


def splitk(plan, A, B, out, ws):
    bg.bi_gemm_run_splitk(plan, A, B, out.c, ws)
    bg.bi_gemm_sync_status(plan)
    out.check()
    return out.c


@pytest.mark.parametrize("splits", [2, 4, 8])
@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (37, 384, 2112), (130, 4096, 7168)])
def test_splitk_integers_bit_exact(splits, M, N, K):
    A = inputs.bf16_integers((M, K), seed=3100 + M, device=DEV)
    B = inputs.bf16_integers((N, K), seed=3101 + N, device=DEV)
    plan = bg.bi_gemm_plan_splitk(N, K, splits)
    out, ws = run_splitk(plan, A, N)
    C = splitk(plan, A, B, out, ws)
    rows = sorted({0, M - 1, M // 2, min(127, M - 1), min(128, M - 1)})
    _, cbits = oracle.gemm_bf16_rows(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B), rows)
    parity.assert_bits_equal_values(parity.bits(C)[rows], cbits, f"split-K {splits} {M}x{N}x{K}")


@pytest.mark.parametrize("splits", [2, 4, 8])
def test_splitk_gaussian_within_tolerance(splits):
    M, N, K = 64, 4096, 7168
    A = inputs.bf16_gaussian((M, K), seed=3200, device=DEV)
    B = inputs.bf16_gaussian((N, K), seed=3201, std=K ** -0.5, device=DEV)
    plan = bg.bi_gemm_plan_splitk(N, K, splits)
    out, ws = run_splitk(plan, A, N)
    C = splitk(plan, A, B, out, ws)
    rows = [0, 1, 31, 63]
    cref, _ = oracle.gemm_bf16_rows(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B), rows)
    parity.assert_within_tolerance(parity.bits(C)[rows], cref, K, parity.rms_t(A), parity.rms_t(B),
                                   f"split-K {splits} decode")


def test_splitk_rows_invariant_across_m():
    N, K = 4096, 7168
    B = inputs.bf16_gaussian((N, K), seed=3301, std=K ** -0.5, device=DEV)
    plan = bg.bi_gemm_plan_splitk(N, K, 4)
    test_rows = inputs.bf16_gaussian((16, K), seed=3302, device=DEV)
    ref = []
    for i in range(16):
        out, ws = run_splitk(plan, test_rows[i:i + 1], N)
        ref.append(splitk(plan, test_rows[i:i + 1].contiguous(), B, out, ws).view(torch.int16).clone())
    ref = torch.cat(ref)
    rng = np.random.default_rng(3303)
    for M in [2, 16, 64, 128, 256, 300]:
        batch = inputs.bf16_gaussian((M, K), seed=3304 + M, device=DEV)
        k = min(16, M)
        pos = rng.choice(M, size=k, replace=False)
        batch[torch.from_numpy(pos).to(DEV)] = test_rows[:k]
        out, ws = run_splitk(plan, batch, N)
        C = splitk(plan, batch, B, out, ws).view(torch.int16)
        bad = (C[torch.from_numpy(pos).to(DEV)] != ref[:k]).any(dim=1)
        assert not bad.any(), f"M={M}: {int(bad.sum())} rows differ from their M=1 bits"
