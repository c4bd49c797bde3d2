"""Stream order across back-to-back launches.

Every launch is a programmatic dependent of the previous kernel in its stream: it may start and
set up its shared and tensor memory while that kernel is finishing, and must not read or write
global memory before that kernel has completed.  These tests launch chains in which each GEMM
reads the previous one's output (read after write) or overwrites a buffer the previous one
reads (write after read), with no synchronisation between the launches, and require the results
to be bit-identical to the same launches separated by device synchronisations -- with and
without BI_PLAN_RESIDENT_WEIGHTS, which lets a launch request B before the previous kernel ends.
"""
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
from invariant_deterministic_gemm_bi_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (N, K) of a chain whose outputs feed the next GEMM's A: 7168 -> 2048 -> 7168 -> 4096
CHAIN = [(2048, 7168), (7168, 2048), (4096, 7168)]


def _weights(seed):
    return [inputs.bf16_gaussian((N, K), seed=seed + i, std=K ** -0.5, device=DEV)
            for i, (N, K) in enumerate(CHAIN)]


def _chain(plans, Bs, A0, outs, sync):
    a = A0
    for plan, B, C in zip(plans, Bs, outs):
        bg.bi_gemm_run(plan, a, B, C)
        if sync:
            torch.cuda.synchronize()
        a = C
    return outs


def _plan(N, K, resident):
    plan = bg.bi_gemm_plan(N, K)
    if resident:
        bg.bi_gemm_plan_set_flags(plan, bg.BI_PLAN_RESIDENT_WEIGHTS)
    return plan


@pytest.mark.parametrize("resident", [False, True])
@pytest.mark.parametrize("M", [1, 64, 512])
def test_chained_gemms_read_after_write(M, resident):
    plans = [_plan(N, K, resident) for N, K in CHAIN]
    Bs = _weights(9100)
    A0 = inputs.bf16_gaussian((M, CHAIN[0][1]), seed=9000 + M, device=DEV)
    ref = [torch.empty((M, N), dtype=torch.bfloat16, device=DEV) for N, _ in CHAIN]
    _chain(plans, Bs, A0, ref, sync=True)
    got = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV) for N, _ in CHAIN]
    for rep in range(20):
        for g in got:
            g.fill_(float("nan"))
        torch.cuda.synchronize()
        _chain(plans, Bs, A0, got, sync=False)
        torch.cuda.synchronize()
        for i, (r, g) in enumerate(zip(ref, got)):
            assert torch.equal(r.view(torch.int16), g.view(torch.int16)), (
                f"M={M} rep {rep}: GEMM {i} of the chain differs from the synchronised run")
    for plan in plans:
        bg.bi_gemm_sync_status(plan)


@pytest.mark.parametrize("M", [1, 17, 64, 300])
def test_resident_weights_flag_changes_no_bits(M):
    N, K = 4096, 7168
    B = inputs.bf16_gaussian((N, K), seed=9300, std=K ** -0.5, device=DEV)
    A = inputs.bf16_gaussian((M, K), seed=9301 + M, device=DEV)
    outs = []
    for resident in (False, True):
        plan = _plan(N, K, resident)
        C = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        bg.bi_gemm_run(plan, A, B, C)
        bg.bi_gemm_sync_status(plan)
        outs.append(C.view(torch.int16))
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("resident", [False, True])
@pytest.mark.parametrize("M", [1, 64, 512])
def test_overwrite_of_previous_input_waits(M, resident):
    # GEMM 1 reads X; GEMM 2, launched right after, writes its output into X's buffer.
    N1, K = 2048, 7168
    p1 = _plan(N1, K, resident)
    p2 = _plan(K, 2048, resident)      # output rows of width K = 7168 land in X
    B1 = inputs.bf16_gaussian((N1, K), seed=9200, std=K ** -0.5, device=DEV)
    B2 = inputs.bf16_gaussian((K, 2048), seed=9201, std=2048 ** -0.5, device=DEV)
    X0 = inputs.bf16_gaussian((M, K), seed=9202 + M, device=DEV)
    Y = inputs.bf16_gaussian((M, 2048), seed=9203 + M, device=DEV)
    ref1 = torch.empty((M, N1), dtype=torch.bfloat16, device=DEV)
    bg.bi_gemm_run(p1, X0, B1, ref1)
    ref2 = torch.empty((M, K), dtype=torch.bfloat16, device=DEV)
    bg.bi_gemm_run(p2, Y, B2, ref2)
    torch.cuda.synchronize()
    for rep in range(20):
        X = X0.clone()
        C1 = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device=DEV)
        torch.cuda.synchronize()
        bg.bi_gemm_run(p1, X, B1, C1)
        bg.bi_gemm_run(p2, Y, B2, X)   # overwrites GEMM 1's input
        torch.cuda.synchronize()
        assert torch.equal(C1.view(torch.int16), ref1.view(torch.int16)), (
            f"M={M} rep {rep}: GEMM 1 read part of its input after GEMM 2 overwrote it")
        assert torch.equal(X.view(torch.int16), ref2.view(torch.int16)), f"M={M} rep {rep}"
    bg.bi_gemm_sync_status(p1)
    bg.bi_gemm_sync_status(p2)
