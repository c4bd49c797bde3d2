"""bi_gemm_run_host_batch: host-buffer GEMMs pipelined behind the ABI (copy-in, kernel and
copy-out on three streams, one staging region per batch reused in turn, a batch's copy-outs
enqueued two batches later or by a flush, calls whose host rows follow one another moved with
one copy).

Each batch's results must equal the same GEMMs run by bi_gemm_run on device buffers, bit for bit
(batch invariance: a row's bits do not depend on which call, region or stream carried it), and the
integer variant must match the oracle exactly.  Consecutive batches reuse the regions without any
synchronisation in between, and a change of staging buffer mid-stream must still order every
copy correctly.
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


def device_run(plan, A, B, scale_a=None, scale_b=None):
    C = torch.empty((A.shape[0], B.shape[0]), dtype=torch.bfloat16, device=DEV)
    bg.bi_gemm_run(plan, A.to(DEV), B, C, scale_a=None if scale_a is None else scale_a.to(DEV),
                   scale_b=scale_b)
    bg.bi_gemm_sync_status(plan)
    return C.cpu()


def test_batches_match_device_runs_and_the_oracle():
    N, K = 4096, 7168
    plan = bg.bi_gemm_plan(N, K)
    Bs = [inputs.bf16_integers((N, K), seed=5301 + i, device=DEV) for i in range(2)]
    Ms = [1, 3, 0, 17, 64, 200, 8]
    cin, cmp, cout = (torch.cuda.Stream() for _ in range(3))
    batches = []
    for b in range(4):
        calls, want = [], []
        for i, M in enumerate(Ms):
            A = inputs.bf16_integers((M, K), seed=5400 + 31 * b + i).pin_memory()
            C = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
            calls.append((A, Bs[(b + i) % 2], C))
        batches.append(calls)
    need = bg.bi_gemm_host_batch_staging_bytes(plan, batches[0], 3)
    staging = [torch.empty(need, dtype=torch.uint8, device=DEV) for _ in range(2)]
    torch.cuda.synchronize()
    for b, calls in enumerate(batches):   # no synchronisation between batches; staging changes at b = 2
        bg.bi_gemm_run_host_batch(plan, calls, staging[b // 2], copy_in=cin, compute=cmp, copy_out=cout)
    bg.bi_gemm_host_batch_flush(plan, copy_in=cin, compute=cmp, copy_out=cout)
    cout.synchronize()
    bg.bi_gemm_sync_status(plan, stream=cmp)
    for b, calls in enumerate(batches):
        for i, (A, B, C) in enumerate(calls):
            if A.shape[0] == 0:
                continue
            ref = device_run(plan, A, B)
            assert torch.equal(C.view(torch.int16), ref.view(torch.int16)), f"batch {b} call {i}"
            _, cb = oracle.gemm_bf16_exact_integers(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B))
            parity.assert_bits_equal_values(parity.bits(C), cb, f"batch {b} call {i}")


def test_fp8_batch_matches_device_runs():
    M0, N, K = 48, 512, 1024
    KB = K // 128
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    qb = inputs.e4m3_gaussian((N, K), seed=5501, device=DEV)
    sb = inputs.scales_log_uniform((N // 128, KB), seed=5502, device=DEV)
    calls = []
    for i, M in enumerate([M0, 5, 130]):
        qa = inputs.e4m3_gaussian((M, K), seed=5510 + i).pin_memory()
        sa = inputs.scales_log_uniform((KB, M), seed=5520 + i).pin_memory()   # K-block-major
        C = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
        calls.append((qa, qb, C, sa, sb))
    staging = torch.empty(bg.bi_gemm_host_batch_staging_bytes(plan, calls), dtype=torch.uint8, device=DEV)
    s = torch.cuda.Stream()
    bg.bi_gemm_run_host_batch(plan, calls, staging, copy_in=s, compute=s, copy_out=s)
    bg.bi_gemm_host_batch_flush(plan, copy_in=s, compute=s, copy_out=s)
    s.synchronize()
    for i, (qa, qb_, C, sa, sb_) in enumerate(calls):
        ref = device_run(plan, qa, qb_, scale_a=sa, scale_b=sb_)
        assert torch.equal(C.view(torch.int16), ref.view(torch.int16)), f"call {i}"


def test_batches_captured_in_a_graph_match_device_runs():
    """Under stream capture a batch forks its copy streams from the compute stream and joins them
    back; replays of a graph holding two batches give the same bits as direct runs."""
    N, K = 256, 512
    plan = bg.bi_gemm_plan(N, K)
    B = inputs.bf16_gaussian((N, K), seed=5601, device=DEV)
    Ms = [1, 9, 64, 130]
    batches = []
    for b in range(2):
        calls = []
        for i, M in enumerate(Ms):
            A = inputs.bf16_gaussian((M, K), seed=5610 + 7 * b + i).pin_memory()
            C = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
            calls.append((A, B, C))
        batches.append(calls)
    staging = torch.empty(bg.bi_gemm_host_batch_staging_bytes(plan, batches[0], 3), dtype=torch.uint8,
                          device=DEV)
    cin, cout, cap = (torch.cuda.Stream() for _ in range(3))
    for calls in batches:   # once outside capture (first-use set-up)
        bg.bi_gemm_run_host_batch(plan, calls, staging, copy_in=cin, compute=cap, copy_out=cout)
    bg.bi_gemm_host_batch_flush(plan, copy_in=cin, compute=cap, copy_out=cout)
    torch.cuda.synchronize()
    for calls in batches:
        for _, _, C in calls:
            C.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for calls in batches:
            bg.bi_gemm_run_host_batch(plan, calls, staging, copy_in=cin, compute=cap, copy_out=cout)
        bg.bi_gemm_host_batch_flush(plan, copy_in=cin, compute=cap, copy_out=cout)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for b, calls in enumerate(batches):
        for i, (A, B_, C) in enumerate(calls):
            ref = device_run(plan, A, B_)
            assert torch.equal(C.view(torch.int16), ref.view(torch.int16)), f"batch {b} call {i}"
    del g


def test_back_to_back_host_rows_share_copies_and_match_device_runs():
    """With BI_PLAN_HOST_ROW_BLOCKS a batch whose A (and C) slices lie back to back in one pinned
    block moves them with one copy each way; interleaved with batches whose slices do not (and
    whose staging region therefore has another size), every result still equals the device run
    bit for bit."""
    N, K = 4096, 7168
    plan = bg.bi_gemm_plan(N, K)
    bg.bi_gemm_plan_set_flags(plan, bg.BI_PLAN_HOST_ROW_BLOCKS)   # each block is one allocation
    B = inputs.bf16_gaussian((N, K), seed=5701, std=K ** -0.5, device=DEV)
    Ms = [1, 2, 4, 8, 16, 32, 64, 128, 256]
    offs = np.concatenate([[0], np.cumsum(Ms)])
    blocks = []
    for b in range(3):
        A = inputs.bf16_gaussian((int(offs[-1]), K), seed=5710 + b).pin_memory()
        C = torch.full((int(offs[-1]), N), float("nan"), dtype=torch.bfloat16).pin_memory()
        blocks.append((A, C))
    def calls_of(b, adjacent):
        A, C = blocks[b]
        if adjacent:
            return [(A[offs[i]:offs[i + 1]], B, C[offs[i]:offs[i + 1]]) for i in range(len(Ms))]
        # the same slices in reverse call order: no call's rows follow the previous call's
        return [(A[offs[i]:offs[i + 1]], B, C[offs[i]:offs[i + 1]]) for i in reversed(range(len(Ms)))]
    batches = [calls_of(0, True), calls_of(1, False), calls_of(2, True)]
    need = max(bg.bi_gemm_host_batch_staging_bytes(plan, c, 3) for c in batches)
    staging = torch.empty(need, dtype=torch.uint8, device=DEV)
    cin, cmp, cout = (torch.cuda.Stream() for _ in range(3))
    torch.cuda.synchronize()
    for calls in batches:
        bg.bi_gemm_run_host_batch(plan, calls, staging, copy_in=cin, compute=cmp, copy_out=cout)
    bg.bi_gemm_host_batch_flush(plan, copy_in=cin, compute=cmp, copy_out=cout)
    cout.synchronize()
    bg.bi_gemm_sync_status(plan, stream=cmp)
    for b, calls in enumerate(batches):
        for i, (A, B_, C) in enumerate(calls):
            ref = device_run(plan, A, B_)
            assert torch.equal(C.view(torch.int16), ref.view(torch.int16)), f"batch {b} call {i}"

