"""GPU tests of the e2m1-weight x e4m3-activation GEMM (bi_gemm_run_w4a8) against the oracle.

The weights follow "DeepSeek V4的batch invariance：大模型确定性推理的工程基石" (lshu.cn), section
4.3: W = q * scale + zero per output channel, scale in {2^-j : j = 1..12}, zero fp16-exact.
On inputs whose every partial sum is exact in fp32 (integer activations, power-of-two scales,
zero points on a 2^-6 grid) the kernel must match the oracle's bf16 bits exactly; on Gaussian
activations it must stay within the elementwise tolerance.  Rows must be bitwise independent of
M, of their position and of their batch-mates, in every scheduling form of the plan.
"""
import numpy as np
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
import oracle
from invariant_deterministic_gemm_bi_b200 import inputs
from tests import parity
from tests.gpu_util import GuardedC, kblock_major_scales, strided_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"
W4 = bg.BI_DTYPE_E2M1_W4A8

_PLANS = {}


def plan_for(N, K):
    if (N, K) not in _PLANS:
        _PLANS[(N, K)] = bg.bi_gemm_plan(N, K, W4)
    return _PLANS[(N, K)]


def case(M, N, K, seed, integer=False, zero=True):
    KB = K // 128
    if integer:
        qa = inputs.e4m3_integers((M, K), seed)
        sa = inputs.scales_pow2((M, KB), seed + 1, lo=-2, hi=2)
        ws = inputs.channel_scales_pow2(N, seed + 3, lo=1, hi=4)
        wz = inputs.channel_zeros_grid(N, seed + 4) if zero else None
    else:
        qa = inputs.e4m3_gaussian((M, K), seed)
        sa = inputs.scales_log_uniform((M, KB), seed + 1)
        ws = inputs.channel_scales_pow2(N, seed + 3)
        wz = inputs.channel_zeros_fp16(ws, seed + 4) if zero else None
    qw = inputs.e2m1_packed_uniform(N, K, seed + 2)
    return qa, sa, qw, ws, wz


def run(qa, sa, qw, ws, wz, plan=None, ldw_extra=0, guarded=True):
    M, K = qa.shape
    N = qw.shape[0]
    plan = plan or plan_for(N, K)
    A = qa.to(DEV)
    W = strided_rows(qw.to(DEV), K // 2 + ldw_extra // 2) if ldw_extra else qw.to(DEV).contiguous()
    sa_d = kblock_major_scales(sa.to(DEV))
    ws_d = ws.to(DEV).contiguous()
    wz_d = wz.to(DEV).contiguous() if wz is not None else None
    work = torch.empty(max(bg.bi_gemm_w4a8_workspace_bytes(M) // 4, 1), dtype=torch.float32, device=DEV)
    g = GuardedC(M, N)
    bg.bi_gemm_run_w4a8(plan, A, sa_d, W, ws_d, g.c, w_zero=wz_d, workspace=work)
    st = bg.bi_gemm_sync_status(plan, raise_on_error=False)
    assert st == 0, bg.bi_status_string(st)
    if guarded:
        g.check()
    return g.c


def dequant_rms(qa, sa, qw, ws, wz):
    a = parity.e4m3_bits_to_f64(inputs.to_numpy_bits(qa)) * np.repeat(sa.numpy().astype(np.float64), 128, axis=1)
    codes = np.empty((qw.shape[0], qw.shape[1] * 2), np.uint8)
    q = qw.numpy()
    codes[:, 0::2], codes[:, 1::2] = q & 0xF, q >> 4
    vals = oracle.e2m1_to_f64(np.arange(16, dtype=np.uint8))[codes]
    w = vals * ws.numpy().astype(np.float64)[:, None]
    if wz is not None:
        w = w + wz.numpy().astype(np.float64)[:, None]
    return parity.rms(a), parity.rms(w)


def oracle_of(qa, sa, qw, ws, wz, rows=None):
    args = (inputs.to_numpy_bits(qa), sa.numpy(), qw.numpy(), ws.numpy(),
            None if wz is None else wz.numpy())
    if rows is None:
        return oracle.gemm_w4a8(*args)
    return oracle.gemm_w4a8_rows(*args[:4], args[4], rows)


@pytest.mark.parametrize("M,N,K,zero", [(1, 256, 512, True), (3, 256, 512, False), (17, 200, 384, True),
                                        (64, 256, 512, True), (100, 330, 512, False),
                                        (300, 256, 256, True), (130, 6400, 256, True),
                                        (200, 6432, 384, False)])
def test_integers_bit_exact(M, N, K, zero):
    qa, sa, qw, ws, wz = case(M, N, K, seed=6000 + M + N, integer=True, zero=zero)
    C = run(qa, sa, qw, ws, wz)
    _, cbits = oracle_of(qa, sa, qw, ws, wz)
    parity.assert_bits_equal_values(parity.bits(C), cbits, f"w4a8 integer {M}x{N}x{K} zero={zero}")


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (64, 256, 512), (129, 300, 384), (130, 6400, 256)])
def test_gaussian_within_tolerance(M, N, K):
    qa, sa, qw, ws, wz = case(M, N, K, seed=6100 + M + N)
    C = run(qa, sa, qw, ws, wz)
    cref, _ = oracle_of(qa, sa, qw, ws, wz)
    ra, rw = dequant_rms(qa, sa, qw, ws, wz)
    parity.assert_within_tolerance(parity.bits(C), cref, K, ra, rw, f"w4a8 {M}x{N}x{K}")


def test_strided_weights_and_no_zero_points_match():
    M, N, K = 40, 256, 512
    qa, sa, qw, ws, wz = case(M, N, K, seed=6200, integer=True)
    C1 = run(qa, sa, qw, ws, wz)
    C2 = run(qa, sa, qw, ws, wz, ldw_extra=128)       # W row pitch K + 128 values
    assert torch.equal(parity_bits(C1), parity_bits(C2))
    # all-zero zero points give the values of the no-zero-point path
    C3 = run(qa, sa, qw, ws, torch.zeros_like(ws))
    C4 = run(qa, sa, qw, ws, None)
    assert torch.equal(C3.float(), C4.float())


def parity_bits(t):
    return t.view(torch.int16)


@pytest.mark.parametrize("M", [1, 64, 2048])
def test_full_size_sampled_rows(M):
    N = K = 7168
    qa, sa, qw, ws, wz = case(M, N, K, seed=6300 + M)
    C = run(qa, sa, qw, ws, wz, guarded=False)
    rows = sorted({0, M - 1, M // 2, min(127, M - 1), min(128, M - 1)})
    cref, _ = oracle_of(qa, sa, qw, ws, wz, rows)
    ra, rw = dequant_rms(qa[rows], sa[rows], qw, ws, wz)
    parity.assert_within_tolerance(parity.bits(C)[rows], cref, K, ra, rw, f"w4a8 full M={M}")


def test_rows_invariant_across_m_and_scheduling_forms():
    # N = K = 7168: M <= 64 takes the small-batch form, M <= 128*148/56 the plan's form and larger
    # batches the wide lockstep form; a row must come out the same in all of them
    N = K = 7168
    plan = plan_for(N, K)
    base = 6400
    qa_t, sa_t, qw, ws, wz = case(16, N, K, seed=base)
    ref = run(qa_t, sa_t, qw, ws, wz, plan, guarded=False)
    for M in (1, 7, 64, 65, 200, 1000, 4096):
        qa, sa, _, _, _ = case(M, N, K, seed=base + 17 * M + 1)
        g = torch.Generator().manual_seed(M)
        pos = torch.randperm(M, generator=g)[: min(16, M)]
        qa = qa.clone()
        sa = sa.clone()
        qa[pos] = qa_t[: len(pos)]
        sa[pos] = sa_t[: len(pos)]
        C = run(qa, sa, qw, ws, wz, plan, guarded=False)
        for i, p in enumerate(pos.tolist()):
            assert torch.equal(C[p].view(torch.int16), ref[i].view(torch.int16)), (M, p)


def test_bad_scale_or_zero_is_reported():
    M, N, K = 8, 256, 512
    plan = bg.bi_gemm_plan(N, K, W4)
    for bad in ("scale3", "scale_big", "scale_small", "zero_inexact"):
        qa, sa, qw, ws, wz = case(M, N, K, seed=6500, integer=True)
        ws, wz = ws.clone(), wz.clone()
        if bad == "scale3":
            ws[5] = 0.375
        elif bad == "scale_big":
            ws[7] = 1.0
        elif bad == "scale_small":
            ws[9] = 2.0 ** -13
        else:
            wz[11] = 1.0 + 2.0 ** -12
        A, W = qa.to(DEV), qw.to(DEV)
        C = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
        work = torch.empty(64, dtype=torch.float32, device=DEV)
        bg.bi_gemm_run_w4a8(plan, A, kblock_major_scales(sa.to(DEV)), W, ws.to(DEV), C,
                            w_zero=wz.to(DEV), workspace=work)
        st = bg.bi_gemm_sync_status(plan, raise_on_error=False)
        assert bg.binding.STATUS_NAMES[st] == "BI_ERR_INVALID_ARG", bad
    # the status word was cleared by the read: a good call reports OK again
    qa, sa, qw, ws, wz = case(M, N, K, seed=6501, integer=True)
    run(qa, sa, qw, ws, wz, plan)
