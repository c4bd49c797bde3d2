"""GPU tests of the e2m1 weight quantisation (bi_quantize_e2m1) against the oracle.

W_fp4 = round((W - zero) / scale) per output channel ("DeepSeek V4的batch invariance：大模型确定性
推理的工程基石" (lshu.cn), section 4.3), read as round to nearest even with saturation at +-6.  The
codes are integers, so the kernel must reproduce the oracle's bytes exactly, ties, saturation,
signed zeros, NaN and infinities included.
"""
import numpy as np
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
import oracle
from invariant_deterministic_gemm_bi_b200 import inputs
from tests.gpu_util import kblock_major_scales, strided_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def weights(N, K, seed, dtype):
    """N(0, 1) * 2^-2 weights with planted ties, out-of-range values, infinities and NaN."""
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(N, K, generator=g) * 0.25
    ws = inputs.channel_scales_pow2(N, seed + 1, lo=1, hi=6)
    wz = inputs.channel_zeros_fp16(ws, seed + 2)
    # exact ties (x = midpoint between two e2m1 values) on some entries of each row
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -5.0, 7.0, -7.0])
    cols = torch.randint(0, K, (N, mids.numel()), generator=g)
    for r in range(N):
        w[r, cols[r]] = mids * ws[r] + wz[r]
    w[0, 0], w[0, 1] = float("nan"), float("inf")
    w[min(1, N - 1), 2] = float("-inf")
    w[min(2, N - 1), 3] = 1e30 if dtype == torch.bfloat16 else 6e4
    w = w.to(dtype)
    return w, ws, wz


def run(w, ws, wz, ldq_extra=0):
    N, K = w.shape
    Wd = w.to(DEV)
    Q = torch.full((N, (K + ldq_extra) // 2), 0xEE, dtype=torch.uint8, device=DEV)
    bg.bi_quantize_e2m1(Wd, ws.to(DEV), Q[:, : K // 2] if not ldq_extra else Q,
                        w_zero=None if wz is None else wz.to(DEV))
    torch.cuda.synchronize()
    return Q.cpu().numpy()


def oracle_codes(w, ws, wz):
    bits = w.view(torch.int16).numpy().view(np.uint16)
    return oracle.quantize_e2m1(bits, ws.numpy(), None if wz is None else wz.numpy(),
                                fp16=w.dtype == torch.float16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("N,K,zero", [(3, 64, True), (37, 130, True), (256, 512, False), (129, 7168, True)])
def test_codes_match_the_oracle_exactly(dtype, N, K, zero):
    w, ws, wz = weights(N, K, seed=7000 + N + K, dtype=dtype)
    wz = wz if zero else None
    got = run(w, ws, wz)
    want = oracle_codes(w, ws, wz)
    assert np.array_equal(got[:, : K // 2], want), np.argwhere(got[:, : K // 2] != want)[:5]


def test_strided_weights_and_codes():
    N, K = 40, 256
    w, ws, wz = weights(N, K, seed=7100, dtype=torch.bfloat16)
    want = oracle_codes(w, ws, wz)
    Wd = strided_rows(w.to(DEV), K + 64)
    Q = torch.full((N, (K + 128) // 2), 0xEE, dtype=torch.uint8, device=DEV)
    bg.bi_quantize_e2m1(Wd, ws.to(DEV), Q[:, : K // 2], w_zero=wz.to(DEV))
    got = Q.cpu().numpy()
    assert np.array_equal(got[:, : K // 2], want)
    assert np.all(got[:, K // 2:] == 0xEE)        # the row padding is left alone


def test_quantised_weights_feed_the_w4a8_gemm():
    # quantise on the GPU, multiply with bi_gemm_run_w4a8, compare with the oracle GEMM of the
    # oracle's own codes (bit-exact: integer activations and small power-of-two scales)
    M, N, K = 24, 256, 512
    w, ws, wz = weights(N, K, seed=7200, dtype=torch.bfloat16)
    w = torch.nan_to_num(w.float(), posinf=1.0, neginf=-1.0).to(torch.bfloat16)
    ws = inputs.channel_scales_pow2(N, 7201, lo=1, hi=4)
    wz = inputs.channel_zeros_grid(N, 7202)
    Q = torch.empty((N, K // 2), dtype=torch.uint8, device=DEV)
    bg.bi_quantize_e2m1(w.to(DEV), ws.to(DEV), Q, w_zero=wz.to(DEV))
    codes = oracle_codes(w, ws, wz)
    assert np.array_equal(Q.cpu().numpy(), codes)
    qa = inputs.e4m3_integers((M, K), 7203)
    sa = inputs.scales_pow2((M, K // 128), 7204, lo=-2, hi=2)
    C = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    work = torch.empty(bg.bi_gemm_w4a8_workspace_bytes(M) // 4, dtype=torch.float32, device=DEV)
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_E2M1_W4A8)
    bg.bi_gemm_run_w4a8(plan, qa.to(DEV), kblock_major_scales(sa.to(DEV)), Q, ws.to(DEV), C,
                        w_zero=wz.to(DEV), workspace=work)
    bg.bi_gemm_sync_status(plan)
    _, want = oracle.gemm_w4a8(inputs.to_numpy_bits(qa), sa.numpy(), codes, ws.numpy(), wz.numpy())
    got = C.view(torch.int16).cpu().numpy().view(np.uint16)
    zero = ((got & 0x7FFF) == 0) & ((want & 0x7FFF) == 0)
    assert np.all((got == want) | zero)


@pytest.mark.parametrize("fp16", [False, True])
def test_vector_rows_with_a_ragged_tail(fp16):
    # 16-byte-aligned rows (pitch 144 values) whose K = 138 leaves one code byte past the last
    # whole 8-value group
    N, K = 33, 138
    dtype = torch.float16 if fp16 else torch.bfloat16
    w, ws, wz = weights(N, K, seed=7300, dtype=dtype)
    want = oracle_codes(w, ws, wz)
    Wd = strided_rows(w.to(DEV), 144)
    Q = torch.full((N, 72), 0xEE, dtype=torch.uint8, device=DEV)
    bg.bi_quantize_e2m1(Wd, ws.to(DEV), Q[:, : K // 2], w_zero=wz.to(DEV))
    got = Q.cpu().numpy()
    assert np.array_equal(got[:, : K // 2], want), np.argwhere(got[:, : K // 2] != want)[:5]
    assert np.all(got[:, K // 2:] == 0xEE)


@pytest.mark.parametrize("N,K", [(64, 512), (21, 130)])
def test_scales_that_are_not_powers_of_two(N, K):
    # any non-zero fp32 scale is accepted: these divide in fp64 instead of multiplying by an exact
    # reciprocal (512: the vector kernel; 130: the scalar one)
    w, _, wz = weights(N, K, seed=7400 + K, dtype=torch.bfloat16)
    ws = inputs.scales_log_uniform((N,), seed=7401) * 0.1
    ws[0] = -0.3                                 # a negative scale flips the codes' signs
    want = oracle_codes(w, ws, wz)
    got = run(w, ws, wz)
    assert np.array_equal(got[:, : K // 2], want), np.argwhere(got[:, : K // 2] != want)[:5]
