"""Bit-exact parity at the workloads' own shapes, whole output matrices.

On the integer variant (entries uniform in {-4..4}, exact in bf16) every product and every
partial sum of a K = 7168 reduction is an integer of magnitude at most 16 * 7168 < 2^24, so it is
exact in fp32 whatever the order, and the GPU's bf16 result must equal the oracle's bit for bit
("DeepSeek V4的batch invariance：大模型确定性推理的工程基石" (lshu.cn), section 5.1 checks batch
invariance with a bitwise equality).  These cases run every scheduling form of the plans on the
real shapes:

* decode 4096 x 7168 at every M of the sweep: the tiny-batch (M <= 8), small-batch (<= 32),
  plan (64) and wide lockstep forms (128, 256), with A boxes of exactly M rows below a tile;
* prefill 7168 x 2048 and 2048 x 7168 at M = 1024 and 4096 (CTA-pair tiles, several waves);
* grouped 64 x 2048 x 7168 at T = 64 and 1024 tokens routed top-8 by a seeded softmax (the
  routing comes from the oracle's MoE steps), every row.

The expected bits come from ``oracle.gemm_bf16_exact_integers`` (the exact integer product,
rounded once to bf16), which the CPU tests pin to the scalar oracle and to int64 arithmetic.
"""
import numpy as np
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
import oracle
from invariant_deterministic_gemm_bi_b200 import inputs
from tests import parity
from tests import routing as routing_mod
from tests.gpu_util import GuardedC

pytestmark = pytest.mark.gpu
DEV = "cuda"

DECODE_M = [1, 2, 4, 8, 16, 32, 64, 128, 256]


def run_dense(plan, A, B):
    out = GuardedC(A.shape[0], B.shape[0])
    bg.bi_gemm_run(plan, A, B, out.c)
    bg.bi_gemm_sync_status(plan)
    out.check()
    return parity.bits(out.c)


@pytest.fixture(scope="module")
def decode_weights():
    B = inputs.bf16_integers((4096, 7168), seed=4701, device=DEV)
    return B, inputs.to_numpy_bits(B)


@pytest.mark.parametrize("M", DECODE_M)
def test_decode_integers_whole_matrix_bit_exact(decode_weights, M):
    B, Bb = decode_weights
    plan = bg.bi_gemm_plan(4096, 7168)
    A = inputs.bf16_integers((M, 7168), seed=4702 + M, device=DEV)
    got = run_dense(plan, A, B)
    _, want = oracle.gemm_bf16_exact_integers(inputs.to_numpy_bits(A), Bb)
    parity.assert_bits_equal_values(got, want, f"decode integers M={M}")


@pytest.mark.parametrize("N,K", [(7168, 2048), (2048, 7168)])
@pytest.mark.parametrize("M", [1024, 4096])
def test_prefill_integers_whole_matrix_bit_exact(N, K, M):
    plan = bg.bi_gemm_plan(N, K)
    B = inputs.bf16_integers((N, K), seed=4801 + N, device=DEV)
    A = inputs.bf16_integers((M, K), seed=4802 + M, device=DEV)
    got = run_dense(plan, A, B)
    _, want = oracle.gemm_bf16_exact_integers(inputs.to_numpy_bits(A), inputs.to_numpy_bits(B))
    parity.assert_bits_equal_values(got, want, f"prefill integers {N}x{K} M={M}")


@pytest.fixture(scope="module")
def moe_weights():
    B = inputs.bf16_integers((64, 2048, 7168), seed=4901, device=DEV)
    return B, inputs.to_numpy_bits(B)


@pytest.mark.parametrize("T", [64, 1024])
def test_grouped_integers_every_row_bit_exact(moe_weights, T):
    B, Bb = moe_weights
    E, N, K = B.shape
    r = routing_mod.softmax_top8_routing(T, E, seed=4902 + T)
    tokens = inputs.bf16_integers((T, K), seed=4903 + T, device=DEV)
    A = tokens[r.token_of_row.to(DEV)].contiguous()
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_BF16, E)
    out = GuardedC(A.shape[0], N)
    bg.bi_grouped_gemm_run(plan, A, B, out.c, r.offsets.to(DEV))
    bg.bi_gemm_sync_status(plan)
    out.check()
    _, want = oracle.grouped_gemm_bf16_exact_integers(inputs.to_numpy_bits(A), Bb, r.offsets.numpy())
    parity.assert_bits_equal_values(parity.bits(out.c), want, f"MoE integers T={T}")
    assert np.count_nonzero(np.diff(r.offsets.numpy())) > (8 if T == 1 else 32)
