"""Dual-kernel decode attention on the GPU: the no-split and split-KV kernels are bitwise equal,
a sequence's output does not depend on its batch-mates, and both match the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
from oracle import attention as oatt
from oracle import oracle as orc
from invariant_deterministic_gemm_bi_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 128


def make(B, Hq, Hkv, Lmax, seed):
    Q = inputs.bf16_gaussian((B, Hq, D), seed=seed, device=DEV)
    K = inputs.bf16_gaussian((B, Lmax, Hkv, D), seed=seed + 1, device=DEV)
    V = inputs.bf16_gaussian((B, Lmax, Hkv, D), seed=seed + 2, device=DEV)
    return Q, K, V


def run(Q, K, V, lengths, splits):
    B, Hq, _ = Q.shape
    O = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = None
    n = bg.bi_decode_attention_workspace_bytes(B, Hq, D, max(splits, 4))
    if n:
        ws = torch.empty(n // 4, dtype=torch.float32, device=DEV)
    bg.bi_decode_attention(Q, K, V, lengths, O, 1.0 / math.sqrt(D), splits=splits, workspace=ws)
    torch.cuda.synchronize()
    return O


def lengths_for(B, Lmax, seed):
    g = inputs.generator(seed, "cpu")
    L = torch.randint(1, Lmax + 1, (B,), generator=g, dtype=torch.int32)
    L[0] = 1
    L[-1] = Lmax
    return L


# The K/V pipeline depth follows the CTA count (6 stages up to two CTAs per SM, else 2), so these
# cases compare kernels of both depths: (16, 32, 8) runs the no-split kernel deep and split-4
# shallow, (48, 32, 8) every kernel shallow.
@pytest.mark.parametrize("B,Hq,Hkv,Lmax", [(4, 8, 2, 300), (16, 32, 8, 1024), (3, 16, 2, 5),
                                           (48, 32, 8, 200)])
def test_split_kernels_match_the_no_split_kernel_bitwise(B, Hq, Hkv, Lmax):
    Q, K, V = make(B, Hq, Hkv, Lmax, 9900 + B)
    L = lengths_for(B, Lmax, 9910 + B).to(DEV)
    ref = run(Q, K, V, L, 1).view(torch.int16)
    for s in (2, 4, 0):
        got = run(Q, K, V, L, s).view(torch.int16)
        assert torch.equal(got, ref), f"splits={s} differs from the no-split kernel"


@pytest.mark.parametrize("B,Hq,Hkv,Lmax", [(4, 8, 2, 300), (5, 32, 8, 777), (2, 8, 1, 7)])
def test_matches_oracle(B, Hq, Hkv, Lmax):
    Q, K, V = make(B, Hq, Hkv, Lmax, 9920 + B)
    L = lengths_for(B, Lmax, 9930 + B)
    O = run(Q, K, V, L.to(DEV), 4)
    ref, _ = oatt.decode_attention(inputs.to_numpy_bits(Q), inputs.to_numpy_bits(K),
                                   inputs.to_numpy_bits(V), L.numpy(), 1.0 / math.sqrt(D))
    got = orc.bf16_to_f64(inputs.to_numpy_bits(O))
    vmax = float(orc.bf16_to_f64(inputs.to_numpy_bits(V)).__abs__().max())
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -7 * np.abs(ref) + 2.0 ** -12 * vmax), float(err.max())


def test_sequence_output_independent_of_batch_mates():
    Hq, Hkv, Lmax = 16, 4, 640
    Q, K, V = make(12, Hq, Hkv, Lmax, 9940)
    L = lengths_for(12, Lmax, 9941).to(DEV)
    for splits in (1, 4):
        full = run(Q, K, V, L, splits).view(torch.int16)
        for b in (0, 5, 11):
            alone = run(Q[b:b + 1].contiguous(), K[b:b + 1].contiguous(), V[b:b + 1].contiguous(),
                        L[b:b + 1].contiguous(), splits).view(torch.int16)
            assert torch.equal(alone[0], full[b]), f"sequence {b} changes with its batch (splits={splits})"


def test_invalid_length_gives_nan_and_rejects_bad_shapes():
    Q, K, V = make(2, 8, 2, 16, 9950)
    L = torch.tensor([0, 17], dtype=torch.int32, device=DEV)
    O = run(Q, K, V, L, 1)
    assert torch.isnan(O.float()).all()
    with pytest.raises(bg.BiGemmError):
        Qbad = inputs.bf16_gaussian((1, 6, D), seed=1, device=DEV)   # 6 heads over 4 kv heads
        Kbad = inputs.bf16_gaussian((1, 8, 4, D), seed=2, device=DEV)
        bg.bi_decode_attention(Qbad, Kbad, Kbad, L[:1], torch.empty_like(Qbad), 0.1)
