"""Pins of the decode-attention oracle (oracle/attention.py) against closed forms."""
import math

import numpy as np

from oracle import attention
from oracle import oracle as orc


def bits(x):
    return orc.f64_to_bf16(np.asarray(x, dtype=np.float64))


def test_equal_scores_average_the_values():
    # K = 0: every score is 0, the softmax is uniform, O = mean of V (integer V: exact mean)
    B, Hq, Hkv, D, L = 1, 4, 2, 8, 6
    Q = bits(np.ones((B, Hq, D)))
    K = bits(np.zeros((B, L, Hkv, D)))
    Vv = np.arange(B * L * Hkv * D, dtype=np.float64).reshape(B, L, Hkv, D) % 7
    O, _ = attention.decode_attention(Q, K, bits(Vv), [L], 0.125)
    for h in range(Hq):
        assert np.allclose(O[0, h], Vv[0, :, h // 2, :].mean(axis=0), rtol=0, atol=1e-12)


def test_single_key_returns_its_value():
    Q = bits(np.random.default_rng(1).normal(size=(2, 2, 8)))
    K = bits(np.random.default_rng(2).normal(size=(2, 5, 1, 8)))
    Vv = np.random.default_rng(3).integers(-4, 5, size=(2, 5, 1, 8)).astype(np.float64)
    O, _ = attention.decode_attention(Q, K, bits(Vv), [1, 1], 0.5)
    assert (O[:, 0] == Vv[:, 0, 0]).all() and (O[:, 1] == Vv[:, 0, 0]).all()


def test_two_keys_closed_form_softmax():
    # scores a, b: O = (v0 e^a + v1 e^b) / (e^a + e^b)
    D = 4
    Q = bits(np.ones((1, 1, D)))
    Kv = np.zeros((1, 2, 1, D))
    Kv[0, 0, 0, 0] = 2.0      # score 2 * scale
    Kv[0, 1, 0, 0] = -1.0     # score -scale
    Vv = np.zeros((1, 2, 1, D))
    Vv[0, 0, 0] = [1, 0, 0, 0]
    Vv[0, 1, 0] = [0, 1, 0, 0]
    scale = 0.5
    O, _ = attention.decode_attention(Q, bits(Kv), bits(Vv), [2], scale)
    ea, eb = math.exp(2 * scale), math.exp(-1 * scale)
    assert abs(O[0, 0, 0] - ea / (ea + eb)) < 1e-15 and abs(O[0, 0, 1] - eb / (ea + eb)) < 1e-15


def test_key_permutation_invariance_and_padding_ignored():
    rng = np.random.default_rng(4)
    B, Hq, Hkv, D, L, Lmax = 1, 8, 2, 16, 37, 64
    Q = bits(rng.normal(size=(B, Hq, D)))
    K = bits(rng.normal(size=(B, Lmax, Hkv, D)))
    V = bits(rng.normal(size=(B, Lmax, Hkv, D)))
    O1, _ = attention.decode_attention(Q, K, V, [L], 0.25)
    perm = rng.permutation(L)
    K2, V2 = K.copy(), V.copy()
    K2[:, :L], V2[:, :L] = K[:, perm], V[:, perm]
    K2[:, L:] = bits(np.full((B, Lmax - L, Hkv, D), 1e3))    # padding beyond L must not matter
    O2, _ = attention.decode_attention(Q, K2, V2, [L], 0.25)
    assert np.allclose(O1, O2, rtol=1e-12, atol=1e-14)
