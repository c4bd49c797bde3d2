"""CPU oracle for the dual-kernel decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import this module.
Plain numpy in fp64: for each sequence b and query head h (key/value head h // (Hq / Hkv)),
s_j = scale * q . k_j over the sequence's L_b keys, O = sum_j softmax(s)_j v_j -- the attention
the split-KV and no-split kernels of "DeepSeek V4的batch invariance：大模型确定性推理的工程基石"
(lshu.cn), section 4.1, both compute.  Exact in the order of the sum up to fp64 rounding, so it
pins the result, not the kernels' (fixed) reduction order, which the GPU tests check by comparing
the kernels with each other bitwise.

Pins: ``tests/test_oracle_attention.py`` (uniform keys, one dominant key, L = 1, key permutation,
a softmax closed form).
"""
from __future__ import annotations

import numpy as np

from .oracle import bf16_to_f64, f64_to_bf16


def decode_attention(Q_bits, K_bits, V_bits, lengths, scale: float):
    """Q_bits [B, Hq, D], K_bits / V_bits [B, Lmax, Hkv, D] (bf16 bits), lengths [B].
    Returns the fp64 output [B, Hq, D] and its bf16 bits (one rounding)."""
    Q = bf16_to_f64(np.asarray(Q_bits, dtype=np.uint16))
    K = bf16_to_f64(np.asarray(K_bits, dtype=np.uint16))
    V = bf16_to_f64(np.asarray(V_bits, dtype=np.uint16))
    B, Hq, D = Q.shape
    Hkv = K.shape[2]
    G = Hq // Hkv
    sc = float(np.float32(scale))
    O = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        L = int(lengths[b])
        for h in range(Hq):
            kv = h // G
            s = sc * (K[b, :L, kv, :] @ Q[b, h])
            w = np.exp(s - s.max())
            O[b, h] = (w[:, None] * V[b, :L, kv, :]).sum(axis=0) / w.sum()
    return O, f64_to_bf16(O)
