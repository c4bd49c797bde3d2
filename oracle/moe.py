"""CPU oracle for the MoE steps around the grouped GEMM -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import this module;
the product package never does.  Plain numpy, fp64 for the floating-point steps, written from the
definitions of the workload these steps serve: each token is routed to the top k experts by
router logit (ties to the lower expert index), its k (token, slot) pairs are grouped by expert in
a stable order, the grouped rows are gathered, and the k expert outputs are combined with the
token's softmax probabilities.  The pages ("DeepSeek不惜代价保住它！V4关键特性被挖出来了"
(QbitAI), on what V4 is built from) name MoE but give no formula.  Readings: the weights are the
softmax over all experts of the selected ones (not renormalised over the k), and the combine adds
a token's expert outputs in slot order (descending logit).  The routing helpers of
``invariant_deterministic_gemm_bi_b200.inputs`` are not used here: this is an independent
restatement.

Pins: ``tests/test_oracle_moe.py`` (closed forms, hand-worked dispatch, exact combines).
"""
from __future__ import annotations

import numpy as np

from .oracle import bf16_to_f64, f64_to_bf16


def route_topk(logits: np.ndarray, k: int):
    """Top-k experts per token and their softmax probabilities over all experts.

    experts[t, j] is the j-th expert of token t in descending logit order, ties going to the
    lower expert index; weights[t, j] = exp(l - max) / sum_e exp(l_e - max), in fp64.
    """
    L = np.asarray(logits, dtype=np.float32)
    T, E = L.shape
    experts = np.empty((T, k), dtype=np.int64)
    weights = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        row = L[t].astype(np.float64)
        order = sorted(range(E), key=lambda e: (-row[e], e))
        sel = order[:k]
        ex = np.exp(row - row.max())
        experts[t] = sel
        weights[t] = ex[sel] / ex.sum()
    return experts, weights


def dispatch(experts: np.ndarray, num_experts: int):
    """Stable grouping of the T*k (token, slot) pairs by expert.

    Pair i = t*k + j is placed at row r_i; rows are ordered by expert, then by i.  Returns
    offsets [E+1], token_of_row [R] and row_of_slot [T*k] (int64).  Expert ids outside [0, E)
    are left out (their row_of_slot entries are -1).
    """
    X = np.asarray(experts, dtype=np.int64)
    T, k = X.shape
    flat = X.reshape(-1)
    offsets = np.zeros(num_experts + 1, dtype=np.int64)
    token_of_row = []
    row_of_slot = np.full(flat.size, -1, dtype=np.int64)
    r = 0
    for e in range(num_experts):
        pairs = np.nonzero(flat == e)[0]          # ascending pair index
        for i in pairs:
            token_of_row.append(i // k)
            row_of_slot[i] = r
            r += 1
        offsets[e + 1] = r
    return offsets, np.asarray(token_of_row, dtype=np.int64), row_of_slot


def gather_rows(X_bits: np.ndarray, token_of_row: np.ndarray) -> np.ndarray:
    """A_perm[r] = X[token_of_row[r]] (raw bf16 bits, an exact copy)."""
    return np.asarray(X_bits)[np.asarray(token_of_row, dtype=np.int64)]


def combine(C_bits: np.ndarray, row_of_slot: np.ndarray, weights: np.ndarray):
    """Y[t] = sum_j weights[t, j] * C[row_of_slot[t*k + j]], summed in fp64 (the unrounded
    reference) and rounded once to bf16.  weights are the fp32 values the combine is given."""
    C = bf16_to_f64(np.asarray(C_bits, dtype=np.uint16))
    W = np.asarray(weights, dtype=np.float32).astype(np.float64)
    T, k = W.shape
    rows = np.asarray(row_of_slot, dtype=np.int64).reshape(T, k)
    Y = np.zeros((T, C.shape[1]), dtype=np.float64)
    for j in range(k):
        Y += W[:, j:j + 1] * C[rows[:, j]]
    return Y, f64_to_bf16(Y)
