"""Pins of the MoE-step oracle (oracle/moe.py) against closed forms and hand-worked cases."""
import math

import numpy as np

from oracle import moe
from oracle import oracle as orc


def test_equal_logits_pick_the_lowest_experts_with_weight_one_over_e():
    E, k = 64, 8
    experts, weights = moe.route_topk(np.zeros((3, E), dtype=np.float32), k)
    assert (experts == np.arange(k)).all()
    assert (weights == 1.0 / E).all()          # 2^-6 exactly


def test_distinct_logits_closed_form_softmax():
    # logits 0, 1, ..., E-1: top k are E-1, E-2, ...; p_e = e^(e-E+1) (1 - 1/e) / (1 - e^-E)
    E, k = 64, 8
    logits = np.arange(E, dtype=np.float32)[None, :]
    experts, weights = moe.route_topk(logits, k)
    assert list(experts[0]) == list(range(E - 1, E - 1 - k, -1))
    for j, e in enumerate(experts[0]):
        closed = math.exp(e - E + 1) * (1 - math.exp(-1)) / (1 - math.exp(-E))
        assert abs(weights[0, j] - closed) <= 1e-15 * closed


def test_ties_go_to_the_lower_expert_index():
    E, k = 16, 4
    row = np.array([1, 3, 3, 0, 2, 3, 2, 0, 0, 1, 3, 2, 0, 0, 1, 1], dtype=np.float32)
    experts, weights = moe.route_topk(row[None, :], k)
    assert list(experts[0]) == [1, 2, 5, 10]            # the four 3s in index order
    assert len(set(weights[0])) == 1                     # equal logits, equal weights


def test_dispatch_hand_worked():
    experts = np.array([[1, 0], [1, 2], [0, 1]])
    offsets, tok, ros = moe.dispatch(experts, 3)
    assert list(offsets) == [0, 2, 5, 6]
    assert list(tok) == [0, 2, 0, 1, 2, 1]
    assert list(ros) == [2, 0, 3, 5, 1, 4]


def test_dispatch_invariants_and_out_of_range_ids():
    rng = np.random.default_rng(7)
    T, k, E = 50, 8, 16
    experts = rng.integers(0, E, size=(T, k))
    offsets, tok, ros = moe.dispatch(experts, E)
    assert offsets[-1] == T * k and (np.diff(offsets) >= 0).all()
    assert sorted(ros) == list(range(T * k))                      # a permutation
    flat = experts.reshape(-1)
    assert (tok[ros] == np.arange(T * k) // k).all()              # rows point back at their token
    assert (np.diff(flat[np.argsort(ros)]) >= 0).all()            # rows ordered by expert
    bad = experts.copy()
    bad[0, 0] = E                                                 # out of range: left out
    offsets2, _, ros2 = moe.dispatch(bad, E)
    assert offsets2[-1] == T * k - 1 and ros2[0] == -1


def test_gather_is_a_row_copy():
    X = np.arange(5 * 8, dtype=np.uint16).reshape(5, 8)
    out = moe.gather_rows(X, np.array([4, 0, 0, 2]))
    assert (out == X[[4, 0, 0, 2]]).all()


def test_combine_exact_with_power_of_two_weights():
    # integer C values and weights 2^-j: every product and partial sum is exact
    T, k, N = 3, 4, 8
    vals = np.arange(T * k * N, dtype=np.float64).reshape(T * k, N) - 40
    C_bits = orc.f64_to_bf16(vals)
    w = np.array([[2.0 ** -j for j in range(k)]] * T, dtype=np.float32)
    ros = np.arange(T * k)[::-1].copy()
    Y, Ybits = moe.combine(C_bits, ros, w)
    expect = np.zeros((T, N))
    for t in range(T):
        for j in range(k):
            expect[t] += w[t, j] * vals[ros[t * k + j]]
    assert (Y == expect).all()
    assert (orc.bf16_to_f64(Ybits) == orc.bf16_to_f64(orc.f64_to_bf16(expect))).all()
