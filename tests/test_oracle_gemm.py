"""Pins for the oracle's GEMMs (dense bf16, FP8 block-scaled, grouped).

Every check compares the oracle with something it does not compute itself: hand-worked golden
cases, closed forms (identity, permutation and rank-1 operands), exact integer matmuls, exact
rational brute force with round-to-nearest-even by table lookup, and reductions of the FP8 and
grouped oracles to special cases whose answers are fixed independently.  A transposed operand,
a dropped or repeated K term, a wrong sign, a wrong scale index or a double rounding each fail
at least one of them.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from invariant_deterministic_gemm_bi_b200 import inputs
from tests import exact, golden_io
from tests import routing as routing_mod


def bf16_bits(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def bf16_values(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).astype(np.uint32).view(np.float32) \
        .astype(np.float64)


def e4m3_values(codes):
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8).copy()).view(torch.float8_e4m3fn) \
        .to(torch.float32).numpy().astype(np.float64)


# ---------------------------------------------------------------------------------------------
# dense bf16
# ---------------------------------------------------------------------------------------------

def test_golden_worked_examples():
    n = 0
    for name, A, B, C in golden_io.gemm_cases():
        cref, cbits = oracle.gemm_bf16(bf16_bits(A), bf16_bits(B))
        assert np.array_equal(bf16_values(cbits), C), name
        n += 1
    assert n >= 4


def test_identity_selects_columns():
    M, N, K = 9, 24, 40
    A = inputs.to_numpy_bits(inputs.bf16_gaussian((M, K), seed=1))
    B = np.zeros((N, K), dtype=np.float32)
    B[np.arange(N), np.arange(N)] = 1.0
    cref, cbits = oracle.gemm_bf16(A, bf16_bits(B))
    assert np.array_equal(cbits, A[:, :N])
    assert np.array_equal(cref, bf16_values(A[:, :N]))


def test_permutation_permutes_columns():
    M, N, K = 5, 33, 33
    rng = np.random.default_rng(3)
    perm = rng.permutation(K)[:N]
    A = inputs.to_numpy_bits(inputs.bf16_gaussian((M, K), seed=2))
    B = np.zeros((N, K), dtype=np.float32)
    B[np.arange(N), perm] = 1.0
    _, cbits = oracle.gemm_bf16(A, bf16_bits(B))
    assert np.array_equal(cbits, A[:, perm])
    # a negated permutation flips exactly the sign bit
    _, cneg = oracle.gemm_bf16(A, bf16_bits(-B))
    assert np.array_equal(cneg, A[:, perm] ^ 0x8000)


def test_rank_one_closed_form():
    # A = u x^T, B = v y^T  =>  C = (x . y) u v^T, exact in fp64 and in bf16 for these ranges
    rng = np.random.default_rng(5)
    M, N, K = 7, 11, 13
    u = rng.integers(-3, 4, size=M)
    v = rng.integers(-3, 4, size=N)
    x = rng.integers(-4, 5, size=K)
    y = rng.integers(-4, 5, size=K)
    A = np.outer(u, x).astype(np.float32)
    B = np.outer(v, y).astype(np.float32)
    cref, cbits = oracle.gemm_bf16(bf16_bits(A), bf16_bits(B))
    want = float(x @ y) * np.outer(u, v).astype(np.float64)
    assert np.array_equal(cref, want)
    assert np.array_equal(cbits, np.array([[exact.rne_bf16(Fraction(int(w))) for w in r]
                                           for r in want], dtype=np.uint16))


def test_small_integers_exact_against_integer_matmul():
    # the small workload's integer variant: entries in {-4..4}, K = 512
    M, N, K = 17, 256, 512
    A = inputs.to_numpy_bits(inputs.bf16_integers((M, K), seed=1001))
    B = inputs.to_numpy_bits(inputs.bf16_integers((N, K), seed=1002))
    Ai = bf16_values(A).astype(np.int64)
    Bi = bf16_values(B).astype(np.int64)
    want = Ai @ Bi.T
    cref, cbits = oracle.gemm_bf16(A, B)
    assert np.array_equal(cref, want.astype(np.float64))
    table = {int(w): exact.rne_bf16(Fraction(int(w))) for w in np.unique(want)}
    assert np.array_equal(cbits, np.vectorize(table.get)(want).astype(np.uint16))


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_exact_rationals(seed):
    rng = np.random.default_rng(100 + seed)
    M, N, K = rng.integers(1, 9, size=3)
    # wide exponent spread, so that a wrong order or an intermediate rounding would show
    A = rng.standard_normal((M, K)) * np.exp2(rng.integers(-6, 7, size=(M, K)))
    B = rng.standard_normal((N, K)) * np.exp2(rng.integers(-6, 7, size=(N, K)))
    Ab, Bb = bf16_bits(A), bf16_bits(B)
    cref, cbits = oracle.gemm_bf16(Ab, Bb)
    C = exact.exact_gemm(bf16_values(Ab), bf16_values(Bb))
    for m in range(M):
        for n in range(N):
            q = C[m][n]
            assert cbits[m, n] == exact.rne_bf16(q), (m, n)
            bound = K * 2.0 ** -53 * float(sum(abs(Fraction(float(a)) * Fraction(float(b)))
                                               for a, b in zip(bf16_values(Ab)[m],
                                                               bf16_values(Bb)[n])))
            assert abs(Fraction(cref[m, n]) - q) <= Fraction(bound)


def test_empty_and_degenerate_shapes():
    cref, cbits = oracle.gemm_bf16(np.zeros((0, 8), np.uint16), np.zeros((3, 8), np.uint16))
    assert cref.shape == (0, 3)
    cref, cbits = oracle.gemm_bf16(np.zeros((2, 0), np.uint16), np.zeros((3, 0), np.uint16))
    assert np.array_equal(cref, np.zeros((2, 3))) and np.array_equal(cbits, np.zeros((2, 3)))


def test_threads_do_not_change_bits():
    A = inputs.to_numpy_bits(inputs.bf16_gaussian((37, 96), seed=9))
    B = inputs.to_numpy_bits(inputs.bf16_gaussian((29, 96), seed=10))
    c1 = oracle.gemm_bf16(A, B, threads=1)
    c7 = oracle.gemm_bf16(A, B, threads=7)
    assert np.array_equal(c1[0], c7[0]) and np.array_equal(c1[1], c7[1])


# ---------------------------------------------------------------------------------------------
# FP8 block-scaled
# ---------------------------------------------------------------------------------------------

def test_fp8_golden_worked_examples():
    n = 0
    for case in golden_io.fp8_cases():
        cref, cbits = oracle.gemm_fp8_blockscaled(case["qa"], case["qb"], case["sa"], case["sb"])
        assert np.array_equal(bf16_values(cbits), case["c"]), case["name"]
        n += 1
    assert n >= 2


def test_fp8_unit_scales_reduce_to_plain_gemm_of_decoded_codes():
    M, N, K = 6, 10, 256
    qa = inputs.to_numpy_bits(inputs.e4m3_integers((M, K), seed=41))
    qb = inputs.to_numpy_bits(inputs.e4m3_integers((N, K), seed=42))
    sa = np.ones((M, 2), np.float32)
    sb = np.ones((1, 2), np.float32)
    cref, _ = oracle.gemm_fp8_blockscaled(qa, qb, sa, sb)
    want = e4m3_values(qa).astype(np.int64) @ e4m3_values(qb).astype(np.int64).T
    assert np.array_equal(cref, want.astype(np.float64))


def test_fp8_pow2_scales_exact_blockwise_closed_form():
    # C[m,n] = sum_kb sa[m,kb] sb[n//128,kb] (sum_{k in kb} qa qb), fixed in exact rationals;
    # N = 200 spans two B scale blocks, K = 384 three K blocks.
    M, N, K = 5, 200, 384
    qa = inputs.to_numpy_bits(inputs.e4m3_integers((M, K), seed=51))
    qb = inputs.to_numpy_bits(inputs.e4m3_integers((N, K), seed=52))
    sa = inputs.scales_pow2((M, 3), seed=53).numpy()
    sb = inputs.scales_pow2((2, 3), seed=54).numpy()
    cref, cbits = oracle.gemm_fp8_blockscaled(qa, qb, sa, sb)
    va = e4m3_values(qa).astype(np.int64)
    vb = e4m3_values(qb).astype(np.int64)
    for m in range(M):
        for n in range(N):
            q = Fraction(0)
            for kb in range(3):
                part = int(va[m, kb * 128:(kb + 1) * 128] @ vb[n, kb * 128:(kb + 1) * 128])
                q += part * Fraction(float(sa[m, kb])) * Fraction(float(sb[n // 128, kb]))
            assert cref[m, n] == float(q)
            assert cbits[m, n] == exact.rne_bf16(q)


def test_fp8_single_scale_changes_only_its_block():
    M, N, K = 3, 130, 256
    qa = inputs.to_numpy_bits(inputs.e4m3_gaussian((M, K), seed=61))
    qb = inputs.to_numpy_bits(inputs.e4m3_gaussian((N, K), seed=62))
    sa = np.ones((M, 2), np.float32)
    sb = np.ones((2, 2), np.float32)
    base, _ = oracle.gemm_fp8_blockscaled(qa, qb, sa, sb)
    sa2 = sa.copy()
    sa2[1, 1] = 2.0     # row 1, K block 1
    sb2 = sb.copy()
    sb2[1, 0] = 4.0     # N block 1 (columns 128..129), K block 0
    c2, _ = oracle.gemm_fp8_blockscaled(qa, qb, sa2, sb2)
    va, vb = e4m3_values(qa), e4m3_values(qb)
    blk = lambda m, n, kb: float(va[m, kb * 128:(kb + 1) * 128] @ vb[n, kb * 128:(kb + 1) * 128])
    for m in range(M):
        for n in range(N):
            want = sum(blk(m, n, kb) * float(sa2[m, kb]) * float(sb2[n // 128, kb]) for kb in range(2))
            assert abs(c2[m, n] - want) <= 1e-9 * (1 + abs(want)), (m, n)
            if m != 1 and n < 128:
                assert c2[m, n] == base[m, n], (m, n)


def test_fp8_log_uniform_scales_vs_dequantised_float64_matmul():
    M, N, K = 8, 256, 512
    qa = inputs.to_numpy_bits(inputs.e4m3_gaussian((M, K), seed=71))
    qb = inputs.to_numpy_bits(inputs.e4m3_gaussian((N, K), seed=72))
    sa = inputs.scales_log_uniform((M, 4), seed=73).numpy()
    sb = inputs.scales_log_uniform((2, 4), seed=74).numpy()
    a = e4m3_values(qa) * np.repeat(sa.astype(np.float64), 128, axis=1)
    b = e4m3_values(qb) * np.repeat(np.repeat(sb.astype(np.float64), 128, axis=0), 128, axis=1)
    want = a @ b.T
    cref, _ = oracle.gemm_fp8_blockscaled(qa, qb, sa, sb)
    bound = K * 2.0 ** -52 * (np.abs(a) @ np.abs(b).T)
    assert np.all(np.abs(cref - want) <= bound)


# ---------------------------------------------------------------------------------------------
# grouped
# ---------------------------------------------------------------------------------------------

def test_grouped_single_expert_is_dense():
    A = inputs.to_numpy_bits(inputs.bf16_gaussian((21, 64), seed=81))
    B = inputs.to_numpy_bits(inputs.bf16_gaussian((1, 40, 64), seed=82))
    g = oracle.grouped_gemm_bf16(A, B, np.array([0, 21], np.int32))
    d = oracle.gemm_bf16(A, B[0])
    assert np.array_equal(g[0], d[0]) and np.array_equal(g[1], d[1])


def test_grouped_segments_use_their_own_expert_exact():
    # integer data so every value is exact; expert e's weights are (e+1) * identity-like rows
    E, N, K = 4, 8, 16
    offsets = np.array([0, 3, 3, 4, 9], np.int32)   # expert 1 is empty
    R = int(offsets[-1])
    A = inputs.to_numpy_bits(inputs.bf16_integers((R, K), seed=91))
    B = np.zeros((E, N, K), np.float32)
    for e in range(E):
        B[e, np.arange(N), np.arange(N)] = e + 1
        B[e, :, K - 1] = -(e + 1)
    cref, cbits = oracle.grouped_gemm_bf16(A, bf16_bits(B), offsets)
    va = bf16_values(A)
    for e in range(E):
        for r in range(offsets[e], offsets[e + 1]):
            want = (e + 1) * (va[r, :N] - va[r, K - 1])
            assert np.array_equal(cref[r], want), (e, r)


def test_grouped_brute_force_with_empty_experts():
    rng = np.random.default_rng(5)
    E, N, K = 5, 3, 6
    offsets = np.array([0, 0, 2, 2, 5, 6], np.int32)
    R = 6
    A = bf16_bits(rng.standard_normal((R, K)))
    B = bf16_bits(rng.standard_normal((E, N, K)))
    _, cbits = oracle.grouped_gemm_bf16(A, B, offsets)
    for e in range(E):
        for r in range(offsets[e], offsets[e + 1]):
            C = exact.exact_gemm(bf16_values(A[r:r + 1]), bf16_values(B[e]))
            assert [cbits[r, n] for n in range(N)] == [exact.rne_bf16(q) for q in C[0]]


@pytest.mark.parametrize("bad", [[1, 2, 3], [0, 3, 2], [0, 1, 4]])
def test_grouped_rejects_malformed_offsets(bad):
    A = np.zeros((3, 8), np.uint16)
    B = np.zeros((2, 4, 8), np.uint16)
    with pytest.raises(ValueError):
        oracle.grouped_gemm_bf16(A, B, np.array(bad, np.int32))


def test_routing_is_stable_top8_grouped_by_expert():
    """The grouped-GEMM tests' routing helper (built on the oracle's MoE steps) groups every token's
    top-8 experts by expert, token order inside a segment, no duplicates, ties to the lower id."""
    r = routing_mod.softmax_top8_routing(T=50, num_experts=64, seed=5)
    off = r.offsets.numpy()
    assert off[0] == 0 and off[-1] == 400 and np.all(np.diff(off) >= 0)
    e = r.expert_of_row.numpy()
    t = r.token_of_row.numpy()
    for x in range(64):
        seg = slice(off[x], off[x + 1])
        assert np.all(e[seg] == x)
        assert np.all(np.diff(t[seg]) > 0)   # token order inside a segment, no duplicates
    # every token appears exactly 8 times, with its 8 largest logits
    g = inputs.generator(5, "cpu")
    logits = torch.randn(50, 64, generator=g, dtype=torch.float32).numpy()
    for tok in range(50):
        experts = sorted(e[t == tok].tolist())
        assert experts == sorted(np.argsort(-logits[tok], kind="stable")[:8].tolist())
    # ties go to the lower expert index
    assert routing_mod.topk_experts(torch.zeros(1, 16), 8).tolist() == [list(range(8))]


# ---------------------------------------------------------------------------------------------
# exact-integer GEMMs (the integer variants at full size)
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K,lo,hi", [(7, 33, 64, -4, 4), (40, 17, 300, -4, 4), (3, 5, 7, -256, 256)])
def test_exact_integer_gemm_equals_the_scalar_oracle_and_int64(M, N, K, lo, hi):
    A = inputs.bf16_integers((M, K), seed=M + 1, lo=lo, hi=hi)
    B = inputs.bf16_integers((N, K), seed=N + 2, lo=lo, hi=hi)
    Ab, Bb = inputs.to_numpy_bits(A), inputs.to_numpy_bits(B)
    cref, cb = oracle.gemm_bf16_exact_integers(Ab, Bb)
    cref2, cb2 = oracle.gemm_bf16(Ab, Bb)
    assert np.array_equal(cb, cb2) and np.array_equal(cref, cref2)
    exact = A.to(torch.int64).numpy() @ B.to(torch.int64).numpy().T
    assert np.array_equal(cref, exact.astype(np.float64))


def test_exact_integer_gemm_refuses_inputs_it_cannot_sum_exactly():
    ok = inputs.to_numpy_bits(inputs.bf16_integers((2, 8), seed=1))
    half = inputs.to_numpy_bits(torch.full((2, 8), 0.5, dtype=torch.bfloat16))
    big = inputs.to_numpy_bits(torch.full((2, 8), 512.0, dtype=torch.bfloat16))
    for bad in (half, big):
        with pytest.raises(ValueError):
            oracle.gemm_bf16_exact_integers(bad, ok)
        with pytest.raises(ValueError):
            oracle.gemm_bf16_exact_integers(ok, bad)


def test_exact_integer_grouped_gemm_equals_the_scalar_oracle():
    E, N, K = 5, 24, 96
    off = np.array([0, 3, 3, 10, 11, 20], dtype=np.int32)   # expert 1 empty, expert 3 one row
    A = inputs.to_numpy_bits(inputs.bf16_integers((20, K), seed=7))
    B = inputs.to_numpy_bits(inputs.bf16_integers((E, N, K), seed=8))
    cref, cb = oracle.grouped_gemm_bf16_exact_integers(A, B, off)
    cref2, cb2 = oracle.grouped_gemm_bf16(A, B, off)
    assert np.array_equal(cb, cb2) and np.array_equal(cref, cref2)
    with pytest.raises(ValueError):
        oracle.grouped_gemm_bf16_exact_integers(A, B, np.array([0, 3, 2, 10, 11, 20], np.int32))
