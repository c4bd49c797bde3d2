"""Pins for the oracle's e2m1-weight x e4m3-activation GEMM and its e2m1 codec.

The GEMM follows the weight quantisation of "DeepSeek V4的batch invariance：大模型确定性推理的工程
基石" (lshu.cn), section 4.3: W = q * scale + zero per output channel, scale a power of two.  The
pins compare the oracle with hand-derived values (the e2m1 table, worked cases), with the FP8
oracle (itself pinned) on weights that e4m3 holds exactly, with the closed form of the zero-point
term, and with exact rational brute force.  A swapped nibble order, a scale or zero point on the
wrong index, a zero point multiplied by the scale, or a dropped sign fails at least one of them.
"""
from fractions import Fraction

import numpy as np
import torch

import oracle
from invariant_deterministic_gemm_bi_b200 import inputs
from tests import exact, golden_io


def bf16_values(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).astype(np.uint32).view(np.float32) \
        .astype(np.float64)


def e4m3_values(codes):
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8).copy()).view(torch.float8_e4m3fn) \
        .to(torch.float32).numpy().astype(np.float64)


E2M1_TABLE = {code: (val, neg) for code, val, neg, _ in golden_io.e2m1_cases()}


def unpack(qw: np.ndarray) -> np.ndarray:
    """Packed [rows, K/2] -> codes [rows, K] (test-side, low four bits first)."""
    out = np.empty((qw.shape[0], qw.shape[1] * 2), np.uint8)
    out[:, 0::2] = qw & 0xF
    out[:, 1::2] = qw >> 4
    return out


def table_values(codes: np.ndarray) -> np.ndarray:
    lut = np.array([float(E2M1_TABLE[c][0]) for c in range(16)], dtype=np.float64)
    return lut[codes]


def test_e2m1_decode_matches_the_hand_derived_table():
    assert sorted(E2M1_TABLE) == list(range(16))
    got = oracle.e2m1_to_f64(np.arange(16, dtype=np.uint8))
    for code, (val, neg_zero) in E2M1_TABLE.items():
        assert got[code] == float(val), hex(code)
        if val == 0:
            assert bool(np.signbit(got[code])) == neg_zero, hex(code)


def test_e2m1_magnitudes_increase_and_bit3_is_the_sign():
    got = oracle.e2m1_to_f64(np.arange(16, dtype=np.uint8))
    assert np.all(np.diff(got[:8]) > 0)
    assert np.array_equal(got[8:], -got[:8])
    # every e2m1 value is an e4m3 value (the reduction below relies on it)
    as_e4m3 = torch.from_numpy(got.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64)
    assert np.array_equal(as_e4m3.numpy(), got)


def test_w4a8_golden_worked_examples():
    n = 0
    for case in golden_io.w4a8_cases():
        cref, cbits = oracle.gemm_w4a8(case["qa"], case["sa"], case["qw"], case["scale"], case["zero"])
        assert np.array_equal(cref, case["c"]), case["name"]
        assert np.array_equal(bf16_values(cbits), case["c"]), case["name"]
        n += 1
    assert n >= 2


def test_w4a8_without_zero_points_is_the_fp8_gemm_of_the_scaled_weights():
    # q * 2^-j (j <= 4) is an e4m3 value, so the weights can be handed to the FP8 oracle as
    # e4m3 codes with unit block scales; the two oracles must then agree exactly.
    M, N, K = 5, 150, 384
    qa = inputs.to_numpy_bits(inputs.e4m3_gaussian((M, K), seed=611))
    sa = inputs.scales_log_uniform((M, 3), seed=612).numpy()
    qw = inputs.e2m1_packed_uniform(N, K, seed=613).numpy()
    ws = inputs.channel_scales_pow2(N, seed=614, lo=1, hi=4).numpy()
    w = table_values(unpack(qw)) * ws[:, None].astype(np.float64)
    qb = torch.from_numpy(w.astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(qb.to(torch.float64).numpy(), w)
    sb = np.ones(((N + 127) // 128, 3), np.float32)
    want_ref, want_bits = oracle.gemm_fp8_blockscaled(qa, qb.view(torch.uint8).numpy(), sa, sb)
    cref, cbits = oracle.gemm_w4a8(qa, sa, qw, ws, None)
    assert np.array_equal(cref, want_ref)
    assert np.array_equal(cbits, want_bits)


def test_w4a8_zero_point_adds_zero_times_the_activation_row_sum():
    M, N, K = 4, 40, 256
    qa = inputs.to_numpy_bits(inputs.e4m3_integers((M, K), seed=621))
    sa = inputs.scales_pow2((M, 2), seed=622).numpy()
    qw = inputs.e2m1_packed_uniform(N, K, seed=623).numpy()
    ws = inputs.channel_scales_pow2(N, seed=624).numpy()
    wz = inputs.channel_zeros_grid(N, seed=625).numpy()
    base, _ = oracle.gemm_w4a8(qa, sa, qw, ws, None)
    with_z, _ = oracle.gemm_w4a8(qa, sa, qw, ws, wz)
    a = e4m3_values(qa) * np.repeat(sa.astype(np.float64), 128, axis=1)
    rowsum = a.sum(axis=1)                 # exact: small integers times powers of two
    # every product is a multiple of 2^-17 and every sum below 2^17, so fp64 holds both exactly
    assert np.array_equal(with_z - base, np.outer(rowsum, wz.astype(np.float64)))
    # all-zero codes leave the zero point alone: C = zero * rowsum
    zq = np.zeros_like(qw)
    only_z, _ = oracle.gemm_w4a8(qa, sa, zq, ws, wz)
    assert np.array_equal(only_z, np.outer(rowsum, wz.astype(np.float64)))


def test_w4a8_brute_force_exact_rationals():
    rng = np.random.default_rng(631)
    M, N, K = 3, 5, 256
    qa = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)) \
        .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    sa = np.exp2(rng.integers(-3, 4, (M, 2))).astype(np.float32)
    codes = rng.integers(0, 16, (N, K)).astype(np.uint8)
    qw = golden_io.pack_e2m1(codes)
    ws = np.exp2(-rng.integers(1, 13, N)).astype(np.float32)
    wz = torch.from_numpy(rng.standard_normal(N).astype(np.float32) * ws).to(torch.float16) \
        .to(torch.float32).numpy()
    cref, cbits = oracle.gemm_w4a8(qa, sa, qw, ws, wz)
    va = e4m3_values(qa)
    for m in range(M):
        for n in range(N):
            q = Fraction(0)
            for k in range(K):
                av = Fraction(float(va[m, k])) * Fraction(float(sa[m, k // 128]))
                wv = E2M1_TABLE[int(codes[n, k])][0] * Fraction(float(ws[n])) + Fraction(float(wz[n]))
                q += av * wv
            assert abs(Fraction(float(cref[m, n])) - q) <= abs(q) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)
            assert cbits[m, n] == exact.rne_bf16(q), (m, n)


# ---------------------------------------------------------------------------------------------
# e2m1 quantisation of 16-bit weights: W_fp4 = round((W - zero) / scale)
# ---------------------------------------------------------------------------------------------

def test_e2m1_rounding_golden_cases():
    n = 0
    for x, code, why in golden_io.e2m1_rounding_cases():
        assert int(oracle.f64_to_e2m1([x])[0]) == code, (x, why)
        n += 1
    assert n >= 15


def test_e2m1_rounding_round_trips_every_value():
    vals = [float(v) if not neg else -0.0 for _, (v, neg) in sorted(E2M1_TABLE.items())]
    codes = oracle.f64_to_e2m1(vals)
    assert list(codes) == list(range(16))


def test_e2m1_rounding_is_nearest_with_ties_to_even_brute_force():
    rng = np.random.default_rng(641)
    xs = list(rng.uniform(-9, 9, 400))
    # every midpoint between neighbouring values, and both of its neighbours in binary64
    mags = [float(E2M1_TABLE[c][0]) for c in range(8)]
    for a, b in zip(mags, mags[1:]):
        mid = (a + b) / 2
        xs += [mid, np.nextafter(mid, 0), np.nextafter(mid, 9), -mid]
    got = oracle.f64_to_e2m1(xs)
    for x, c in zip(xs, got):
        fx = Fraction(float(x))
        cands = sorted(range(8), key=lambda cc: (abs(abs(fx) - E2M1_TABLE[cc][0]), cc & 1))
        want = cands[0] if abs(fx) <= 6 else 7
        if fx < 0 or (fx == 0 and np.signbit(x)):
            want |= 8
        assert int(c) == want, (x, int(c), want)


def test_fp16_decode_exhaustive_vs_numpy_bit_view():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    want = bits.view(np.float16).astype(np.float64)
    got = oracle.fp16_to_f64(bits)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def test_quantize_applies_zero_then_scale_and_packs_low_nibble_first():
    # row 0: scale 2^-2, zero 0.5: (W - 0.5) * 4 for W = [2, -0.25, 0.5, 1.875] -> [6, -3, 0, 5.5]
    #   -> codes [0x7, 0xD, 0x0, 0x7 (5.5 is nearer 6)]
    # row 1: scale 2^-1, no zero point effect (zero 0): W = [0.25, 0.375, -1, 8] -> [0.5, 0.75, -2, 16]
    #   -> codes [0x1, 0x2 (tie -> 1), 0xC, 0x7]
    W = np.array([[2.0, -0.25, 0.5, 1.875], [0.25, 0.375, -1.0, 8.0]], np.float32)
    ws = np.array([0.25, 0.5], np.float32)
    wz = np.array([0.5, 0.0], np.float32)
    want = golden_io.pack_e2m1(np.array([[0x7, 0xD, 0x0, 0x7], [0x1, 0x2, 0xC, 0x7]], np.uint8))
    bf = torch.from_numpy(W).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.quantize_e2m1(bf, ws, wz), want)
    hf = W.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.quantize_e2m1(hf, ws, wz, fp16=True), want)


def test_quantize_then_gemm_reproduces_exactly_representable_weights():
    # weights that are e2m1 values times the channel scale plus its zero point quantise to those
    # values, so quantise -> W4A8 GEMM equals the W4A8 GEMM of the original codes
    N, K = 20, 256
    codes = np.random.default_rng(651).integers(0, 16, (N, K)).astype(np.uint8)
    ws = np.exp2(-np.random.default_rng(652).integers(1, 5, N)).astype(np.float32)
    wz = (np.random.default_rng(653).integers(-8, 9, N) * 2.0 ** -3).astype(np.float32)
    w = table_values(codes) * ws[:, None].astype(np.float64) + wz[:, None].astype(np.float64)
    bf = torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(bf.to(torch.float64).numpy(), w)        # exact in bf16
    q = oracle.quantize_e2m1(bf.view(torch.int16).numpy().view(np.uint16), ws, wz)
    vals = table_values(unpack(q))
    assert np.array_equal(vals, table_values(codes))              # -0 and +0 both decode to 0
