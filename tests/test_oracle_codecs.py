"""Pins for the oracle's codecs (bf16 decode/encode, e4m3 decode).

Each codec is checked against something other than itself: hand-derived golden values, a
numpy bit view, torch's own conversions, and an exact round-to-nearest-even by table lookup.
"""
import math
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests import exact, golden_io


def test_bf16_decode_exhaustive_vs_numpy_bit_view():
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    ref = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    got = oracle.bf16_to_f64(bits.astype(np.uint16))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_encode_roundtrips_every_pattern():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_to_f64(bits)
    back = oracle.f64_to_bf16(vals)
    finite_or_inf = ~np.isnan(vals)
    assert np.array_equal(back[finite_or_inf], bits[finite_or_inf])
    # every NaN encodes to a NaN pattern of the same sign
    nanback = back[~finite_or_inf]
    assert np.all((nanback & 0x7F80) == 0x7F80) and np.all((nanback & 0x007F) != 0)


def test_bf16_encode_golden_cases():
    for value, want, reason in golden_io.bf16_rounding_cases():
        got = int(oracle.f64_to_bf16(np.array([float(value)]))[0])
        assert got == want, f"{reason}: got {got:#06x}, want {want:#06x}"
        # the golden values are themselves checked by the exact table lookup
        assert exact.rne_bf16(value) == want, reason


def test_bf16_encode_matches_torch_on_random_fp32():
    rng = np.random.default_rng(7)
    raw = rng.integers(0, 1 << 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    x = raw.view(np.float32)
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_encode_matches_exact_rne_on_random_fp64():
    rng = random.Random(11)
    for _ in range(3000):
        # fp64 values with more precision than fp32, across the whole bf16 range
        e = rng.randint(-140, 130)
        m = rng.getrandbits(53) | (1 << 52)
        v = math.ldexp(m, e - 52) * (1 if rng.random() < 0.5 else -1)
        want = exact.rne_bf16(Fraction(v))
        got = int(oracle.f64_to_bf16(np.array([v]))[0])
        assert got == want, (v, hex(got), hex(want))
    # exact halfway points between neighbours, both parities
    for b in list(range(0, 0x7F7F, 977)) + [0x7F7E]:
        lo, hi = exact.bf16_bits_to_fraction(b), exact.bf16_bits_to_fraction(b + 1)
        mid = (lo + hi) / 2
        want = b if b % 2 == 0 else b + 1
        assert int(oracle.f64_to_bf16(np.array([float(mid)]))[0]) == want


def test_e4m3_decode_golden_cases():
    for code, value, neg_zero, reason in golden_io.e4m3_cases():
        got = float(oracle.e4m3_to_f64(np.array([code], dtype=np.uint8))[0])
        if value is None:
            assert math.isnan(got), reason
        else:
            assert got == float(value), reason
            if value == 0:
                assert math.copysign(1.0, got) == (-1.0 if neg_zero else 1.0), reason


def test_e4m3_decode_exhaustive_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    got = oracle.e4m3_to_f64(codes)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert nan.sum() == 2  # 0x7F and 0xFF only
    assert np.array_equal(got[~nan], want[~nan].astype(np.float64))
    assert np.nanmax(got) == 448.0 and np.nanmin(got) == -448.0


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_bf16_encode_specials(bad):
    got = int(oracle.f64_to_bf16(np.array([bad]))[0])
    if np.isnan(bad):
        assert (got & 0x7F80) == 0x7F80 and (got & 0x7F) != 0
    else:
        assert got == (0x7F80 if bad > 0 else 0xFF80)
