"""Plant plausible mistakes in a temporary copy of the oracle and check that the pins catch each.

The oracle source itself is never edited: every mutant is a text substitution applied to a copy
under pytest's tmp_path, compiled with the oracle's own flags and loaded through ctypes.  The
battery below re-runs the independent pins (hand-worked golden cases, closed forms, exact
rationals); a mutant survives only if all of them still pass, which fails this test.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests import exact, golden_io

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "bi_oracle.c")

MUTANTS = {
    "B read transposed": ("s += arow[kk] * brow[kk];",
                          "s += arow[kk] * bmat[kk * j->n_cols + n];"),
    "last K term dropped": ("for (int64_t kk = 0; kk < j->k; ++kk)",
                            "for (int64_t kk = 0; kk + 1 < j->k; ++kk)"),
    "first K term dropped": ("for (int64_t kk = 0; kk < j->k; ++kk)",
                             "for (int64_t kk = 1; kk < j->k; ++kk)"),
    "bf16 sign ignored": ("    return sign ? -v : v;\n}\n\n/* e4m3",
                          "    return v;\n}\n\n/* e4m3"),
    "double rounding through fp32": ("oracle_f64_to_bf16_rne(s)",
                                     "oracle_f64_to_bf16_rne((double)(float)s)"),
    "truncating instead of rounding": ("double r = nearbyint(n);", "double r = floor(n);"),
    "ties away from zero": ("double r = nearbyint(n);", "double r = round(n);"),
    "bf16 subnormal exponent off by one": ("ldexp((double)frac, -126 - 7)",
                                           "ldexp((double)frac, -127 - 7)"),
    "e4m3 bias 8": ("ldexp((double)(8 + frac), expo - 7 - 3)",
                    "ldexp((double)(8 + frac), expo - 8 - 3)"),
    "e4m3 subnormal scale": ("ldexp((double)frac, -9)", "ldexp((double)frac, -10)"),
    "A scale of the first K block only": ("(double)SA[m * kb + k / 128]", "(double)SA[m * kb]"),
    "B scale indexed by row, not row block": ("(double)SB[(n / 128) * kb + k / 128]",
                                               "(double)SB[(n % 2) * kb + k / 128]"),
    "B scale ignored": ("* (double)SB[(n / 128) * kb + k / 128]", ""),
    "e2m1 nibbles swapped": ("(k % 2 == 0) ? (uint8_t)(byte & 0xF) : (uint8_t)(byte >> 4)",
                             "(k % 2 == 1) ? (uint8_t)(byte & 0xF) : (uint8_t)(byte >> 4)"),
    "e2m1 bias 2": ("ldexp((double)(2 + frac), expo - 1 - 1)", "ldexp((double)(2 + frac), expo - 2 - 1)"),
    "e2m1 sign ignored": ("    return sign ? -v : v;\n}\n\n/* fp16 bit pattern",
                          "    return v;\n}\n\n/* fp16 bit pattern"),
    "fp16 sign ignored": ("    return sign ? -v : v;\n}\n\n/* fp64 -> e2m1",
                          "    return v;\n}\n\n/* fp64 -> e2m1"),
    "e2m1 zero point scaled": ("w += (double)WZ[n];", "w += (double)WZ[n] * (double)WS[n];"),
    "e2m1 zero point ignored": ("w += (double)WZ[n];", "w += 0.0;"),
    "e2m1 scale of channel 0": ("oracle_e2m1_to_f64(code) * (double)WS[n]",
                                "oracle_e2m1_to_f64(code) * (double)WS[0]"),
    "e2m1 rounding ties away from zero": ("double v = nearbyint(a / q) * q;", "double v = round(a / q) * q;"),
    "e2m1 rounding truncates": ("double v = nearbyint(a / q) * q;", "double v = floor(a / q) * q;"),
    "e2m1 no saturation": ("    if (v > 6.0)\n        v = 6.0;\n", ""),
    "e2m1 rounding drops the sign": ("uint8_t sign = signbit(x) ? 8 : 0;", "uint8_t sign = 0;"),
    "quantise ignores the zero point": ("double z = WZ ? (double)WZ[n] : 0.0;", "double z = 0.0;"),
    "quantise multiplies by the scale": ("code[h] = oracle_f64_to_e2m1((w - z) / (double)WS[n]);",
                                         "code[h] = oracle_f64_to_e2m1((w - z) * (double)WS[n]);"),
    "quantise packs high nibble first": ("(uint8_t)(code[0] | (code[1] << 4))",
                                         "(uint8_t)(code[1] | (code[0] << 4))"),
    "fp16 bias 16": ("ldexp((double)(1024 + frac), expo - 15 - 10)", "ldexp((double)(1024 + frac), expo - 16 - 10)"),
    "grouped rows use expert 0": ("row_b[r] = e * N * K;", "row_b[r] = 0;"),
    "grouped rows use the next expert": ("row_b[r] = e * N * K;",
                                         "row_b[r] = ((e + 1) % E) * N * K;"),
}


def bf16_bits(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def bf16_values(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).astype(np.uint32).view(np.float32) \
        .astype(np.float64)


def e4m3_values(codes):
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8).copy()).view(torch.float8_e4m3fn) \
        .to(torch.float32).numpy().astype(np.float64)


def battery(lib):
    """Return the list of pin names that fail for this oracle build."""
    failed = []

    def check(name, cond):
        if not cond:
            failed.append(name)

    # golden GEMM cases
    ok = True
    for _, A, B, C in golden_io.gemm_cases():
        _, cb = oracle.gemm_bf16(bf16_bits(A), bf16_bits(B), lib=lib)
        ok &= np.array_equal(bf16_values(cb), C)
    check("golden gemm", ok)

    # bf16 rounding golden + decode table
    ok = all(int(oracle.f64_to_bf16(np.array([float(v)]), lib=lib)[0]) == b
             for v, b, _ in golden_io.bf16_rounding_cases())
    check("golden bf16 rounding", ok)
    bits = np.arange(0, 1 << 16, 97, dtype=np.uint32)
    ref = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    got = oracle.bf16_to_f64(bits.astype(np.uint16), lib=lib)
    fin = np.isfinite(ref)
    check("bf16 decode vs bit view", np.array_equal(got[fin], ref[fin]))

    # e4m3 table
    codes = np.arange(256, dtype=np.uint8)
    want = e4m3_values(codes)
    got = oracle.e4m3_to_f64(codes, lib=lib)
    nan = np.isnan(want)
    check("e4m3 decode vs torch", np.array_equal(got[~nan], want[~nan]))

    # rank-1 closed form, non-square
    rng = np.random.default_rng(5)
    u, v = rng.integers(-3, 4, 7), rng.integers(-3, 4, 11)
    x, y = rng.integers(-4, 5, 13), rng.integers(-4, 5, 13)
    cref, _ = oracle.gemm_bf16(bf16_bits(np.outer(u, x)), bf16_bits(np.outer(v, y)), lib=lib)
    check("rank-1", np.array_equal(cref, float(x @ y) * np.outer(u, v)))

    # brute force with exact rationals
    ok = True
    for seed in range(3):
        r = np.random.default_rng(200 + seed)
        A = bf16_bits(r.standard_normal((4, 7)) * np.exp2(r.integers(-6, 7, (4, 7))))
        B = bf16_bits(r.standard_normal((5, 7)) * np.exp2(r.integers(-6, 7, (5, 7))))
        _, cb = oracle.gemm_bf16(A, B, lib=lib)
        C = exact.exact_gemm(bf16_values(A), bf16_values(B))
        ok &= all(cb[m, n] == exact.rne_bf16(C[m][n]) for m in range(4) for n in range(5))
    check("brute force", ok)

    # FP8 golden + power-of-two scales closed form across two N blocks
    ok = True
    for case in golden_io.fp8_cases():
        _, cb = oracle.gemm_fp8_blockscaled(case["qa"], case["qb"], case["sa"], case["sb"], lib=lib)
        ok &= np.array_equal(bf16_values(cb), case["c"])
    check("golden fp8", ok)
    r = np.random.default_rng(9)
    qa = torch.from_numpy(r.integers(-4, 5, (3, 256)).astype(np.float32)) \
        .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    qb = torch.from_numpy(r.integers(-4, 5, (200, 256)).astype(np.float32)) \
        .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    sa = np.exp2(r.integers(-4, 5, (3, 2))).astype(np.float32)
    sb = np.exp2(r.integers(-4, 5, (2, 2))).astype(np.float32)
    cref, _ = oracle.gemm_fp8_blockscaled(qa, qb, sa, sb, lib=lib)
    va, vb = e4m3_values(qa), e4m3_values(qb)
    ok = True
    for m in range(3):
        for n in range(200):
            q = sum(Fraction(float(va[m, k * 128:(k + 1) * 128] @ vb[n, k * 128:(k + 1) * 128]))
                    * Fraction(float(sa[m, k])) * Fraction(float(sb[n // 128, k])) for k in range(2))
            ok &= cref[m, n] == float(q)
    check("fp8 pow2 closed form", ok)

    # e2m1 table and the worked W4A8 cases
    got = oracle.e2m1_to_f64(np.arange(16, dtype=np.uint8), lib=lib)
    ok = all(got[c] == float(v) and (v != 0 or bool(np.signbit(got[c])) == nz)
             for c, v, nz, _ in golden_io.e2m1_cases())
    check("e2m1 table", ok)
    ok = True
    for case in golden_io.w4a8_cases():
        cref, _ = oracle.gemm_w4a8(case["qa"], case["sa"], case["qw"], case["scale"], case["zero"],
                                   lib=lib)
        ok &= np.array_equal(cref, case["c"])
    check("golden w4a8", ok)
    # zero point: all-zero codes give C = zero[n] * rowsum(a)[m]; a second channel scale differs
    r = np.random.default_rng(13)
    qa = torch.from_numpy(r.integers(-4, 5, (2, 128)).astype(np.float32)) \
        .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    sa = np.exp2(r.integers(-2, 3, (2, 1))).astype(np.float32)
    ws = np.array([0.5, 0.125, 0.25], np.float32)
    wz = np.array([0.25, -0.75, 1.5], np.float32)
    cref, _ = oracle.gemm_w4a8(qa, sa, np.zeros((3, 64), np.uint8), ws, wz, lib=lib)
    rs = (e4m3_values(qa) * sa.astype(np.float64)).sum(axis=1)
    check("w4a8 zero-point closed form", np.array_equal(cref, np.outer(rs, wz.astype(np.float64))))

    # e2m1 rounding golden cases, fp16 decode, and a quantisation worked by hand
    ok = all(int(oracle.f64_to_e2m1([x], lib=lib)[0]) == c for x, c, _ in golden_io.e2m1_rounding_cases())
    check("e2m1 rounding golden", ok)
    hb = np.arange(0, 1 << 16, 61, dtype=np.uint32).astype(np.uint16)
    hv = hb.view(np.float16).astype(np.float64)
    hg = oracle.fp16_to_f64(hb, lib=lib)
    fin = np.isfinite(hv)
    check("fp16 decode vs numpy", np.array_equal(hg[fin], hv[fin]))
    Wq = np.array([[2.0, -0.25, 0.5, 1.875], [0.25, 0.375, -1.0, 8.0]], np.float32)
    bq = torch.from_numpy(Wq).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.quantize_e2m1(bq, np.array([0.25, 0.5], np.float32), np.array([0.5, 0.0], np.float32),
                               lib=lib)
    want = golden_io.pack_e2m1(np.array([[0x7, 0xD, 0x0, 0x7], [0x1, 0x2, 0xC, 0x7]], np.uint8))
    check("quantise worked case", np.array_equal(got, want))

    # grouped: integer data, distinct experts, one empty
    E, N, K = 3, 4, 8
    off = np.array([0, 2, 2, 5], np.int32)
    A = bf16_bits(np.random.default_rng(3).integers(-4, 5, (5, K)))
    B = bf16_bits(np.stack([np.eye(N, K) * (e + 1) for e in range(E)]))
    cref, _ = oracle.grouped_gemm_bf16(A, B, off, lib=lib)
    va = bf16_values(A)
    ok = all(np.array_equal(cref[r], (e + 1) * va[r, :N])
             for e in range(E) for r in range(off[e], off[e + 1]))
    check("grouped segments", ok)
    return failed


def test_unmutated_oracle_passes_the_battery():
    assert battery(oracle.OracleLib(oracle.build())) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) >= 1, f"mutation site for {name!r} no longer exists"
    mutated = tmp_path / "bi_oracle_mutant.c"
    mutated.write_text(src.replace(old, new, 1), encoding="utf-8")
    so = oracle.compile_copy(str(mutated), str(tmp_path / "libmutant.so"))
    failed = battery(oracle.OracleLib(so))
    assert failed, f"mutant {name!r} passed every pin"
