"""Readers for the hand-written fixtures under ``tests/golden``."""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if line:
                yield line


def gemm_cases():
    """Yield (name, A, B, C) float64 arrays from gemm_worked.txt."""
    it = _lines("gemm_worked.txt")
    for line in it:
        assert line.startswith("case "), line
        name = line.split()[1]
        mats = {}
        for line in it:
            if line == "end":
                break
            tag, r, c = line.split()
            rows = [[float(Fraction(v)) for v in next(it).split()] for _ in range(int(r))]
            mats[tag] = np.array(rows, dtype=np.float64).reshape(int(r), int(c))
        yield name, mats["A"], mats["B"], mats["C"]


def bf16_rounding_cases():
    """Yield (Fraction value, expected bits, reason)."""
    for line in _lines("bf16_rounding.txt"):
        m, e, bits, *reason = line.split()
        yield Fraction(int(m)) * Fraction(2) ** int(e), int(bits, 16), " ".join(reason)


def e4m3_cases():
    """Yield (code, value as Fraction or None for NaN, negative_zero flag, reason)."""
    for line in _lines("e4m3_codes.txt"):
        code, m, e, *reason = line.split()
        if m == "nan":
            yield int(code, 16), None, False, " ".join(reason)
        else:
            neg_zero = m == "-0"
            val = Fraction(int(m)) * Fraction(2) ** int(e)
            yield int(code, 16), val, neg_zero, " ".join(reason)


def fp8_cases():
    """Yield dicts with M, N, K, qa, qb (uint8 arrays), sa, sb (float32), c (float64)."""
    it = _lines("fp8_worked.txt")
    for line in it:
        parts = line.split()
        assert parts[0] == "case", line
        name, M, N, K = parts[1], int(parts[2]), int(parts[3]), int(parts[4])
        kb, nb = math.ceil(K / 128), math.ceil(N / 128)
        case = {"name": name, "M": M, "N": N, "K": K}
        for line in it:
            if line == "end":
                break
            tag, *vals = line.split()
            if tag == "qa":
                case["qa"] = np.full((M, K), int(vals[0], 16), dtype=np.uint8)
            elif tag == "qb":
                case["qb"] = np.full((N, K), int(vals[0], 16), dtype=np.uint8)
            elif tag == "sa":
                case["sa"] = np.array([float(v) for v in vals], dtype=np.float32).reshape(M, kb)
            elif tag == "sb":
                case["sb"] = np.array([float(v) for v in vals], dtype=np.float32).reshape(nb, kb)
            elif tag == "c":
                case["c"] = np.array([float(v) for v in vals], dtype=np.float64).reshape(M, N)
            elif tag == "c_pattern":
                out = []
                for v, cnt in zip(vals[0::2], vals[1::2]):
                    out += [float(v)] * int(cnt)
                case["c"] = np.array(out, dtype=np.float64).reshape(M, N)
        yield case


def e2m1_cases():
    """Yield (code, value as Fraction, negative_zero flag, reason) from e2m1_codes.txt."""
    for line in _lines("e2m1_codes.txt"):
        code, m, e, *reason = line.split()
        yield int(code, 16), Fraction(int(m)) * Fraction(2) ** int(e), m == "-0", " ".join(reason)


def pack_e2m1(codes: np.ndarray) -> np.ndarray:
    """[rows, K] 4-bit codes -> [rows, K/2] bytes, value k in byte k//2, even k in the low bits."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def w4a8_cases():
    """Yield dicts with qa (uint8 [M,K]), sa (float32 [M,KB]), qw (packed uint8 [N,K/2]),
    scale (float32 [N]), zero (float32 [N] or None) and c (float64 [M,N]) from w4a8_worked.txt."""
    it = _lines("w4a8_worked.txt")
    for line in it:
        parts = line.split()
        assert parts[0] == "case", line
        name, M, N, K = parts[1], int(parts[2]), int(parts[3]), int(parts[4])
        kb = math.ceil(K / 128)
        qa = np.zeros((M, K), np.uint8)
        codes = np.zeros((N, K), np.uint8)
        case = {"name": name, "M": M, "N": N, "K": K, "zero": None}
        for line in it:
            if line == "end":
                break
            tag, *vals = line.split()
            if tag == "a":
                qa[int(vals[0]), int(vals[1])] = int(vals[2], 16)
            elif tag == "w":
                codes[int(vals[0]), int(vals[1])] = int(vals[2], 16)
            elif tag == "sa":
                case["sa"] = np.array([float(v) for v in vals], dtype=np.float32).reshape(M, kb)
            elif tag == "scale":
                case["scale"] = np.array([float(v) for v in vals], dtype=np.float32)
            elif tag == "zero":
                if vals != ["none"]:
                    case["zero"] = np.array([float(v) for v in vals], dtype=np.float32)
            elif tag == "c":
                case["c"] = np.array([float(v) for v in vals], dtype=np.float64).reshape(M, N)
        case["qa"] = qa
        case["qw"] = pack_e2m1(codes)
        yield case


def e2m1_rounding_cases():
    """Yield (x as float, expected code, reason) from e2m1_rounding.txt."""
    for line in _lines("e2m1_rounding.txt"):
        m, e, code, *reason = line.split()
        if m in ("nan", "inf", "-inf"):
            x = float(m)
        else:
            x = float(Fraction(int(m)) * Fraction(2) ** int(e))
        yield x, int(code, 16), " ".join(reason)
