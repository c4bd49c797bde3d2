"""Helpers shared by the GPU parity and invariance tests.

The tolerance is the elementwise bound on the bf16 result:

    |C - Cref| <= 2^-7 |Cref| + 1e-3 sqrt(K) rms(A) rms(B)

with Cref the oracle's unrounded fp64 sum and rms taken over all entries of the (dequantised)
operands.  2^-7 is one bf16 unit in the last place relative to the value (bf16 keeps 8
significant bits, so RNE alone contributes up to 2^-8 |Cref|; the rest covers the fp32
accumulation, which rounds at most K times by 2^-24 relative to the running sum).  The second
term absorbs cancellation, where |Cref| is small but the partial sums are not.  On inputs where
every partial sum is exact in fp32 (small integers, power-of-two scales) the GPU must instead
match the oracle's bf16 result exactly.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_bits_to_f64(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float32).numpy().astype(np.float64)


def rms(x: np.ndarray) -> float:
    x = np.asarray(x, dtype=np.float64)
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0


def rms_t(t: torch.Tensor, chunk: int = 1 << 24) -> float:
    """rms of a (possibly huge, device-resident) tensor, reduced on its own device in fp64."""
    flat = t.reshape(-1)
    acc = torch.zeros((), dtype=torch.float64, device=t.device)
    for i in range(0, flat.numel(), chunk):
        acc += flat[i:i + chunk].double().pow(2).sum()
    return float((acc / max(flat.numel(), 1)).sqrt())


def tolerance(cref: np.ndarray, K: int, rms_a: float, rms_b: float) -> np.ndarray:
    return 2.0 ** -7 * np.abs(cref) + 1e-3 * math.sqrt(max(K, 1)) * rms_a * rms_b


def assert_within_tolerance(c_bits: np.ndarray, cref: np.ndarray, K: int, rms_a: float,
                            rms_b: float, what: str = ""):
    c = bf16_bits_to_f64(c_bits)
    assert np.all(np.isfinite(c)), f"{what}: non-finite output"
    err = np.abs(c - cref)
    tol = tolerance(cref, K, rms_a, rms_b)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance; first at {tuple(i)}: "
                             f"got {c[tuple(i)]!r}, oracle {cref[tuple(i)]!r}, tol {tol[tuple(i)]!r}")
    return float((err / np.maximum(tol, 1e-300)).max()) if err.size else 0.0


def assert_bits_equal_values(c_bits: np.ndarray, want_bits: np.ndarray, what: str = ""):
    """Bit-exact parity, with +0 and -0 counted equal (the two sides may sign an exact zero
    differently: the oracle's fp64 sum of an exact cancellation is +0)."""
    a = np.asarray(c_bits, dtype=np.uint16)
    b = np.asarray(want_bits, dtype=np.uint16)
    zero = ((a & 0x7FFF) == 0) & ((b & 0x7FFF) == 0)
    diff = (a != b) & ~zero
    if diff.any():
        i = np.argwhere(diff)[0]
        raise AssertionError(f"{what}: {diff.sum()} elements differ; first at {tuple(i)}: "
                             f"{int(a[tuple(i)]):#06x} vs {int(b[tuple(i)]):#06x}")


def bits(t: torch.Tensor) -> np.ndarray:
    """Host uint16 bits of a bf16 tensor."""
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def rows_equal_bitwise(x: torch.Tensor, y: torch.Tensor) -> bool:
    return torch.equal(x.view(torch.int16), y.view(torch.int16))
