"""CPU oracle for the batch-invariant GEMM -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this module.  The product package never imports it and has no fallback onto it.

This is a thin ctypes wrapper around ``bi_oracle.c`` (plain C, fp64 accumulation, one RNE
rounding to bf16 at the end).  Inputs are numpy arrays of raw bit patterns (``uint16`` for
bf16, ``uint8`` for e4m3) plus fp32 scales; outputs are the unrounded fp64 sums and the bf16
bit patterns.  See ``bi_oracle.c`` for the definitions and the passages they follow.

Every function here is pinned by ``tests/test_oracle_*.py`` against closed forms, library
routines and exact rational brute force; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bi_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_LIB = None


def build(force: bool = False) -> str:
    """Compile ``bi_oracle.c`` into ``liboracle.so`` next to it (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_copy(_SRC, _LIB_PATH + ".tmp")
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


class OracleLib:
    """ctypes view of one built copy of ``bi_oracle.c`` (the default one, or a test's copy)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_f64_to_bf16_rne.restype = ctypes.c_uint16
        lib.oracle_f64_to_bf16_rne.argtypes = [ctypes.c_double]
        lib.oracle_bf16_to_f64_array.restype = None
        lib.oracle_bf16_to_f64_array.argtypes = [vp, vp, i64]
        lib.oracle_e4m3_to_f64_array.restype = None
        lib.oracle_e4m3_to_f64_array.argtypes = [vp, vp, i64]
        lib.oracle_f64_to_bf16_rne_array.restype = None
        lib.oracle_f64_to_bf16_rne_array.argtypes = [vp, vp, i64]
        lib.oracle_gemm_bf16.restype = i32
        lib.oracle_gemm_bf16.argtypes = [i64, i64, i64, vp, vp, vp, vp, i32]
        lib.oracle_gemm_fp8_blockscaled.restype = i32
        lib.oracle_gemm_fp8_blockscaled.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, i32]
        lib.oracle_e2m1_to_f64.restype = ctypes.c_double
        lib.oracle_e2m1_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_fp16_to_f64.restype = ctypes.c_double
        lib.oracle_fp16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f64_to_e2m1.restype = ctypes.c_uint8
        lib.oracle_f64_to_e2m1.argtypes = [ctypes.c_double]
        lib.oracle_quantize_e2m1.restype = None
        lib.oracle_quantize_e2m1.argtypes = [i64, i64, vp, i32, vp, vp, vp]
        lib.oracle_gemm_w4a8.restype = i32
        lib.oracle_gemm_w4a8.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, i32]
        lib.oracle_grouped_gemm_bf16.restype = i32
        lib.oracle_grouped_gemm_bf16.argtypes = [i64, i64, i64, i64, vp, vp, vp, vp, vp, i32]
        self.c = lib
        self.path = path

    def __getattr__(self, name):
        return getattr(self.c, name)


def compile_copy(src: str, out_path: str) -> str:
    """Compile a (possibly edited) copy of the oracle source with the oracle's own flags."""
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
           "-pthread", src, "-o", out_path, "-lm"]
    subprocess.run(cmd, check=True)
    return out_path


def _lib():
    global _LIB
    if _LIB is None:
        build()
        _LIB = OracleLib(_LIB_PATH)
    return _LIB


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------------------------------------
# codecs (scalar, and over whole arrays by looping in C one element at a time)
# ---------------------------------------------------------------------------------------------

def bf16_to_f64(bits, lib=None) -> np.ndarray:
    """bf16 bit patterns -> exact fp64 values (oracle codec, applied element by element in C)."""
    lib = lib or _lib()
    b = np.asarray(bits, dtype=np.uint16)
    flat = np.ascontiguousarray(b.reshape(-1))
    out = np.empty(b.shape, dtype=np.float64)
    lib.oracle_bf16_to_f64_array(_ptr(flat), _ptr(out), flat.size)
    return out


def e4m3_to_f64(bits, lib=None) -> np.ndarray:
    """e4m3 (fn) bit patterns -> exact fp64 values (oracle codec, element by element in C)."""
    lib = lib or _lib()
    b = np.asarray(bits, dtype=np.uint8)
    flat = np.ascontiguousarray(b.reshape(-1))
    out = np.empty(b.shape, dtype=np.float64)
    lib.oracle_e4m3_to_f64_array(_ptr(flat), _ptr(out), flat.size)
    return out


def e2m1_to_f64(codes, lib=None) -> np.ndarray:
    """e2m1 4-bit codes (one per array element, values 0..15) -> exact fp64 values."""
    lib = lib or _lib()
    b = np.asarray(codes, dtype=np.uint8)
    out = np.empty(b.shape, dtype=np.float64)
    flat, oflat = b.reshape(-1), out.reshape(-1)
    for i in range(flat.size):
        oflat[i] = lib.oracle_e2m1_to_f64(int(flat[i]))
    return out


def fp16_to_f64(bits, lib=None) -> np.ndarray:
    """fp16 bit patterns -> exact fp64 values (oracle codec)."""
    lib = lib or _lib()
    b = np.asarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    flat, oflat = b.reshape(-1), out.reshape(-1)
    for i in range(flat.size):
        oflat[i] = lib.oracle_fp16_to_f64(int(flat[i]))
    return out


def f64_to_e2m1(x, lib=None) -> np.ndarray:
    """fp64 values -> e2m1 codes (round to nearest even, saturating at +-6, NaN -> +0)."""
    lib = lib or _lib()
    v = np.asarray(x, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    flat, oflat = v.reshape(-1), out.reshape(-1)
    for i in range(flat.size):
        oflat[i] = lib.oracle_f64_to_e2m1(float(flat[i]))
    return out


def quantize_e2m1(W_bits, w_scale, w_zero=None, fp16: bool = False, lib=None) -> np.ndarray:
    """Quantise 16-bit weights [N, K] (bf16 bits, or fp16 bits with fp16=True) to packed e2m1
    codes [N, K/2]: q = round_to_nearest_even((W - zero) / scale), saturating at +-6."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    assert K % 2 == 0
    WS = _c(w_scale, np.float32).reshape(N)
    WZ = None if w_zero is None else _c(w_zero, np.float32).reshape(N)
    Q = np.empty((N, K // 2), dtype=np.uint8)
    (lib or _lib()).oracle_quantize_e2m1(N, K, _ptr(W), 1 if fp16 else 0, _ptr(WS),
                                         None if WZ is None else _ptr(WZ), _ptr(Q))
    return Q


def f64_to_bf16(x, lib=None) -> np.ndarray:
    """fp64 values -> bf16 bit patterns, round to nearest even (oracle codec, element by element
    in C)."""
    lib = lib or _lib()
    v = np.asarray(x, dtype=np.float64)
    flat = np.ascontiguousarray(v.reshape(-1))
    out = np.empty(v.shape, dtype=np.uint16)
    lib.oracle_f64_to_bf16_rne_array(_ptr(flat), _ptr(out), flat.size)
    return out


# ---------------------------------------------------------------------------------------------
# GEMMs
# ---------------------------------------------------------------------------------------------

def gemm_bf16(A_bits: np.ndarray, B_bits: np.ndarray, threads: int | None = None, lib=None):
    """C = A . B^T for bf16 A [M,K], B [N,K].  Returns (cref fp64 [M,N], c bf16 bits [M,N])."""
    A = _c(A_bits, np.uint16)
    B = _c(B_bits, np.uint16)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2, "A and B disagree on K"
    cref = np.empty((M, N), dtype=np.float64)
    cbits = np.empty((M, N), dtype=np.uint16)
    rc = (lib or _lib()).oracle_gemm_bf16(M, N, K, _ptr(A), _ptr(B), _ptr(cref), _ptr(cbits),
                                 threads or default_threads())
    if rc != 0:
        raise MemoryError("oracle_gemm_bf16 failed")
    return cref, cbits


def gemm_fp8_blockscaled(QA_bits, QB_bits, SA, SB, threads: int | None = None, lib=None):
    """FP8 e4m3 block-scaled C = deq(A) . deq(B)^T.

    QA [M,K] and QB [N,K] are e4m3 bit patterns; SA is fp32 [M, ceil(K/128)] (one scale per
    row and 128-wide K block); SB is fp32 [ceil(N/128), ceil(K/128)] (one scale per 128x128
    block).  Returns (cref fp64 [M,N], c bf16 bits [M,N]).
    """
    QA = _c(QA_bits, np.uint8)
    QB = _c(QB_bits, np.uint8)
    M, K = QA.shape
    N, K2 = QB.shape
    assert K == K2
    kb = (K + 127) // 128
    SA = _c(SA, np.float32)
    SB = _c(SB, np.float32)
    assert SA.shape == (M, kb), SA.shape
    assert SB.shape == ((N + 127) // 128, kb), SB.shape
    cref = np.empty((M, N), dtype=np.float64)
    cbits = np.empty((M, N), dtype=np.uint16)
    rc = (lib or _lib()).oracle_gemm_fp8_blockscaled(M, N, K, _ptr(QA), _ptr(QB), _ptr(SA), _ptr(SB),
                                            _ptr(cref), _ptr(cbits), threads or default_threads())
    if rc != 0:
        raise MemoryError("oracle_gemm_fp8_blockscaled failed")
    return cref, cbits


def gemm_w4a8(QA_bits, SA, QW_packed, w_scale, w_zero=None, threads: int | None = None, lib=None):
    """e2m1 weights x e4m3 activations, C = deq(A) . deq(W)^T.

    QA [M,K] e4m3 bit patterns with SA fp32 [M, ceil(K/128)]; QW_packed uint8 [N, K/2] (value k
    of a row in byte k//2, the even k in the low four bits); w_scale fp32 [N]; w_zero fp32 [N] or
    None.  Returns (cref fp64 [M,N], c bf16 bits [M,N]).
    """
    QA = _c(QA_bits, np.uint8)
    QW = _c(QW_packed, np.uint8)
    M, K = QA.shape
    N, K2 = QW.shape
    assert K % 2 == 0 and K2 == K // 2, (QA.shape, QW.shape)
    kb = (K + 127) // 128
    SA = _c(SA, np.float32)
    assert SA.shape == (M, kb), SA.shape
    WS = _c(w_scale, np.float32).reshape(N)
    WZ = None if w_zero is None else _c(w_zero, np.float32).reshape(N)
    cref = np.empty((M, N), dtype=np.float64)
    cbits = np.empty((M, N), dtype=np.uint16)
    rc = (lib or _lib()).oracle_gemm_w4a8(M, N, K, _ptr(QA), _ptr(SA), _ptr(QW), _ptr(WS),
                                          None if WZ is None else _ptr(WZ), _ptr(cref), _ptr(cbits),
                                          threads or default_threads())
    if rc != 0:
        raise MemoryError("oracle_gemm_w4a8 failed")
    return cref, cbits


def gemm_w4a8_rows(QA_bits, SA, QW_packed, w_scale, w_zero, rows, threads: int | None = None):
    rows = np.asarray(rows, dtype=np.int64)
    return gemm_w4a8(_c(QA_bits, np.uint8)[rows], _c(SA, np.float32)[rows], QW_packed, w_scale,
                     w_zero, threads)


def grouped_gemm_bf16(A_bits, B_bits, offsets, threads: int | None = None, lib=None):
    """Grouped C[r] = A[r] . B_e^T for rows r of expert e's segment.

    A [R,K] bf16 bits (rows grouped by expert), B [E,N,K] bf16 bits, offsets int32 [E+1].
    Returns (cref fp64 [R,N], c bf16 bits [R,N]).  Raises ValueError on malformed offsets.
    """
    A = _c(A_bits, np.uint16)
    B = _c(B_bits, np.uint16)
    off = _c(offsets, np.int32)
    R, K = A.shape
    E, N, K2 = B.shape
    assert K == K2 and off.shape == (E + 1,)
    cref = np.empty((R, N), dtype=np.float64)
    cbits = np.empty((R, N), dtype=np.uint16)
    rc = (lib or _lib()).oracle_grouped_gemm_bf16(R, N, K, E, _ptr(A), _ptr(B), _ptr(off), _ptr(cref),
                                         _ptr(cbits), threads or default_threads())
    if rc == -2:
        raise ValueError("malformed expert offsets")
    if rc != 0:
        raise MemoryError("oracle_grouped_gemm_bf16 failed")
    return cref, cbits


def gemm_bf16_rows(A_bits, B_bits, rows, threads: int | None = None):
    """The oracle on a subset of output rows of a large problem (for sampled parity checks)."""
    rows = np.asarray(rows, dtype=np.int64)
    A = _c(A_bits, np.uint16)[rows]
    return gemm_bf16(A, B_bits, threads)


def gemm_fp8_rows(QA_bits, QB_bits, SA, SB, rows, threads: int | None = None):
    rows = np.asarray(rows, dtype=np.int64)
    return gemm_fp8_blockscaled(_c(QA_bits, np.uint8)[rows], QB_bits,
                                _c(SA, np.float32)[rows], SB, threads)


# ---------------------------------------------------------------------------------------------
# Exact-integer GEMMs (the integer variants of the workloads, at full size)
# ---------------------------------------------------------------------------------------------

def _exact_integer_operand(bits: np.ndarray, name: str, limit: float) -> np.ndarray:
    """The fp64 values of bf16 bits that must all be integers of magnitude <= limit."""
    x = bf16_to_f64(bits)
    if not np.all(np.isfinite(x)) or not np.all(x == np.round(x)) or np.max(np.abs(x), initial=0) > limit:
        raise ValueError(f"{name} holds values that are not integers of magnitude <= {limit}")
    return x


def gemm_bf16_exact_integers(A_bits: np.ndarray, B_bits: np.ndarray):
    """C = A . B^T for bf16 A [M,K], B [N,K] whose entries are all small integers.

    This is the definition of ``gemm_bf16`` for inputs on which it is exact by construction: with
    |a|, |b| <= 2^8 and K <= 2^30, every product and every partial sum is an integer below 2^53,
    so the fp64 sum is the exact integer result in any order, and a library fp64 matmul computes
    it.  The result is rounded once to bf16 (RNE) as ``gemm_bf16`` does.  Inputs outside that
    range raise ValueError instead of returning a rounded result.  Returns (cref, c bf16 bits).
    """
    A = _exact_integer_operand(_c(A_bits, np.uint16), "A", 256.0)
    B = _exact_integer_operand(_c(B_bits, np.uint16), "B", 256.0)
    assert A.shape[1] == B.shape[1], "A and B disagree on K"
    if A.shape[1] > (1 << 30):
        raise ValueError("K too large for an exact fp64 sum")
    cref = A @ B.T
    return cref, f64_to_bf16(cref)


def grouped_gemm_bf16_exact_integers(A_bits, B_bits, offsets):
    """The grouped GEMM (``grouped_gemm_bf16``) on small-integer inputs, exact as in
    ``gemm_bf16_exact_integers``: C[r] = A[r] . B_e^T for the rows r of expert e's segment."""
    A = _c(A_bits, np.uint16)
    B = _c(B_bits, np.uint16)
    off = _c(offsets, np.int64)
    R, K = A.shape
    E, N, K2 = B.shape
    assert K == K2 and off.shape == (E + 1,)
    if off[0] != 0 or off[E] != R or np.any(np.diff(off) < 0):
        raise ValueError("malformed expert offsets")
    cref = np.zeros((R, N), dtype=np.float64)
    for e in range(E):
        if off[e + 1] > off[e]:
            cref[off[e]:off[e + 1]], _ = gemm_bf16_exact_integers(A[off[e]:off[e + 1]], B[e])
    return cref, f64_to_bf16(cref)
