"""Seeded synthetic inputs for the batch-invariant GEMM workloads.

This module only draws random numbers and rounds them to the storage formats (bf16, e4m3,
fp32 scales); it holds none of the GEMM's arithmetic.  Both the CUDA path (tests, benchmark)
and the CPU oracle receive the arrays it returns, so the two sides always see the same bits.

Recipes (all seeded; a generator is ``torch.Generator(device)`` seeded with the given seed):

* bf16 Gaussian:   x ~ N(0, std^2) drawn in fp32, rounded to bf16 (RNE).
* bf16 integer:    x uniform in {-4, ..., 4}, exact in bf16.
* e4m3 Gaussian:   x ~ N(0, 1) in fp32, clamped to [-448, 448], rounded to e4m3 (RNE).
* e4m3 integer:    x uniform in {-4, ..., 4}, exact in e4m3.
* fp32 scales:     s = 2^u, u ~ U(-4, 4) (log-uniform in [2^-4, 2^4]); or s = 2^j with integer
                   j uniform in [-4, 4] for the exactly representable variant.
* e2m1 weights:    every 4-bit code uniform in 0..15 (the values +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}
                   equally often), packed two per byte, the even K index in the low four bits.
* e2m1 channel scales: 2^-j with integer j uniform in [1, 12]; zero points z = fp16(x * s),
                   x ~ N(0, 1), rounded to fp16 (RNE) and held in fp32; or, for the exactly
                   representable variant, z = i * 2^-6 with integer i uniform in [-64, 64].
* MoE router logits: [T, E] ~ N(0, 1) in fp32 (``torch.randn`` on a seeded generator).  Routing
                   them (top-8, grouping by expert) is arithmetic of the MoE steps: the library's
                   kernels do it on the GPU (include/bi_moe.h), the oracle on the CPU.

Bits are returned as torch tensors (``torch.int16`` views for bf16, ``torch.uint8`` for e4m3)
on the requested device; ``to_numpy_bits`` gives the host copies the oracle takes.
"""
from __future__ import annotations

import numpy as np
import torch


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def bf16_gaussian(shape, seed: int, std: float = 1.0, device="cpu") -> torch.Tensor:
    """bf16 tensor with entries N(0, std^2), drawn in fp32 and rounded to nearest even."""
    g = generator(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def bf16_integers(shape, seed: int, lo: int = -4, hi: int = 4, device="cpu") -> torch.Tensor:
    """bf16 tensor with integer entries uniform in [lo, hi] (exact in bf16)."""
    g = generator(seed, device)
    x = torch.randint(lo, hi + 1, tuple(shape), generator=g, device=device, dtype=torch.int32)
    return x.to(torch.bfloat16)


def e4m3_gaussian(shape, seed: int, device="cpu") -> torch.Tensor:
    """e4m3 (fn) tensor: N(0,1) in fp32, clamped to +-448, rounded to nearest even."""
    g = generator(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    x.clamp_(-448.0, 448.0)
    return x.to(torch.float8_e4m3fn)


def e4m3_integers(shape, seed: int, lo: int = -4, hi: int = 4, device="cpu") -> torch.Tensor:
    g = generator(seed, device)
    x = torch.randint(lo, hi + 1, tuple(shape), generator=g, device=device, dtype=torch.int32)
    return x.to(torch.float32).to(torch.float8_e4m3fn)


def scales_log_uniform(shape, seed: int, lo_exp: float = -4.0, hi_exp: float = 4.0,
                       device="cpu") -> torch.Tensor:
    """fp32 scales 2^u with u ~ U(lo_exp, hi_exp)."""
    g = generator(seed, device)
    u = torch.rand(*shape, generator=g, device=device, dtype=torch.float32)
    u.mul_(hi_exp - lo_exp).add_(lo_exp)
    return torch.exp2(u)


def scales_pow2(shape, seed: int, lo: int = -4, hi: int = 4, device="cpu") -> torch.Tensor:
    """fp32 scales 2^j with integer j uniform in [lo, hi] (exact products)."""
    g = generator(seed, device)
    j = torch.randint(lo, hi + 1, tuple(shape), generator=g, device=device, dtype=torch.int32)
    return torch.exp2(j.to(torch.float32))


def e2m1_packed_uniform(rows: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    """uint8 [rows, K/2]: uniformly drawn e2m1 codes, value k in the low four bits of byte k//2
    when k is even and in the high four bits when k is odd."""
    assert K % 2 == 0
    g = generator(seed, device)
    codes = torch.randint(0, 16, (rows, K), generator=g, device=device, dtype=torch.int32)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).to(torch.uint8)


def channel_scales_pow2(n: int, seed: int, lo: int = 1, hi: int = 12, device="cpu") -> torch.Tensor:
    """fp32 [n]: 2^-j with integer j uniform in [lo, hi]."""
    g = generator(seed, device)
    j = torch.randint(lo, hi + 1, (n,), generator=g, device=device, dtype=torch.int32)
    return torch.exp2(-j.to(torch.float32))


def channel_zeros_fp16(scales: torch.Tensor, seed: int) -> torch.Tensor:
    """fp32 zero points z[n] = fp16(x[n] * scales[n]), x ~ N(0, 1) (values fp16 holds exactly)."""
    g = generator(seed, scales.device)
    x = torch.randn(scales.shape, generator=g, device=scales.device, dtype=torch.float32)
    return (x * scales).to(torch.float16).to(torch.float32)


def channel_zeros_grid(n: int, seed: int, device="cpu") -> torch.Tensor:
    """fp32 zero points i * 2^-6 with integer i uniform in [-64, 64]."""
    g = generator(seed, device)
    i = torch.randint(-64, 65, (n,), generator=g, device=device, dtype=torch.int32)
    return i.to(torch.float32) * 2.0 ** -6


def bits_of(t: torch.Tensor) -> torch.Tensor:
    """Reinterpret a bf16 / e4m3 tensor as its raw integer bit pattern (no copy)."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8)
    raise TypeError(f"no bit view for {t.dtype}")


def to_numpy_bits(t: torch.Tensor) -> np.ndarray:
    """Host numpy copy of the raw bits: uint16 for bf16, uint8 for e4m3, float32 as is."""
    if t.dtype == torch.bfloat16:
        return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.detach().view(torch.uint8).cpu().numpy()
    if t.dtype == torch.float32:
        return t.detach().cpu().numpy()
    if t.dtype == torch.int32:
        return t.detach().cpu().numpy()
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---------------------------------------------------------------------------------------------
# seeds (one base seed per workload; derived seeds for batches, permutations and trials)
# ---------------------------------------------------------------------------------------------

WORKLOAD_BASE_SEED = {
    "small": 1000,
    "decode": 2000,
    "prefill": 3000,
    "fp8": 4000,
    "moe": 5000,
    "w4a8": 6000,
}


def derived_seed(base: int, M: int, trial: int = 0, salt: int = 0) -> int:
    return int(base + 17 * M + trial + 1_000_003 * salt)
