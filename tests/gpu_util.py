"""Device-side helpers for the GPU tests: guarded output buffers and strided operands."""
from __future__ import annotations

import torch

POISON = 0x7FC1       # a bf16 NaN pattern no kernel writes
GUARD_ROWS = 2


class GuardedC:
    """bf16 output C[M, N] with row stride ldc inside a buffer poisoned with a NaN pattern.

    Extra rows above and below and the columns N..ldc-1 are guard bands: check() fails if the
    kernel wrote any of them, or left any element of C[0:M, 0:N] unwritten.
    """

    def __init__(self, M: int, N: int, device="cuda", extra_cols: int = 8):
        self.M, self.N = M, N
        self.ldc = ((N + 7) // 8) * 8 + extra_cols
        self.buf = torch.full((M + 2 * GUARD_ROWS, self.ldc), POISON, dtype=torch.int16,
                              device=device)
        self.c = self.buf[GUARD_ROWS:GUARD_ROWS + M].view(torch.bfloat16)[:, :N]

    def repoison(self):
        self.buf.fill_(POISON)

    def check(self):
        b = self.buf
        g = GUARD_ROWS
        assert torch.all(b[:g] == POISON), "write above C"
        assert torch.all(b[g + self.M:] == POISON), "write below C"
        assert torch.all(b[g:g + self.M, self.N:] == POISON), "write right of C"
        assert not torch.any(b[g:g + self.M, :self.N] == POISON), "element of C left unwritten"


def strided_rows(t: torch.Tensor, ld: int) -> torch.Tensor:
    """Copy a [R, K] tensor into a [R, ld] buffer (ld >= K) and return the [R, K] view."""
    R, K = t.shape
    buf = torch.zeros((R, ld), dtype=t.dtype, device=t.device)
    buf[:, :K] = t
    return buf[:, :K]


def kblock_major_scales(sa_mk: torch.Tensor, ld_sa: int | None = None) -> torch.Tensor:
    """[M, KB] row-major fp32 scales -> the ABI's K-block-major [KB, ld_sa] layout (view [KB, M])."""
    M, KB = sa_mk.shape
    ld = ld_sa or ((M + 3) // 4) * 4
    out = torch.zeros((KB, ld), dtype=torch.float32, device=sa_mk.device)
    out[:, :M] = sa_mk.t()
    return out[:, :M]
