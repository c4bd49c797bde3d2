"""Expert routings for the grouped-GEMM tests -- test infrastructure only.

The grouped GEMM takes rows already grouped by expert plus the expert offsets.  The tests build
those from router logits with the oracle's own MoE steps (``oracle.moe``: top-k experts by logit,
ties to the lower expert index, then a stable grouping of the (token, slot) pairs by expert), so
the routing arithmetic that feeds the GEMM tests is the pinned one
(``tests/test_oracle_moe.py``).  Adversarial routings ("for any MoE routing") are given as an
explicit expert id per grouped row.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from invariant_deterministic_gemm_bi_b200 import inputs
from oracle import moe as omoe


@dataclass
class Routing:
    """T tokens routed to experts, grouped by expert."""
    num_experts: int
    token_of_row: torch.Tensor     # int64 [R]: the token each grouped row comes from
    expert_of_row: torch.Tensor    # int64 [R]
    offsets: torch.Tensor          # int32 [E+1], offsets[0] = 0, offsets[E] = R

    @property
    def rows(self) -> int:
        return int(self.token_of_row.numel())


def route(logits, num_experts: int, k: int = 8) -> Routing:
    """Route by logits [T, E] (torch or numpy, any device): top-k, then grouped by expert."""
    if isinstance(logits, torch.Tensor):
        logits = logits.detach().float().cpu().numpy()
    experts, _ = omoe.route_topk(np.asarray(logits, dtype=np.float32), k)
    offsets, token_of_row, _ = omoe.dispatch(experts, num_experts)
    expert_of_row = np.repeat(np.arange(num_experts, dtype=np.int64), np.diff(offsets))
    return Routing(num_experts, torch.from_numpy(token_of_row.astype(np.int64)),
                   torch.from_numpy(expert_of_row), torch.from_numpy(offsets.astype(np.int32)))


def topk_experts(logits, k: int = 8) -> torch.Tensor:
    """The top-k expert ids per token [T, k] (int64), descending logit, ties to the lower index."""
    if isinstance(logits, torch.Tensor):
        logits = logits.detach().float().cpu().numpy()
    experts, _ = omoe.route_topk(np.asarray(logits, dtype=np.float32), k)
    return torch.from_numpy(experts)


def softmax_top8_routing(T: int, num_experts: int, seed: int) -> Routing:
    """Router logits ~ N(0, 1) [T, E] from the seeded generator; top-8 per token; grouped."""
    g = inputs.generator(seed, "cpu")
    logits = torch.randn(T, num_experts, generator=g, dtype=torch.float32)
    return route(logits, num_experts, 8)


def routing_from_assignment(experts_per_row, num_experts: int, token_of_row=None) -> Routing:
    """A routing given as an explicit expert id per row (rows already grouped by expert)."""
    e = np.asarray(experts_per_row, dtype=np.int64)
    assert np.all(np.diff(e) >= 0), "rows must already be grouped by expert"
    counts = np.bincount(e, minlength=num_experts)
    offsets = np.zeros(num_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    tok = np.arange(e.size) if token_of_row is None else np.asarray(token_of_row)
    return Routing(num_experts, torch.from_numpy(tok.astype(np.int64)), torch.from_numpy(e),
                   torch.from_numpy(offsets.astype(np.int32)))
