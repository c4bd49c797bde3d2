"""Host-side helpers for running the batch-invariant GEMM on several GPUs, one process each.

The GEMM shards with no numerical exchange: split the rows of A (M-sharding: independent token
batches) or the rows of B (N-sharding: column-parallel weights, whole K per output column).  Each
rank runs the same plan -- a pure function of (N, K, dtype) -- so every row gets the same bits on
every GPU as it would alone.  Splitting K is not offered: summing partial products across ranks is
split-K, which the method excludes.  The only collectives are gathers of finished rows (a copy,
exact) and the max of per-rank timings.
"""
from __future__ import annotations


def shard_range(total: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced [begin, end) share of `total` items for `rank` of `world`."""
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(total, world)
    begin = rank * base + min(rank, extra)
    end = begin + base + (1 if rank < extra else 0)
    return begin, end


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar (a timing) over the default process group; identity if none."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_rows(local, total: int, device=None):
    """All-gather the row shards of `local` (rank r holds rows shard_range(total, world, r)) into
    one [total, ...] tensor on every rank.  Shards are padded to equal size for the collective."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size()
    longest = shard_range(total, world, 0)[1]
    # move raw bytes (every backend gathers uint8; bf16/int16 are not universal)
    row_shape = tuple(local.shape[1:])
    raw = local.contiguous().view(torch.uint8).reshape(local.shape[0], -1)
    pad = torch.zeros((longest, raw.shape[1]), dtype=torch.uint8, device=local.device)
    pad[: raw.shape[0]] = raw
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    out = []
    for r in range(world):
        b, e = shard_range(total, world, r)
        out.append(parts[r][: e - b])
    return torch.cat(out).view(local.dtype).reshape((total,) + row_shape)
