"""Host-side helpers for running the batch-invariant GEMM on several GPUs, one process each.

The GEMM shards with no numerical exchange: split the rows of A (M-sharding: independent token
batches) or the rows of B (N-sharding: column-parallel weights, whole K per output column).  With
M-sharding each rank runs the same plan -- a pure function of (N, K, dtype) -- so every row gets
the same bits on every GPU as it would alone.  With N-sharding each rank runs a column-shard plan
of the full plan (bi_gemm_plan_column_shard): a plan made for the shard's own (N/G, K) may pick
another tile and K order, and its columns would differ from the single-GPU ones in the last bits.
Splitting K is not offered: summing partial products across ranks is split-K, which the method
excludes.  The only collectives are gathers of finished rows or columns (a copy, exact) and the
max of per-rank timings.
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


def column_shard_range(n: int, world: int, rank: int, align: int = 32) -> tuple[int, int]:
    """[begin, end) of the output columns rank `rank` of `world` owns in column-parallel sharding:
    contiguous, balanced in units of `align` columns (the tile width, or 128 for FP8 weights,
    whose scale blocks a shard must not split)."""
    if align < 1:
        raise ValueError("bad alignment")
    units = (n + align - 1) // align
    b, e = shard_range(units, world, rank)
    return min(b * align, n), min(e * align, n)


def column_shard_plan(full_plan, world: int, rank: int):
    """(begin, end, plan) of this rank's column shard of a dense plan, made with
    bi_gemm_plan_column_shard so that every column keeps the full plan's tile and K order, and
    so its bits.  FP8 shards are aligned to the 128-column scale blocks."""
    from . import binding
    info = binding.bi_gemm_plan_describe(full_plan)
    align = 128 if info["dtype"] == binding.BI_DTYPE_E4M3_BLOCKSCALED else info["block_n"]
    b, e = column_shard_range(info["n"], world, rank, align)
    return b, e, binding.bi_gemm_plan_column_shard(full_plan, b, e)


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


def gather_columns(local, total_cols: int, align: int = 32, device=None):
    """All-gather the column shards of `local` [rows, cols] (rank r holds the columns
    column_shard_range(total_cols, world, r, align)) into one [rows, total_cols] tensor on every
    rank.  A copy of finished values: exact."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size()
    widths = [e - b for b, e in (column_shard_range(total_cols, world, r, align) for r in range(world))]
    widest = max(widths)
    rows = local.shape[0]
    elt = local.element_size()
    raw = local.contiguous().view(torch.uint8).reshape(rows, -1)
    pad = torch.zeros((rows, widest * elt), dtype=torch.uint8, device=local.device)
    pad[:, : raw.shape[1]] = raw
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    out = torch.cat([parts[r][:, : widths[r] * elt] for r in range(world)], dim=1)
    return out.contiguous().view(local.dtype).reshape(rows, total_cols)
