"""World-size-2 gloo tests of the multi-GPU host logic, on CPU.

Each rank computes its M-shard (rows) or N-shard (columns) of a GEMM with the CPU oracle standing
in for the device (what a rank's GPU computes bit for bit: per the invariance contract for rows,
and for columns with a column-shard plan of the full plan, checked on the GPU by
tests/test_gpu_sharding.py); the shards are gathered and the result must equal the one-process
result bit for bit; timings reduce by max.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from invariant_deterministic_gemm_bi_b200.sharding import (column_shard_range, gather_columns, gather_rows,
                                                          max_over_ranks, shard_range)


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from invariant_deterministic_gemm_bi_b200 import inputs
        M, N, K = 37, 80, 96
        A = inputs.to_numpy_bits(inputs.bf16_gaussian((M, K), seed=1))
        B = inputs.to_numpy_bits(inputs.bf16_gaussian((N, K), seed=2))
        b, e = shard_range(M, world, rank)
        _, local = oracle.gemm_bf16(A[b:e], B, threads=1)
        full = gather_rows(torch.from_numpy(local.view(np.int16)), M)
        _, want = oracle.gemm_bf16(A, B, threads=1)
        ok_rows = bool(np.array_equal(full.numpy().view(np.uint16), want))
        # N-sharding: this rank's columns (rows of B), gathered along N
        cb, ce = column_shard_range(N, world, rank, align=32)
        _, local_cols = oracle.gemm_bf16(A, B[cb:ce], threads=1)
        cols = gather_columns(torch.from_numpy(local_cols.view(np.int16)), N, align=32)
        ok_cols = bool(np.array_equal(cols.numpy().view(np.uint16), want))
        t = max_over_ranks(float(rank + 1) * 1.5)
        q.put((rank, ok_rows and ok_cols, t))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_m_and_n_sharded_results_gather_to_the_single_process_result(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok, t in results:
        assert ok, f"rank {rank}: gathered rows or columns differ"
        assert t == 1.5 * world, "max over ranks"


def test_shard_range_partitions_exactly():
    for total in [0, 1, 7, 256, 1000]:
        for world in [1, 2, 3, 8]:
            spans = [shard_range(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def test_column_shard_range_partitions_in_aligned_units():
    for n in [0, 31, 80, 4096, 7168]:
        for world in [1, 2, 3, 8]:
            for align in [32, 128]:
                spans = [column_shard_range(n, world, r, align) for r in range(world)]
                assert spans[0][0] == 0 and spans[-1][1] == n
                assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
                assert all(b % align == 0 or b == n for b, _ in spans)   # empty tail shards start at n
