"""Column-parallel sharding on one GPU: each column shard computed with a column-shard plan of the
full plan, then placed side by side, must equal the full GEMM bit for bit (the shards run one
after another here; on several GPUs each rank runs its own, and tests/test_dist_gloo.py checks the
gather).  Covers the decode plan (four chains), a CTA-pair prefill plan and an FP8 plan."""
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
from invariant_deterministic_gemm_bi_b200 import inputs
from invariant_deterministic_gemm_bi_b200.sharding import column_shard_plan
from tests.gpu_util import kblock_major_scales

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(plan, A, B, scale_a=None, scale_b=None):
    C = torch.empty((A.shape[0], B.shape[0]), dtype=torch.bfloat16, device=DEV)
    bg.bi_gemm_run(plan, A, B, C, scale_a=scale_a, scale_b=scale_b)
    bg.bi_gemm_sync_status(plan)
    return C


@pytest.mark.parametrize("N,K,M,world", [(4096, 7168, 7, 2), (4096, 7168, 130, 3), (7168, 2048, 300, 4)])
def test_bf16_column_shards_concatenate_to_the_full_gemm(N, K, M, world):
    full = bg.bi_gemm_plan(N, K)
    A = inputs.bf16_gaussian((M, K), seed=5700 + M, device=DEV)
    B = inputs.bf16_gaussian((N, K), seed=5701, std=K ** -0.5, device=DEV)
    want = run(full, A, B)
    parts = []
    for r in range(world):
        b, e, plan = column_shard_plan(full, world, r)
        parts.append(run(plan, A, B[b:e].contiguous()))
    got = torch.cat(parts, dim=1)
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_fp8_column_shards_concatenate_to_the_full_gemm():
    N = K = 7168
    M, world = 40, 3
    KB = K // 128
    full = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    qa = inputs.e4m3_gaussian((M, K), seed=5801, device=DEV)
    qb = inputs.e4m3_gaussian((N, K), seed=5802, device=DEV)
    sa = kblock_major_scales(inputs.scales_log_uniform((M, KB), seed=5803, device=DEV))
    sb = inputs.scales_log_uniform((N // 128, KB), seed=5804, device=DEV)
    want = run(full, qa, qb, sa, sb)
    parts = []
    for r in range(world):
        b, e, plan = column_shard_plan(full, world, r)
        assert b % 128 == 0
        parts.append(run(plan, qa, qb[b:e].contiguous(), sa, sb[b // 128:(e + 127) // 128].contiguous()))
    got = torch.cat(parts, dim=1)
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
