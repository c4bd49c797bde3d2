"""Batch-invariant GEMM for NVIDIA B200 (sm_100a).

C[M,N] = A[M,K] . B[N,K]^T with fp32 accumulation and bf16 output, computed by hand-written
tcgen05/TMA kernels behind the C ABI in ``include/bi_gemm.h``: bf16, FP8 e4m3 with block scales,
and e2m1 weights (per-channel power-of-two scale and zero point) x e4m3 activations.  The MoE
routing, dispatch, gather and combine steps around the grouped GEMM are in ``include/bi_moe.h``,
the dual-kernel decode attention in ``include/bi_attention.h``, and the e2m1 weight quantisation
in ``include/bi_quantize.h``.  Every output row is bit-identical whatever the batch size, the
row's position and the other rows in the batch.

``binding`` holds the ctypes wrapper (same names as the C ABI); ``inputs`` the seeded synthetic
input generators; ``build`` the nvcc build of ``libbigemm.so``.
"""
from .binding import (  # noqa: F401
    BI_DEBUG_SKIP_FIRST_LOAD,
    BI_DTYPE_BF16,
    BI_DTYPE_E2M1_W4A8,
    BI_DTYPE_E4M3_BLOCKSCALED,
    BI_PLAN_RESIDENT_WEIGHTS,
    BI_PLAN_HOST_ROW_BLOCKS,
    BiGemmError,
    Plan,
    bi_decode_attention,
    bi_decode_attention_workspace_bytes,
    bi_gemm_abi_version,
    bi_gemm_debug_set_flags,
    bi_gemm_plan,
    bi_gemm_plan_describe,
    bi_gemm_plan_destroy,
    bi_gemm_plan_set_flags,
    bi_gemm_plan_splitk,
    bi_gemm_run,
    bi_gemm_run_host,
    bi_gemm_run_host_noalloc,
    bi_gemm_run_host_batch,
    bi_gemm_plan_column_shard,
    bi_gemm_host_batch_flush,
    bi_gemm_host_batch_staging_bytes,
    host_gemm_array,
    bi_gemm_run_splitk,
    bi_gemm_run_w4a8,
    bi_gemm_set_wait_timeout,
    bi_gemm_splitk_workspace_bytes,
    bi_gemm_sync_status,
    bi_gemm_w4a8_workspace_bytes,
    bi_grouped_gemm_run,
    bi_moe_combine,
    bi_moe_dispatch,
    bi_moe_gather_rows,
    bi_moe_route_topk,
    bi_quantize_e2m1,
    bi_status_string,
    load_library,
)
