"""CPU oracle for the batch-invariant GEMM -- test infrastructure only (see ``oracle.py``; the MoE
steps around the grouped GEMM are in ``moe.py``, the decode attention in ``attention.py``)."""
from .oracle import (  # noqa: F401
    bf16_to_f64,
    OracleLib,
    build,
    compile_copy,
    default_threads,
    e2m1_to_f64,
    e4m3_to_f64,
    f64_to_bf16,
    f64_to_e2m1,
    fp16_to_f64,
    gemm_bf16,
    gemm_bf16_exact_integers,
    gemm_bf16_rows,
    gemm_fp8_blockscaled,
    gemm_fp8_rows,
    gemm_w4a8,
    gemm_w4a8_rows,
    grouped_gemm_bf16,
    grouped_gemm_bf16_exact_integers,
    quantize_e2m1,
)
from . import attention, moe  # noqa: F401,E402
