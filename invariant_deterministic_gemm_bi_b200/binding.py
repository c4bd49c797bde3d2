"""Thin ctypes binding of libbigemm (include/bi_gemm.h, bi_moe.h, bi_attention.h, bi_quantize.h),
same names as the C ABI.

Argument marshalling only: every function takes torch tensors (device memory owned by torch)
or raw integers, passes their pointers, strides and the current CUDA stream to the C entry
point of the same name, and raises ``BiGemmError`` on a non-OK status.  All arithmetic happens
in the CUDA kernels behind the ABI; there is no fallback of any kind.  If the shared library is
missing, loading fails loudly with instructions to build it.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libbigemm.so")

BI_DTYPE_BF16 = 0
BI_DTYPE_E4M3_BLOCKSCALED = 1
BI_DTYPE_E2M1_W4A8 = 2
BI_DEBUG_SKIP_FIRST_LOAD = 1
BI_PLAN_RESIDENT_WEIGHTS = 1
BI_PLAN_HOST_ROW_BLOCKS = 2

STATUS_NAMES = {
    0: "BI_OK", 1: "BI_ERR_INVALID_ARG", 2: "BI_ERR_ALIGNMENT", 3: "BI_ERR_UNSUPPORTED_SHAPE",
    4: "BI_ERR_DTYPE_MISMATCH", 5: "BI_ERR_CUDA", 6: "BI_ERR_DEVICE_TIMEOUT",
    7: "BI_ERR_BAD_OFFSETS", 8: "BI_ERR_NO_DEVICE",
}
STATUS = {v: k for k, v in STATUS_NAMES.items()}

# every symbol include/bi_gemm.h declares
EXPORTED = [
    "bi_gemm_abi_version", "bi_status_string", "bi_gemm_plan", "bi_gemm_plan_destroy",
    "bi_gemm_plan_describe", "bi_gemm_run", "bi_grouped_gemm_run", "bi_gemm_run_host",
    "bi_gemm_sync_status", "bi_gemm_set_wait_timeout", "bi_gemm_debug_set_flags",
    "bi_gemm_run_host_noalloc", "bi_gemm_plan_set_flags",
    "bi_gemm_host_batch_staging_bytes", "bi_gemm_run_host_batch", "bi_gemm_host_batch_flush",
    "bi_gemm_plan_column_shard",
    "bi_gemm_plan_splitk", "bi_gemm_splitk_workspace_bytes", "bi_gemm_run_splitk",
    "bi_gemm_w4a8_workspace_bytes", "bi_gemm_run_w4a8",
    "bi_moe_route_topk", "bi_moe_dispatch", "bi_moe_gather_rows", "bi_moe_combine",
    "bi_decode_attention", "bi_decode_attention_workspace_bytes",
    "bi_quantize_e2m1",
]


class BiGemmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS_NAMES.get(status, f"status {status}")
        super().__init__(f"{where}: {self.name}")


class PlanInfo(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("dtype", ctypes.c_int),
        ("num_experts", ctypes.c_int), ("block_m", ctypes.c_int), ("block_n", ctypes.c_int),
        ("block_k", ctypes.c_int), ("cta_group", ctypes.c_int), ("mma_m", ctypes.c_int),
        ("mma_n", ctypes.c_int), ("mma_k", ctypes.c_int), ("stages", ctypes.c_int),
        ("k_order_id", ctypes.c_int), ("threads_per_cta", ctypes.c_int),
        ("smem_bytes", ctypes.c_int), ("tmem_columns", ctypes.c_int),
        ("stages_a", ctypes.c_int), ("k_splits", ctypes.c_int),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


class HostGemm(ctypes.Structure):
    """bi_host_gemm_t: one GEMM of a bi_gemm_run_host_batch call."""
    _fields_ = [
        ("M", ctypes.c_int64), ("A_host", ctypes.c_void_p), ("lda", ctypes.c_int64),
        ("B", ctypes.c_void_p), ("ldb", ctypes.c_int64), ("C_host", ctypes.c_void_p),
        ("ldc", ctypes.c_int64), ("scale_a_host", ctypes.c_void_p), ("ld_sa", ctypes.c_int64),
        ("scale_b", ctypes.c_void_p),
    ]


_LIB = None


def load_library(path: str = LIB_PATH):
    """Load libbigemm.so and declare its signatures.  Raises ImportError if it is missing."""
    global _LIB
    if _LIB is not None and path == LIB_PATH:
        return _LIB
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built: run `python -m invariant_deterministic_gemm_bi_b200.build`"
                          " (the CUDA library is required; there is no fallback)")
    lib = ctypes.CDLL(path)
    i64, i32, u32, u64, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_void_p
    lib.bi_gemm_abi_version.restype = i32
    lib.bi_gemm_abi_version.argtypes = []
    lib.bi_status_string.restype = ctypes.c_char_p
    lib.bi_status_string.argtypes = [i32]
    lib.bi_gemm_plan.restype = i32
    lib.bi_gemm_plan.argtypes = [ctypes.POINTER(vp), i64, i64, i32, i32]
    lib.bi_gemm_plan_destroy.restype = i32
    lib.bi_gemm_plan_destroy.argtypes = [vp]
    lib.bi_gemm_plan_describe.restype = i32
    lib.bi_gemm_plan_describe.argtypes = [vp, ctypes.POINTER(PlanInfo)]
    lib.bi_gemm_run.restype = i32
    lib.bi_gemm_run.argtypes = [vp, i64, vp, i64, vp, i64, vp, i64, vp, i64, vp, vp]
    lib.bi_grouped_gemm_run.restype = i32
    lib.bi_grouped_gemm_run.argtypes = [vp, i64, vp, i64, vp, i64, vp, i64, vp, vp]
    lib.bi_gemm_run_host.restype = i32
    lib.bi_gemm_run_host.argtypes = [vp, i64, vp, i64, vp, i64, vp, i64, vp, i64, vp, vp, vp, vp, vp]
    lib.bi_gemm_host_batch_staging_bytes.restype = ctypes.c_size_t
    lib.bi_gemm_host_batch_staging_bytes.argtypes = [vp, i32, ctypes.POINTER(HostGemm), i32]
    lib.bi_gemm_run_host_batch.restype = i32
    lib.bi_gemm_run_host_batch.argtypes = [vp, i32, ctypes.POINTER(HostGemm), vp, ctypes.c_size_t, vp,
                                           vp, vp]
    lib.bi_gemm_plan_column_shard.restype = i32
    lib.bi_gemm_plan_column_shard.argtypes = [ctypes.POINTER(vp), vp, i64, i64]
    lib.bi_gemm_host_batch_flush.restype = i32
    lib.bi_gemm_host_batch_flush.argtypes = [vp, vp, vp, vp]
    lib.bi_gemm_run_host_noalloc.restype = i32
    lib.bi_gemm_run_host_noalloc.argtypes = [vp, i64, vp, i64, vp, i64, vp, i64, vp, i64, vp, vp]
    lib.bi_gemm_sync_status.restype = i32
    lib.bi_gemm_sync_status.argtypes = [vp, vp]
    lib.bi_gemm_set_wait_timeout.restype = i32
    lib.bi_gemm_set_wait_timeout.argtypes = [vp, u64]
    lib.bi_gemm_debug_set_flags.restype = i32
    lib.bi_gemm_debug_set_flags.argtypes = [vp, u32]
    lib.bi_gemm_plan_set_flags.restype = i32
    lib.bi_gemm_plan_set_flags.argtypes = [vp, u32]
    lib.bi_gemm_plan_splitk.restype = i32
    lib.bi_gemm_plan_splitk.argtypes = [ctypes.POINTER(vp), i64, i64, i32]
    lib.bi_gemm_splitk_workspace_bytes.restype = ctypes.c_size_t
    lib.bi_gemm_splitk_workspace_bytes.argtypes = [vp, i64]
    lib.bi_gemm_run_splitk.restype = i32
    lib.bi_gemm_run_splitk.argtypes = [vp, i64, vp, i64, vp, i64, vp, i64, vp, ctypes.c_size_t, vp]
    lib.bi_gemm_w4a8_workspace_bytes.restype = ctypes.c_size_t
    lib.bi_gemm_w4a8_workspace_bytes.argtypes = [i64]
    lib.bi_gemm_run_w4a8.restype = i32
    lib.bi_gemm_run_w4a8.argtypes = [vp, i64, vp, i64, vp, i64, vp, i64, vp, vp, vp, ctypes.c_size_t,
                                     vp, i64, vp]
    lib.bi_moe_route_topk.restype = i32
    lib.bi_moe_route_topk.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp]
    lib.bi_moe_dispatch.restype = i32
    lib.bi_moe_dispatch.argtypes = [vp, i64, i32, i32, vp, vp, vp, vp]
    lib.bi_moe_gather_rows.restype = i32
    lib.bi_moe_gather_rows.argtypes = [vp, i64, i64, vp, i64, vp, i64, vp]
    lib.bi_moe_combine.restype = i32
    lib.bi_moe_combine.argtypes = [vp, i64, i64, vp, vp, i64, i32, vp, i64, vp]
    lib.bi_decode_attention_workspace_bytes.restype = ctypes.c_size_t
    lib.bi_decode_attention_workspace_bytes.argtypes = [i64, i32, i32, i32]
    lib.bi_decode_attention.restype = i32
    lib.bi_decode_attention.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i64, ctypes.c_float, i32,
                                        vp, ctypes.c_size_t, vp, vp]
    lib.bi_quantize_e2m1.restype = i32
    lib.bi_quantize_e2m1.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, i64, vp]
    if path == LIB_PATH:
        _LIB = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise BiGemmError(status, where)


def _stream_handle(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


@dataclass
class Plan:
    """A plan handle; destroy() (or garbage collection) releases it."""
    handle: int
    n: int
    k: int
    dtype: int
    num_experts: int

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass

    def destroy(self):
        if self.handle:
            bi_gemm_plan_destroy(self)
            self.handle = 0


def bi_gemm_abi_version() -> int:
    return load_library().bi_gemm_abi_version()


def bi_status_string(status: int) -> str:
    return load_library().bi_status_string(status).decode()


def bi_gemm_plan(N: int, K: int, dtype: int = BI_DTYPE_BF16, num_experts: int = 1) -> Plan:
    h = ctypes.c_void_p()
    _check(load_library().bi_gemm_plan(ctypes.byref(h), N, K, dtype, num_experts), "bi_gemm_plan")
    return Plan(h.value, N, K, dtype, num_experts)


def bi_gemm_plan_destroy(plan: Plan):
    if plan.handle:
        _check(load_library().bi_gemm_plan_destroy(plan.handle), "bi_gemm_plan_destroy")
        plan.handle = 0


def bi_gemm_plan_describe(plan: Plan) -> dict:
    info = PlanInfo()
    _check(load_library().bi_gemm_plan_describe(plan.handle, ctypes.byref(info)),
           "bi_gemm_plan_describe")
    return info.as_dict()


def bi_gemm_run(plan: Plan, A, B, C, scale_a=None, scale_b=None, stream=None, M: int | None = None):
    """C[:M] = A[:M] . B^T.  A [M, lda], B [N, ldb], C [M, ldc] (row-major, unit inner stride).

    FP8: scale_a is fp32 [ceil(K/128), ld_sa] (K-block-major, ld_sa >= M), scale_b fp32
    [ceil(N/128), ceil(K/128)].
    """
    M = A.shape[0] if M is None else M
    ld_sa = scale_a.stride(0) if scale_a is not None else 0
    st = load_library().bi_gemm_run(plan.handle, M, _ptr(A), A.stride(0), _ptr(B), B.stride(0),
                                    _ptr(C), C.stride(0), _ptr(scale_a), ld_sa, _ptr(scale_b),
                                    _stream_handle(stream))
    _check(st, "bi_gemm_run")
    return C


def bi_grouped_gemm_run(plan: Plan, A, B, C, expert_offsets, stream=None):
    """Grouped: rows of A grouped by expert (device int32 offsets [E+1]); B [E, N, ldb]."""
    ldb = B.stride(-2)
    st = load_library().bi_grouped_gemm_run(plan.handle, A.shape[0], _ptr(A), A.stride(0),
                                            _ptr(B), ldb, _ptr(C), C.stride(0),
                                            _ptr(expert_offsets), _stream_handle(stream))
    _check(st, "bi_grouped_gemm_run")
    return C


def bi_gemm_run_host(plan: Plan, A_host, B, C_host, A_dev, C_dev, scale_a_host=None, scale_b=None,
                     scale_a_dev=None, stream=None):
    """Host-memory variant: copies A (and scale_a) in, runs, copies C out, all on `stream`."""
    M = A_host.shape[0]
    ld_sa = scale_a_host.stride(0) if scale_a_host is not None else 0
    st = load_library().bi_gemm_run_host(plan.handle, M, _ptr(A_host), A_host.stride(0), _ptr(B),
                                         B.stride(0), _ptr(C_host), C_host.stride(0),
                                         _ptr(scale_a_host), ld_sa, _ptr(scale_b), _ptr(A_dev),
                                         _ptr(C_dev), _ptr(scale_a_dev), _stream_handle(stream))
    _check(st, "bi_gemm_run_host")
    return C_host


def bi_gemm_run_host_noalloc(plan: Plan, A_host, B, C_host, scale_a_host=None, scale_b=None,
                             stream=None):
    """Host-memory variant that allocates no device memory: staging copies live in the
    library's static device scratch.  Synchronous: C_host holds the result on return."""
    M = A_host.shape[0]
    ld_sa = scale_a_host.stride(0) if scale_a_host is not None else 0
    st = load_library().bi_gemm_run_host_noalloc(plan.handle, M, _ptr(A_host), A_host.stride(0),
                                                 _ptr(B), B.stride(0), _ptr(C_host),
                                                 C_host.stride(0), _ptr(scale_a_host), ld_sa,
                                                 _ptr(scale_b), _stream_handle(stream))
    _check(st, "bi_gemm_run_host_noalloc")
    return C_host


def host_gemm_array(calls) -> "ctypes.Array":
    """A bi_host_gemm_t array from (A_host, B, C_host[, scale_a_host, scale_b]) tuples of tensors
    (host A / C / scale_a, device B / scale_b; ld_sa is scale_a's row pitch)."""
    arr = (HostGemm * len(calls))()
    for i, c in enumerate(calls):
        A, B, C = c[0], c[1], c[2]
        sa = c[3] if len(c) > 3 else None
        sb = c[4] if len(c) > 4 else None
        arr[i] = HostGemm(A.shape[0], _ptr(A), A.stride(0), _ptr(B), B.stride(0), _ptr(C),
                          C.stride(0), _ptr(sa), sa.stride(0) if sa is not None else 0, _ptr(sb))
    return arr


def bi_gemm_host_batch_staging_bytes(plan: Plan, calls, regions: int = 3) -> int:
    """Bytes of staging for `regions` batches like `calls` in flight (2..32; 0 if invalid)."""
    arr = calls if isinstance(calls, ctypes.Array) else host_gemm_array(calls)
    return int(load_library().bi_gemm_host_batch_staging_bytes(plan.handle, len(arr), arr, regions))


def bi_gemm_run_host_batch(plan: Plan, calls, staging, copy_in=None, compute=None, copy_out=None):
    """Pipelined host-buffer GEMMs: the calls' A come in on copy_in, their GEMMs run on compute,
    and their C go out on copy_out with the next batch call or bi_gemm_host_batch_flush (see
    include/bi_gemm.h).  `calls` is a list of tuples as for host_gemm_array, or such an array;
    `staging` a device tensor of at least bi_gemm_host_batch_staging_bytes bytes.  Returns once
    enqueued."""
    arr = calls if isinstance(calls, ctypes.Array) else host_gemm_array(calls)
    nbytes = staging.numel() * staging.element_size()
    _check(load_library().bi_gemm_run_host_batch(plan.handle, len(arr), arr, _ptr(staging), nbytes,
                                                 _stream_handle(copy_in), _stream_handle(compute),
                                                 _stream_handle(copy_out)),
           "bi_gemm_run_host_batch")


def bi_gemm_plan_column_shard(full: Plan, n_begin: int, n_end: int) -> Plan:
    """A plan for output columns [n_begin, n_end) of `full` with `full`'s tile and K order."""
    h = ctypes.c_void_p()
    _check(load_library().bi_gemm_plan_column_shard(ctypes.byref(h), full.handle, n_begin, n_end),
           "bi_gemm_plan_column_shard")
    return Plan(h.value, n_end - n_begin, full.k, full.dtype, 1)


def bi_gemm_host_batch_flush(plan: Plan, copy_in=None, compute=None, copy_out=None):
    """Enqueue the last host batch's copy-outs (and, under capture, join the copy streams)."""
    _check(load_library().bi_gemm_host_batch_flush(plan.handle, _stream_handle(copy_in),
                                                   _stream_handle(compute), _stream_handle(copy_out)),
           "bi_gemm_host_batch_flush")


def bi_gemm_sync_status(plan: Plan, stream=None, raise_on_error: bool = True) -> int:
    st = load_library().bi_gemm_sync_status(plan.handle, _stream_handle(stream))
    if raise_on_error:
        _check(st, "bi_gemm_sync_status")
    return st


def bi_gemm_set_wait_timeout(plan: Plan, timeout_ns: int):
    _check(load_library().bi_gemm_set_wait_timeout(plan.handle, timeout_ns), "bi_gemm_set_wait_timeout")


def bi_gemm_plan_splitk(N: int, K: int, splits: int) -> Plan:
    """Fixed-split-K research plan (not the batch-invariant product path), bf16."""
    h = ctypes.c_void_p()
    _check(load_library().bi_gemm_plan_splitk(ctypes.byref(h), N, K, splits), "bi_gemm_plan_splitk")
    return Plan(h.value, N, K, BI_DTYPE_BF16, 1)


def bi_gemm_splitk_workspace_bytes(plan: Plan, M: int) -> int:
    return int(load_library().bi_gemm_splitk_workspace_bytes(plan.handle, M))


def bi_gemm_run_splitk(plan: Plan, A, B, C, workspace, stream=None, M: int | None = None):
    """C[:M] = A[:M] . B^T with a split-K plan; workspace is a device tensor of at least
    bi_gemm_splitk_workspace_bytes(plan, M) bytes."""
    M = A.shape[0] if M is None else M
    nbytes = workspace.numel() * workspace.element_size()
    st = load_library().bi_gemm_run_splitk(plan.handle, M, _ptr(A), A.stride(0), _ptr(B), B.stride(0),
                                           _ptr(C), C.stride(0), _ptr(workspace), nbytes,
                                           _stream_handle(stream))
    _check(st, "bi_gemm_run_splitk")
    return C


def bi_gemm_w4a8_workspace_bytes(M: int) -> int:
    return int(load_library().bi_gemm_w4a8_workspace_bytes(M))


def bi_gemm_run_w4a8(plan: Plan, A, scale_a, W, w_scale, C, w_zero=None, workspace=None,
                     stream=None, M: int | None = None):
    """e2m1 weights x e4m3 activations: C[:M] = deq(A[:M]) . deq(W)^T.

    A e4m3 (or uint8) [M, lda]; scale_a fp32 [K/128, ld_sa] (K-block-major); W uint8 [N, ldw/2]
    packed e2m1 (two values per byte, the even K index in the low four bits); w_scale fp32 [N]
    (each 2^-j, j in 1..12); w_zero fp32 [N] or None; workspace a device tensor of at least
    bi_gemm_w4a8_workspace_bytes(M) bytes when w_zero is given.
    """
    M = A.shape[0] if M is None else M
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load_library().bi_gemm_run_w4a8(plan.handle, M, _ptr(A), A.stride(0), _ptr(scale_a),
                                         scale_a.stride(0), _ptr(W), W.stride(0) * 2, _ptr(w_scale),
                                         _ptr(w_zero), _ptr(workspace), nbytes, _ptr(C), C.stride(0),
                                         _stream_handle(stream))
    _check(st, "bi_gemm_run_w4a8")
    return C


def bi_gemm_plan_set_flags(plan: Plan, flags: int):
    """BI_PLAN_RESIDENT_WEIGHTS: B is never written by an earlier kernel on the launch's stream.
    BI_PLAN_HOST_ROW_BLOCKS: touching host buffers of one host batch are one allocation."""
    _check(load_library().bi_gemm_plan_set_flags(plan.handle, flags), "bi_gemm_plan_set_flags")


def bi_gemm_debug_set_flags(plan: Plan, flags: int):
    _check(load_library().bi_gemm_debug_set_flags(plan.handle, flags), "bi_gemm_debug_set_flags")


# ---------------------------------------------------------------------------------------------
# MoE steps either side of the grouped GEMM (include/bi_moe.h)
# ---------------------------------------------------------------------------------------------

def bi_moe_route_topk(logits, k: int, experts, weights, stream=None):
    """logits fp32 [T, E] -> experts int32 [T, k], weights fp32 [T, k] (device tensors)."""
    T, E = logits.shape
    _check(load_library().bi_moe_route_topk(_ptr(logits), logits.stride(0), T, E, k, _ptr(experts),
                                            _ptr(weights), _stream_handle(stream)), "bi_moe_route_topk")
    return experts, weights


def bi_moe_dispatch(experts, num_experts: int, offsets, token_of_row, row_of_slot, stream=None):
    """experts int32 [T, k] -> offsets int32 [E+1], token_of_row int32 [T*k], row_of_slot int32 [T*k]."""
    T, k = experts.shape
    _check(load_library().bi_moe_dispatch(_ptr(experts), T, num_experts, k, _ptr(offsets),
                                          _ptr(token_of_row), _ptr(row_of_slot), _stream_handle(stream)),
           "bi_moe_dispatch")
    return offsets, token_of_row, row_of_slot


def bi_moe_gather_rows(X, token_of_row, A_perm, stream=None):
    """A_perm[r] = X[token_of_row[r]] (bf16 rows)."""
    R = token_of_row.numel()
    K = X.shape[1]
    _check(load_library().bi_moe_gather_rows(_ptr(X), X.stride(0), K, _ptr(token_of_row), R,
                                             _ptr(A_perm), A_perm.stride(0), _stream_handle(stream)),
           "bi_moe_gather_rows")
    return A_perm


def bi_moe_combine(C_perm, row_of_slot, weights, Y, stream=None):
    """Y[t] = sum_j weights[t, j] * C_perm[row_of_slot[t*k + j]] in slot order (bf16 out)."""
    T, k = weights.shape
    N = C_perm.shape[1]
    _check(load_library().bi_moe_combine(_ptr(C_perm), C_perm.stride(0), N, _ptr(row_of_slot),
                                         _ptr(weights), T, k, _ptr(Y), Y.stride(0),
                                         _stream_handle(stream)), "bi_moe_combine")
    return Y


# ---------------------------------------------------------------------------------------------
# Dual-kernel decode attention (include/bi_attention.h)
# ---------------------------------------------------------------------------------------------

def bi_decode_attention_workspace_bytes(B: int, Hq: int, D: int, splits: int) -> int:
    return int(load_library().bi_decode_attention_workspace_bytes(B, Hq, D, splits))


def bi_decode_attention(Q, K, V, lengths, O, scale: float, splits: int = 1, workspace=None,
                        stream=None):
    """Q [B, Hq, D], K/V [B, Lmax, Hkv, D] bf16, lengths int32 [B] (device) -> O [B, Hq, D].
    splits 1 (no split), 2 or 4 (split-KV), or 0 (automatic); every choice gives the same bits."""
    B, Hq, D = Q.shape
    _, Lmax, Hkv, _ = K.shape
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().bi_decode_attention(_ptr(Q), _ptr(K), _ptr(V), _ptr(lengths), B, Hq, Hkv, D,
                                              Lmax, scale, splits, _ptr(workspace), nbytes, _ptr(O),
                                              _stream_handle(stream)), "bi_decode_attention")
    return O


# ---------------------------------------------------------------------------------------------
# e2m1 weight quantisation (include/bi_quantize.h)
# ---------------------------------------------------------------------------------------------

def bi_quantize_e2m1(W, w_scale, Q, w_zero=None, stream=None):
    """Packed e2m1 codes Q (uint8 [N, ldq/2]) of the bf16 or fp16 weights W [N, ldw]:
    q = round_to_nearest_even((W - w_zero) / w_scale), saturating at +-6."""
    import torch
    if W.dtype not in (torch.bfloat16, torch.float16):
        raise TypeError("W must be bf16 or fp16")
    N, K = W.shape
    st = load_library().bi_quantize_e2m1(_ptr(W), 1 if W.dtype == torch.float16 else 0, W.stride(0), N, K,
                                         _ptr(w_scale), _ptr(w_zero), _ptr(Q), Q.stride(0) * 2,
                                         _stream_handle(stream))
    _check(st, "bi_quantize_e2m1")
    return Q
