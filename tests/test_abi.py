"""Host-side tests of the C ABI that need no GPU: the library loads, exports every symbol the
header declares, plans are pure functions of (N, K, dtype, num_experts), and argument errors come
back as status codes without any device call."""
import ctypes
import json
import os
import re
import subprocess
import sys

import pytest

import invariant_deterministic_gemm_bi_b200 as bg
from invariant_deterministic_gemm_bi_b200 import binding

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(REPO, "include", h) for h in sorted(os.listdir(os.path.join(REPO, "include")))
           if h.endswith(".h")]


def declared_functions():
    names = set()
    for header in HEADERS:
        text = open(header, encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(bi_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(binding.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert sorted(binding.EXPORTED) == names


def test_abi_version_and_status_strings():
    assert bg.bi_gemm_abi_version() == 1
    for code, name in binding.STATUS_NAMES.items():
        assert bg.bi_status_string(code).startswith(name)


def test_plan_describe_is_m_free_and_sane():
    for (N, K, dt, E) in [(4096, 7168, 0, 1), (7168, 2048, 0, 1), (2048, 7168, 0, 1),
                          (7168, 7168, 1, 1), (2048, 7168, 0, 64), (256, 512, 0, 1), (5, 3, 0, 1),
                          (7168, 7168, 2, 1), (256, 512, 2, 1)]:
        info = bg.bi_gemm_plan_describe(bg.bi_gemm_plan(N, K, dt, E))
        assert info["n"] == N and info["k"] == K and info["num_experts"] == E
        # dense bf16 plans of 32-column tiles reduce K in four interleaved chains (k_order_id 3)
        # on the 64-row MMA; every other plan in one ascending chain
        narrow_bf16 = dt == 0 and E == 1 and info["block_n"] == 32
        assert info["k_order_id"] == (3 if narrow_bf16 else 0) and info["block_m"] in (64, 128, 256)
        assert info["block_m"] == 64 or not narrow_bf16
        assert info["mma_m"] == info["block_m"] and 2 <= info["stages_a"] <= info["stages"]
        assert info["cta_group"] == (2 if info["block_m"] == 256 else 1)
        assert info["block_k"] * (1 if dt in (1, 2) else 2) in (128, 256, 512)
        assert info["mma_n"] == info["block_n"] and info["block_n"] % 32 == 0
        assert info["smem_bytes"] <= 232448
        assert info["tmem_columns"] <= 512
    # grouped plans run on one CTA (an expert's segment is often a few rows long)
    g = bg.bi_gemm_plan_describe(bg.bi_gemm_plan(2048, 7168, 0, 64))
    assert g["cta_group"] == 1 and g["block_m"] == 128


def test_plan_is_the_same_in_a_fresh_process():
    shapes = [(4096, 7168, 0, 1), (7168, 7168, 1, 1), (2048, 7168, 0, 64), (1000, 100, 0, 1)]
    here = [bg.bi_gemm_plan_describe(bg.bi_gemm_plan(*s)) for s in shapes]
    code = ("import json, invariant_deterministic_gemm_bi_b200 as bg;"
            f"print(json.dumps([bg.bi_gemm_plan_describe(bg.bi_gemm_plan(*s)) for s in {shapes!r}]))")
    out = subprocess.run([sys.executable, "-c", code], cwd=REPO, capture_output=True, text=True,
                         check=True).stdout
    assert json.loads(out.strip().splitlines()[-1]) == here


@pytest.mark.parametrize("args,status", [
    ((-1, 8, 0, 1), "BI_ERR_INVALID_ARG"),
    ((8, -1, 0, 1), "BI_ERR_INVALID_ARG"),
    ((8, 8, 0, 0), "BI_ERR_INVALID_ARG"),
    ((8, 8, 7, 1), "BI_ERR_INVALID_ARG"),
    ((8, 8, 1, 4), "BI_ERR_UNSUPPORTED_SHAPE"),
    ((8, 8, 0, 2048), "BI_ERR_UNSUPPORTED_SHAPE"),
])
def test_plan_rejects_bad_arguments(args, status):
    with pytest.raises(bg.BiGemmError) as e:
        bg.bi_gemm_plan(*args)
    assert e.value.name == status


def test_run_rejects_bad_arguments_without_touching_a_device():
    lib = binding.load_library()
    plan = bg.bi_gemm_plan(64, 64)
    h = plan.handle
    S = binding.STATUS
    # null plan
    assert lib.bi_gemm_run(None, 1, 16, 64, 16, 64, 16, 64, None, 0, None, None) == S["BI_ERR_INVALID_ARG"]
    # negative M
    assert lib.bi_gemm_run(h, -1, 16, 64, 16, 64, 16, 64, None, 0, None, None) == S["BI_ERR_INVALID_ARG"]
    # M = 0 is a no-op
    assert lib.bi_gemm_run(h, 0, None, 64, None, 64, None, 64, None, 0, None, None) == 0
    # null A / C
    assert lib.bi_gemm_run(h, 1, None, 64, 16, 64, 16, 64, None, 0, None, None) == S["BI_ERR_INVALID_ARG"]
    assert lib.bi_gemm_run(h, 1, 16, 64, 16, 64, None, 64, None, 0, None, None) == S["BI_ERR_INVALID_ARG"]
    # strides below the extent, misaligned pointers and strides
    assert lib.bi_gemm_run(h, 1, 16, 32, 16, 64, 16, 64, None, 0, None, None) == S["BI_ERR_INVALID_ARG"]
    assert lib.bi_gemm_run(h, 1, 18, 64, 16, 64, 16, 64, None, 0, None, None) == S["BI_ERR_ALIGNMENT"]
    assert lib.bi_gemm_run(h, 1, 16, 68, 16, 64, 16, 64, None, 0, None, None) == S["BI_ERR_ALIGNMENT"]
    assert lib.bi_gemm_run(h, 1, 16, 64, 16, 64, 16, 66, None, 0, None, None) == S["BI_ERR_ALIGNMENT"]
    # scales on a bf16 plan
    assert lib.bi_gemm_run(h, 1, 16, 64, 16, 64, 16, 64, 16, 1, 16, None) == S["BI_ERR_DTYPE_MISMATCH"]
    # a grouped call on a dense plan and the reverse
    assert lib.bi_grouped_gemm_run(h, 1, 16, 64, 16, 64, 16, 64, 16, None) == S["BI_ERR_INVALID_ARG"]
    gplan = bg.bi_gemm_plan(64, 64, 0, 4)
    assert lib.bi_gemm_run(gplan.handle, 1, 16, 64, 16, 64, 16, 64, None, 0, None, None) == S["BI_ERR_INVALID_ARG"]
    assert lib.bi_grouped_gemm_run(gplan.handle, 1, 16, 64, 16, 64, 16, 64, None, None) == S["BI_ERR_INVALID_ARG"]
    # FP8 without scales, or ld_sa below M
    fplan = bg.bi_gemm_plan(64, 128, 1, 1)
    assert lib.bi_gemm_run(fplan.handle, 4, 16, 128, 16, 128, 16, 64, None, 4, None, None) == S["BI_ERR_DTYPE_MISMATCH"]
    assert lib.bi_gemm_run(fplan.handle, 4, 16, 128, 16, 128, 16, 64, 16, 3, 16, None) == S["BI_ERR_INVALID_ARG"]


def test_noalloc_rejects_bad_arguments_before_any_device_call():
    """The host-buffer entry point without allocation checks every argument before it touches a
    device, so each refusal below comes back on a machine with or without a GPU and launches
    nothing.  The pointer values are never dereferenced."""
    lib = binding.load_library()
    S = binding.STATUS
    run = lib.bi_gemm_run_host_noalloc
    bf = bg.bi_gemm_plan(256, 512)
    f8 = bg.bi_gemm_plan(256, 512, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    # (plan, M, A_host, lda, B, ldb, C_host, ldc, scale_a_host, ld_sa, scale_b, stream)
    assert run(None, 1, 256, 512, 256, 512, 256, 256, None, 0, None, None) == S["BI_ERR_INVALID_ARG"]
    assert run(bf.handle, -1, 256, 512, 256, 512, 256, 256, None, 0, None, None) == S["BI_ERR_INVALID_ARG"]
    # scales on a bf16 plan; FP8 without scale_b; FP8 scale_b not 4-byte aligned
    assert run(bf.handle, 1, 256, 512, 256, 512, 256, 256, 256, 1, 256, None) == S["BI_ERR_DTYPE_MISMATCH"]
    assert run(f8.handle, 1, 256, 512, 256, 512, 256, 256, 256, 1, None, None) == S["BI_ERR_DTYPE_MISMATCH"]
    assert run(f8.handle, 4, 256, 512, 256, 512, 256, 256, 256, 4, 258, None) == S["BI_ERR_ALIGNMENT"]
    assert run(f8.handle, 4, 256, 512, 256, 512, 256, 256, 256, 3, 256, None) == S["BI_ERR_INVALID_ARG"]
    # a grouped plan
    gp = bg.bi_gemm_plan(256, 512, 0, 4)
    assert run(gp.handle, 1, 256, 512, 256, 512, 256, 256, None, 0, None, None) == S["BI_ERR_INVALID_ARG"]
    # pitches whose products would overflow int64 are refused before any offset is computed:
    # a K = 0 plan (C only) with a huge ldc, and huge lda / ld_sa
    k0 = bg.bi_gemm_plan(256, 0)
    assert run(k0.handle, 2, None, 0, None, 0, 256, 2 ** 62, None, 0, None, None) == \
        S["BI_ERR_UNSUPPORTED_SHAPE"]
    assert run(bf.handle, 2, 256, 2 ** 62, 256, 512, 256, 256, None, 0, None, None) == \
        S["BI_ERR_UNSUPPORTED_SHAPE"]
    assert run(f8.handle, 2, 256, 512, 256, 512, 256, 256, 256, 2 ** 61, 256, None) == \
        S["BI_ERR_UNSUPPORTED_SHAPE"]
    assert run(bf.handle, 2 ** 40, 256, 512, 256, 512, 256, 256, None, 0, None, None) == \
        S["BI_ERR_UNSUPPORTED_SHAPE"]
    # 373 decode rows need more than the 8 MiB scratch
    dec = bg.bi_gemm_plan(4096, 7168)
    assert run(dec.handle, 373, 256, 7168, 256, 7168, 256, 4096, None, 0, None, None) == \
        S["BI_ERR_UNSUPPORTED_SHAPE"]
    if not __import__("torch").cuda.is_available():
        # valid arguments (scale_a_host may have any alignment: it is only copied)
        assert run(f8.handle, 4, 256, 512, 256, 512, 256, 256, 258, 4, 256, None) == S["BI_ERR_NO_DEVICE"]
        assert run(dec.handle, 372, 256, 7168, 256, 7168, 256, 4096, None, 0, None, None) == \
            S["BI_ERR_NO_DEVICE"]


def test_run_host_refuses_before_enqueueing_a_copy():
    lib = binding.load_library()
    S = binding.STATUS
    f8 = bg.bi_gemm_plan(256, 512, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    bf = bg.bi_gemm_plan(256, 512)
    # (plan, M, A_host, lda, B, ldb, C_host, ldc, sa_host, ld_sa, scale_b, A_dev, C_dev, sa_dev, stream)
    assert lib.bi_gemm_run_host(f8.handle, 4, 256, 512, 256, 512, 256, 256, 256, 4, 258, 256, 256, 256,
                                None) == S["BI_ERR_ALIGNMENT"]
    assert lib.bi_gemm_run_host(f8.handle, 4, 256, 512, 256, 512, 256, 256, 256, 4, 256, 256, 256, 258,
                                None) == S["BI_ERR_ALIGNMENT"]
    assert lib.bi_gemm_run_host(bf.handle, 4, 256, 512, 256, 512, 256, 256, None, 0, 256, 256, 256, None,
                                None) == S["BI_ERR_DTYPE_MISMATCH"]


def test_host_batch_rejects_bad_arguments_before_any_device_call():
    """The pipelined host-buffer batch checks every call and the staging buffer before it touches
    a device; the pointer values are never dereferenced."""
    lib = binding.load_library()
    S = binding.STATUS
    HG = binding.HostGemm
    plan = bg.bi_gemm_plan(256, 512)
    ok = HG(4, 4096, 512, 4096, 512, 4096, 256, None, 0, None)
    arr = (HG * 2)(ok, HG(0, None, 512, None, 512, None, 256, None, 0, None))
    slot = 4 * 512 * 2 + 4 * 256 * 2                  # the largest A and C
    need = lib.bi_gemm_host_batch_staging_bytes(plan.handle, 2, arr, 6)
    assert need == 6 * slot
    assert lib.bi_gemm_host_batch_staging_bytes(plan.handle, 2, arr, 1) == 0
    assert lib.bi_gemm_host_batch_staging_bytes(plan.handle, 2, arr, 33) == 0
    many = (HG * 1025)(*([ok] * 1025))
    assert lib.bi_gemm_host_batch_staging_bytes(plan.handle, 1025, many, 3) == 0
    assert lib.bi_gemm_run_host_batch(plan.handle, 1025, many, 4096, 1 << 30, None, None, None) == \
        S["BI_ERR_INVALID_ARG"]
    # with BI_PLAN_HOST_ROW_BLOCKS, calls whose host rows follow one another share one copy and
    # one run of the region: one-row calls with a 1040-byte pitch take 2080 bytes of A together
    # (2304 rounded), 2 x 1280 apart
    apart = (HG * 2)(HG(1, 4096, 520, 4096, 512, 1 << 20, 256, None, 0, None),
                     HG(1, 8192, 520, 4096, 512, 2 << 20, 256, None, 0, None))
    adjacent = (HG * 2)(HG(1, 4096, 520, 4096, 512, 1 << 20, 256, None, 0, None),
                        HG(1, 4096 + 1040, 520, 4096, 512, (1 << 20) + 512, 256, None, 0, None))
    # without BI_PLAN_HOST_ROW_BLOCKS touching buffers are copied apart (they may be two allocations)
    assert lib.bi_gemm_host_batch_staging_bytes(plan.handle, 2, apart, 2) == 2 * (2560 + 1024)
    assert lib.bi_gemm_host_batch_staging_bytes(plan.handle, 2, adjacent, 2) == 2 * (2560 + 1024)
    assert lib.bi_gemm_plan_set_flags(plan.handle, 4) == S["BI_ERR_INVALID_ARG"]
    assert lib.bi_gemm_plan_set_flags(plan.handle, binding.BI_PLAN_HOST_ROW_BLOCKS) == 0
    assert lib.bi_gemm_host_batch_staging_bytes(plan.handle, 2, apart, 2) == 2 * (2560 + 1024)
    assert lib.bi_gemm_host_batch_staging_bytes(plan.handle, 2, adjacent, 2) == 2 * (2304 + 1024)
    assert lib.bi_gemm_plan_set_flags(plan.handle, 0) == 0
    # three calls, the first two touching in A and the last two in C: two A runs, two C runs
    mixed = (HG * 3)(HG(1, 4096, 520, 4096, 512, 1 << 20, 256, None, 0, None),
                     HG(1, 4096 + 1040, 520, 4096, 512, 3 << 20, 256, None, 0, None),
                     HG(1, 1 << 16, 520, 4096, 512, (3 << 20) + 512, 256, None, 0, None))
    assert lib.bi_gemm_plan_set_flags(plan.handle, binding.BI_PLAN_HOST_ROW_BLOCKS) == 0
    # A: run of 2080 bytes, then a run of 1040 at 2304 -> 3344 -> 3584; C: 512 at 0, then a run of
    # 1024 at 512 -> 1536
    assert lib.bi_gemm_host_batch_staging_bytes(plan.handle, 3, mixed, 3) == 3 * (3584 + 1536)
    assert lib.bi_gemm_plan_set_flags(plan.handle, 0) == 0
    assert lib.bi_gemm_host_batch_staging_bytes(plan.handle, 3, mixed, 3) == 3 * (3840 + 1536)
    # FP8: each call's scale_a block has its own 256-byte run after A and C
    f8p = bg.bi_gemm_plan(256, 512, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    f8calls = (HG * 2)(HG(2, 4096, 512, 4096, 512, 1 << 20, 256, 8192, 2, 4096),
                       HG(3, 1 << 16, 512, 4096, 512, 2 << 20, 256, 16384, 3, 4096))
    # A: 1024 (-> 1024) + 1536 -> 2560; C: 1024 + 1536 -> 2560; scales: 4 x 2 x 4 = 32 -> 256,
    # 4 x 3 x 4 = 48 -> 256
    assert lib.bi_gemm_host_batch_staging_bytes(f8p.handle, 2, f8calls, 2) == 2 * (2560 + 2560 + 512)
    run = lib.bi_gemm_run_host_batch
    assert run(None, 2, arr, 4096, need, None, None, None) == S["BI_ERR_INVALID_ARG"]
    assert run(plan.handle, 0, None, None, 0, None, None, None) == 0           # empty batch
    assert run(plan.handle, 2, arr, None, need, None, None, None) == S["BI_ERR_INVALID_ARG"]
    assert run(plan.handle, 2, arr, 4096, 2 * slot - 256, None, None, None) == S["BI_ERR_INVALID_ARG"]
    assert run(plan.handle, 2, arr, 4096 + 16, need, None, None, None) == S["BI_ERR_ALIGNMENT"]
    bad = [HG(4, 4096, 512, 4096, 512, 4096, 256, 4096, 4, 4096),     # scales on a bf16 plan
           HG(4, 4096, 500, 4096, 512, 4096, 256, None, 0, None),     # lda below K
           HG(4, 4096, 516, 4096, 512, 4096, 256, None, 0, None),     # lda not a 16-byte pitch
           HG(-1, 4096, 512, 4096, 512, 4096, 256, None, 0, None),
           HG(4, None, 512, 4096, 512, 4096, 256, None, 0, None)]
    want = ["BI_ERR_DTYPE_MISMATCH", "BI_ERR_INVALID_ARG", "BI_ERR_ALIGNMENT", "BI_ERR_INVALID_ARG",
            "BI_ERR_INVALID_ARG"]
    for b, w in zip(bad, want):
        one = (HG * 1)(b)
        assert run(plan.handle, 1, one, 4096, 1 << 20, None, None, None) == S[w], w
    gp = bg.bi_gemm_plan(256, 512, 0, 4)
    assert run(gp.handle, 2, arr, 4096, need, None, None, None) == S["BI_ERR_INVALID_ARG"]
    f8 = bg.bi_gemm_plan(256, 512, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    one = (HG * 1)(HG(4, 4096, 512, 4096, 512, 4096, 256, 4096, 4, 4098))  # scale_b misaligned
    assert run(f8.handle, 1, one, 4096, 1 << 20, None, None, None) == S["BI_ERR_ALIGNMENT"]
    if not __import__("torch").cuda.is_available():
        assert run(plan.handle, 2, arr, 4096, need, None, None, None) == S["BI_ERR_NO_DEVICE"]


def test_column_shard_plans_keep_the_full_plan():
    """A shard of the decode plan keeps its tile and four-chain K order, where a plan made for the
    shard's own shape would not (2048 x 7168 is the prefill table entry: a CTA-pair tile with one
    chain), so its columns would differ from the full GEMM's in the last bits."""
    lib = binding.load_library()
    S = binding.STATUS
    full = bg.bi_gemm_plan(4096, 7168)
    fi = bg.bi_gemm_plan_describe(full)
    shard = bg.bi_gemm_plan_column_shard(full, 2048, 4096)
    si = bg.bi_gemm_plan_describe(shard)
    for key in ("block_m", "block_n", "block_k", "cta_group", "mma_m", "mma_n", "mma_k", "k_order_id",
                "threads_per_cta", "tmem_columns"):
        assert si[key] == fi[key], key
    assert si["n"] == 2048 and si["k"] == 7168
    own = bg.bi_gemm_plan_describe(bg.bi_gemm_plan(2048, 7168))
    assert (own["block_m"], own["k_order_id"]) != (fi["block_m"], fi["k_order_id"])
    import ctypes
    h = ctypes.c_void_p()
    assert lib.bi_gemm_plan_column_shard(ctypes.byref(h), full.handle, 10, 4097) == S["BI_ERR_INVALID_ARG"]
    assert lib.bi_gemm_plan_column_shard(ctypes.byref(h), full.handle, 20, 10) == S["BI_ERR_INVALID_ARG"]
    assert lib.bi_gemm_plan_column_shard(None, full.handle, 0, 10) == S["BI_ERR_INVALID_ARG"]
    grouped = bg.bi_gemm_plan(2048, 7168, 0, 64)
    assert lib.bi_gemm_plan_column_shard(ctypes.byref(h), grouped.handle, 0, 10) == S["BI_ERR_INVALID_ARG"]
    f8 = bg.bi_gemm_plan(7168, 7168, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    assert lib.bi_gemm_plan_column_shard(ctypes.byref(h), f8.handle, 64, 7168) == S["BI_ERR_UNSUPPORTED_SHAPE"]
    assert bg.bi_gemm_plan_describe(bg.bi_gemm_plan_column_shard(f8, 3584, 7168))["block_n"] == 64


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="a GPU is present")
def test_valid_run_without_a_device_reports_no_device():
    lib = binding.load_library()
    plan = bg.bi_gemm_plan(64, 64)
    st = lib.bi_gemm_run(plan.handle, 1, 16, 64, 16, 64, 16, 64, None, 0, None, None)
    assert binding.STATUS_NAMES[st] == "BI_ERR_NO_DEVICE"


def test_plan_flags_accept_known_bits_only():
    lib = binding.load_library()
    plan = bg.bi_gemm_plan(64, 64)
    S = binding.STATUS
    assert lib.bi_gemm_plan_set_flags(None, 0) == S["BI_ERR_INVALID_ARG"]
    assert lib.bi_gemm_plan_set_flags(plan.handle, bg.BI_PLAN_RESIDENT_WEIGHTS) == 0
    assert lib.bi_gemm_plan_set_flags(plan.handle, 0) == 0
    assert lib.bi_gemm_plan_set_flags(plan.handle, 4) == S["BI_ERR_INVALID_ARG"]
    assert lib.bi_gemm_plan_set_flags(plan.handle, 0x80000000) == S["BI_ERR_INVALID_ARG"]
    # the flags change when B is read, never the plan
    before = bg.bi_gemm_plan_describe(plan)
    bg.bi_gemm_plan_set_flags(plan, bg.BI_PLAN_RESIDENT_WEIGHTS)
    assert bg.bi_gemm_plan_describe(plan) == before


def test_splitk_research_plan_arguments():
    lib = binding.load_library()
    S = binding.STATUS
    import ctypes
    h = ctypes.c_void_p()
    assert lib.bi_gemm_plan_splitk(ctypes.byref(h), 4096, 7168, 3) == S["BI_ERR_INVALID_ARG"]
    assert lib.bi_gemm_plan_splitk(ctypes.byref(h), 4096, 7168, 16) == S["BI_ERR_INVALID_ARG"]
    assert lib.bi_gemm_plan_splitk(None, 4096, 7168, 4) == S["BI_ERR_INVALID_ARG"]
    # K = 192 is 3 chunks of 128 bytes: fewer than 4 splits
    assert lib.bi_gemm_plan_splitk(ctypes.byref(h), 256, 192, 4) == S["BI_ERR_UNSUPPORTED_SHAPE"]
    plan = bg.bi_gemm_plan_splitk(4096, 7168, 4)
    info = bg.bi_gemm_plan_describe(plan)
    assert info["k_splits"] == 4 and info["k_order_id"] == 1
    assert info["block_n"] == 128            # 32 column tiles x 4 splits = 128 work units
    assert bg.bi_gemm_splitk_workspace_bytes(plan, 64) == 4 * 64 * 4096 * 4
    assert bg.bi_gemm_splitk_workspace_bytes(plan, 0) == 0
    # a split-K plan is refused by the product entry points, and a product plan by the split one
    h2 = plan.handle
    assert lib.bi_gemm_run(h2, 1, 16, 7168, 16, 7168, 16, 4096, None, 0, None, None) == S["BI_ERR_INVALID_ARG"]
    prod = bg.bi_gemm_plan(4096, 7168)
    assert bg.bi_gemm_plan_describe(prod)["k_splits"] == 1
    assert lib.bi_gemm_run_splitk(prod.handle, 1, 16, 7168, 16, 7168, 16, 4096, 16, 1 << 20, None) == S["BI_ERR_INVALID_ARG"]
    # missing or short workspace
    assert lib.bi_gemm_run_splitk(h2, 2, 16, 7168, 16, 7168, 16, 4096, None, 0, None) == S["BI_ERR_INVALID_ARG"]
    need = bg.bi_gemm_splitk_workspace_bytes(plan, 2)
    assert lib.bi_gemm_run_splitk(h2, 2, 16, 7168, 16, 7168, 16, 4096, 16, need - 4, None) == S["BI_ERR_INVALID_ARG"]


def test_w4a8_plan_and_argument_checks():
    lib = binding.load_library()
    S = binding.STATUS
    W4 = bg.BI_DTYPE_E2M1_W4A8
    # K must be a multiple of 128; no grouped e2m1 plan
    for args in [(64, 200, W4, 1), (64, 64, W4, 1), (64, 128, W4, 4)]:
        with pytest.raises(bg.BiGemmError) as e:
            bg.bi_gemm_plan(*args)
        assert e.value.name == "BI_ERR_UNSUPPORTED_SHAPE", args
    plan = bg.bi_gemm_plan(7168, 7168, W4)
    info = bg.bi_gemm_plan_describe(plan)
    fp8 = bg.bi_gemm_plan_describe(bg.bi_gemm_plan(7168, 7168, bg.BI_DTYPE_E4M3_BLOCKSCALED))
    # the e2m1 plan uses the FP8 tile and MMA shape (kind::f8f6f4, K = 32 per instruction)
    for key in ("block_m", "block_n", "block_k", "cta_group", "mma_m", "mma_n", "mma_k", "stages",
                "stages_a", "k_order_id", "tmem_columns"):
        assert info[key] == fp8[key], key
    assert info["dtype"] == W4 and info["cta_group"] == 1
    assert bg.bi_gemm_w4a8_workspace_bytes(0) == 0
    assert bg.bi_gemm_w4a8_workspace_bytes(5) == 256
    assert bg.bi_gemm_w4a8_workspace_bytes(100) == 512
    h = plan.handle
    K = N = 7168
    ws = bg.bi_gemm_w4a8_workspace_bytes(4)
    run = lib.bi_gemm_run_w4a8
    # (plan, M, A, lda, scale_a, ld_sa, W, ldw, w_scale, w_zero, workspace, bytes, C, ldc, stream)
    ok = (h, 4, 256, K, 256, 4, 256, K, 256, 256, 256, ws, 256, N, None)

    def call(**kw):
        a = list(ok)
        names = ["plan", "M", "A", "lda", "sa", "ld_sa", "W", "ldw", "ws", "wz", "work", "nbytes", "C",
                 "ldc", "stream"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return run(*a)

    assert call(plan=None) == S["BI_ERR_INVALID_ARG"]
    assert call(M=-1) == S["BI_ERR_INVALID_ARG"]
    assert call(M=0) == 0
    assert call(sa=None) == S["BI_ERR_INVALID_ARG"]
    assert call(ws=None) == S["BI_ERR_INVALID_ARG"]
    assert call(ld_sa=3) == S["BI_ERR_INVALID_ARG"]
    assert call(W=272) == S["BI_ERR_ALIGNMENT"]           # not 32-byte aligned
    assert call(ldw=K + 32) == S["BI_ERR_ALIGNMENT"]      # row pitch of 3600 bytes: not 32-byte
    assert call(ldw=K - 64) == S["BI_ERR_INVALID_ARG"]    # below K
    assert call(A=264) == S["BI_ERR_ALIGNMENT"]
    assert call(ws=258) == S["BI_ERR_ALIGNMENT"]
    assert call(work=None) == S["BI_ERR_INVALID_ARG"]     # zero points need the row-sum workspace
    assert call(nbytes=ws - 4) == S["BI_ERR_INVALID_ARG"]
    assert call(work=264) == S["BI_ERR_ALIGNMENT"]
    # the dtypes do not cross: bi_gemm_run refuses an e2m1 plan, bi_gemm_run_w4a8 other plans
    assert lib.bi_gemm_run(h, 4, 256, K, 256, K, 256, N, 256, 4, 256, None) == S["BI_ERR_DTYPE_MISMATCH"]
    f8 = bg.bi_gemm_plan(7168, 7168, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    assert call(plan=f8.handle) == S["BI_ERR_DTYPE_MISMATCH"]
    assert lib.bi_gemm_run_host(h, 4, 256, K, 256, K, 256, N, 256, 4, 256, 256, 256, 256, None) == \
        S["BI_ERR_DTYPE_MISMATCH"]
    if not __import__("torch").cuda.is_available():
        assert call() == S["BI_ERR_NO_DEVICE"]
        assert call(wz=None, work=None, nbytes=0) == S["BI_ERR_NO_DEVICE"]


def test_quantize_argument_checks():
    lib = binding.load_library()
    S = binding.STATUS
    q = lib.bi_quantize_e2m1
    # (W, is_fp16, ldw, N, K, w_scale, w_zero, Q, ldq, stream)
    ok = [256, 0, 64, 4, 64, 256, 256, 256, 64, None]

    def call(i=None, v=None):
        a = list(ok)
        if i is not None:
            a[i] = v
        return q(*a)

    assert call(3, 0) == 0 and call(4, 0) == 0            # empty: no-op
    assert call(3, -1) == S["BI_ERR_INVALID_ARG"]
    assert call(4, 63) == S["BI_ERR_INVALID_ARG"]         # odd K
    assert call(1, 2) == S["BI_ERR_INVALID_ARG"]          # neither bf16 nor fp16
    assert call(0, None) == S["BI_ERR_INVALID_ARG"]
    assert call(7, None) == S["BI_ERR_INVALID_ARG"]
    assert call(5, None) == S["BI_ERR_INVALID_ARG"]
    assert call(2, 32) == S["BI_ERR_INVALID_ARG"]         # ldw < K
    assert call(8, 62) == S["BI_ERR_INVALID_ARG"]         # ldq < K
    assert call(8, 65) == S["BI_ERR_INVALID_ARG"]         # odd ldq
    assert call(0, 257) == S["BI_ERR_ALIGNMENT"]
    assert call(5, 258) == S["BI_ERR_ALIGNMENT"]
    assert call(6, 258) == S["BI_ERR_ALIGNMENT"]
    if not __import__("torch").cuda.is_available():   # valid arguments: only without a GPU
        assert call() == S["BI_ERR_NO_DEVICE"]
        assert call(6, None) == S["BI_ERR_NO_DEVICE"]
