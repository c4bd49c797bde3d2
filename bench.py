"""Benchmark of the batch-invariant GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}] [--no-extras]

One step is one pass of the decode-shaped workload: the bf16 GEMM C = A . B^T with N = 4096,
K = 7168, swept over M = 1, 2, 4, ..., 256 (nine GEMM calls, each through the C ABI).  The
weights rotate over enough copies that every call reads them from HBM (the copies together
are larger than twice the 126 MB L2).  A step is captured once per rotation phase as a CUDA
graph and replayed, so the timed region measures the kernels, not Python.  The metric is the
algorithmic HBM throughput: weight, activation and output bytes, each counted once, over the
device time (CUDA events on the launching stream, max over ranks).

Under torchrun (N > 1) every rank runs the same sweep on its own GPU with its own data: the
units are independent problems (weak scaling), and the only collectives are the barriers and
the max of the timings.  Rank 0 prints one JSON line.

``--impl reference`` times the CPU oracle instead (the only other place this file runs it), on a
bounded sample of the same workload, scaled to the same unit.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

REPO = os.path.dirname(os.path.abspath(__file__))
if REPO not in sys.path:
    sys.path.insert(0, REPO)

METRIC = "batch-invariant GEMM TFLOP/s & HBM GB/s vs M, % roofline; 0 bitwise row diffs"
N_DEC, K_DEC = 4096, 7168
M_SWEEP = [1, 2, 4, 8, 16, 32, 64, 128, 256]
WORKLOAD = ("decode-shaped bf16 GEMM C=A.B^T, N=4096, K=7168, M swept 1,2,4,...,256 "
            "(9 GEMMs per step); A~N(0,1), B~N(0,1/K) in bf16")



def weight_plan(N, K, dtype=None, experts=1):
    """A plan for the benchmark's weights: they are written once before the timed region and
    only read inside it, so every plan declares them resident (BI_PLAN_RESIDENT_WEIGHTS)."""
    import invariant_deterministic_gemm_bi_b200 as bg
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_BF16 if dtype is None else dtype, experts)
    bg.bi_gemm_plan_set_flags(plan, bg.BI_PLAN_RESIDENT_WEIGHTS)
    return plan


def sweep_bytes(n=N_DEC, k=K_DEC, ms=M_SWEEP, elt=2):
    """Algorithmic bytes of one step: each operand once plus the output."""
    return sum(n * k * elt + m * k * elt + 2 * m * n for m in ms)


def sweep_flops(n=N_DEC, k=K_DEC, ms=M_SWEEP):
    return sum(2 * m * n * k for m in ms)


def sweep_macs(n=N_DEC, k=K_DEC, ms=M_SWEEP):
    return sum(m * n * k for m in ms)


def moe_routed_rows(bg, inputs, T, E, K, seed, dev, stream=None, topk=8):
    """The grouped GEMM's inputs for T tokens, built on the GPU by the library's own MoE steps:
    router logits ~ N(0, 1) (seeded, drawn on the host), bi_moe_route_topk (top-8, ties to the
    lower expert), bi_moe_dispatch (stable grouping by expert) and bi_moe_gather_rows.  Returns
    (A_perm [T*8, K] bf16, expert offsets int32 [E+1], number of experts with rows)."""
    import torch
    g = inputs.generator(seed, "cpu")
    logits = torch.randn(T, E, generator=g, dtype=torch.float32).to(dev)
    tokens = inputs.bf16_gaussian((T, K), seed=seed + 1, device=dev)
    R = T * topk
    ex = torch.empty((T, topk), dtype=torch.int32, device=dev)
    w = torch.empty((T, topk), dtype=torch.float32, device=dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    tok = torch.empty(R, dtype=torch.int32, device=dev)
    ros = torch.empty(R, dtype=torch.int32, device=dev)
    A = torch.empty((R, K), dtype=torch.bfloat16, device=dev)
    bg.bi_moe_route_topk(logits, topk, ex, w, stream=stream)
    bg.bi_moe_dispatch(ex, E, off, tok, ros, stream=stream)
    bg.bi_moe_gather_rows(tokens, tok, A, stream=stream)
    torch.cuda.synchronize()
    active = int((off[1:] > off[:-1]).sum().item())
    return A, off, active


def load_peaks():
    path = os.path.join(REPO, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p.get("hbm_gbs", 6650.0), "bf16_tflops": p.get("bf16_tflops", 1590.0),
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", 1400.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------

class ClockSampler:
    """Polls NVML (SM clock and throttle reasons) from a thread while the timed region runs."""

    REASONS = {
        "hw_slowdown": 0x0000000000000008, "sw_thermal_slowdown": 0x0000000000000020,
        "hw_thermal_slowdown": 0x0000000000000040, "sw_power_cap": 0x0000000000000004,
        "hw_power_brake_slowdown": 0x0000000000000080,
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None

    def _handle(self, device_index):
        """The NVML handle of this process's CUDA device (NVML numbers every GPU of the host)."""
        import torch
        nv = self.nvml
        props = torch.cuda.get_device_properties(device_index)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return nv.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
            except Exception:
                pass
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            devid = getattr(props, "pci_device_id", 0)
            try:
                return nv.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{devid:02x}.0")
            except Exception:
                pass
        return nv.nvmlDeviceGetHandleByIndex(device_index)

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------------
# CPU oracle (the baseline leg and the reference arm)
# ---------------------------------------------------------------------------------------------

def oracle_sample(seconds_budget: float, rng_seed: int = 2000):
    """Time the CPU oracle on a bounded sample of the decode sweep.

    The sample keeps every row of the sweep (sum of M = 511 rows) and the first n_cols output
    columns, with n_cols chosen from a calibration run so the sample takes about
    ``seconds_budget``; when a whole step takes less than that, the whole step is repeated
    instead.  The oracle's cost is proportional to multiply-adds, so its throughput is reported
    as the full workload's algorithmic bytes scaled by the (fractional) number of steps done,
    per second.
    """
    import numpy as np

    import oracle
    from invariant_deterministic_gemm_bi_b200 import inputs

    threads = oracle.default_threads()
    rows = sum(M_SWEEP)
    A = inputs.to_numpy_bits(inputs.bf16_gaussian((rows, K_DEC), seed=rng_seed))
    Bfull = inputs.to_numpy_bits(inputs.bf16_gaussian((N_DEC, K_DEC), seed=rng_seed + 1,
                                                      std=K_DEC ** -0.5))
    oracle.gemm_bf16(A, Bfull[:8], threads=threads)    # warm-up (thread start, page-in)
    t0 = time.perf_counter()
    oracle.gemm_bf16(A, Bfull[:128], threads=threads)
    per_col = max((time.perf_counter() - t0) / 128, 1e-6)
    if per_col * N_DEC >= seconds_budget:   # a column slice of one step fills the budget
        n_cols, reps = int(max(1, seconds_budget / per_col)), 1
    else:                                   # whole steps, repeated to fill the budget
        n_cols, reps = N_DEC, max(1, int(round(seconds_budget / (per_col * N_DEC))))
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.gemm_bf16(A, Bfull[:n_cols], threads=threads)
    dt = time.perf_counter() - t0
    frac = n_cols / N_DEC
    value = sweep_bytes() * frac * reps / dt / 1e9
    what = (f"all {rows} rows of the M sweep x first {n_cols} of {N_DEC} output columns "
            f"({frac:.4f} of the step's multiply-adds)" if reps == 1 else
            f"the whole step (all {rows} rows of the M sweep x all {N_DEC} output columns), "
            f"{reps} times")
    return {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{what} in {dt:.2f} s; value = step bytes x steps done / time",
            "seconds": dt, "n_cols": n_cols}


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    steps, warmup = args.steps, args.warmup
    budget = max(0.02, min(5.0, 90.0 / max(1, steps + warmup)))
    cal = oracle_sample(budget)
    n_cols = cal["n_cols"]

    import oracle
    from invariant_deterministic_gemm_bi_b200 import inputs
    rows = sum(M_SWEEP)
    A = inputs.to_numpy_bits(inputs.bf16_gaussian((rows, K_DEC), seed=2000))
    B = inputs.to_numpy_bits(inputs.bf16_gaussian((N_DEC, K_DEC), seed=2001, std=K_DEC ** -0.5))[:n_cols]
    threads = oracle.default_threads()
    for _ in range(warmup):
        oracle.gemm_bf16(A, B, threads=threads)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.gemm_bf16(A, B, threads=threads)
    dt = time.perf_counter() - t0
    frac = n_cols / N_DEC
    value = sweep_bytes() * frac * steps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warmup,
        "ms_per_step": dt / steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": f"first {n_cols} of {N_DEC} output columns per step"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"all {rows} sweep rows x {n_cols} output columns per step, "
                                   f"scaled by the fraction of multiply-adds ({frac:.4f})"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="skip the other workloads' timings")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["decode", "prefill", "fp8", "w4a8", "moe", "attention"],
                    default=None,
                    help="launch one workload --profile-launches times, untimed (for ncu captures)")
    ap.add_argument("--profile-m", type=int, default=64,
                    help="M for --profile (MoE: tokens T; attention: batch, sequences of length 4096)")
    ap.add_argument("--profile-splits", type=int, default=4, help="attention: KV splits (1, 2, 4)")
    ap.add_argument("--profile-launches", type=int, default=4)
    ap.add_argument("--profile-nk", choices=["7168x2048", "2048x7168"], default="7168x2048",
                    help="prefill: the (N, K) of the weight")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return reference_arm(args)
    if args.profile:
        return profile_case(args)

    import torch
    import torch.distributed as dist

    import invariant_deterministic_gemm_bi_b200 as bg
    from invariant_deterministic_gemm_bi_b200 import inputs

    global max_over_ranks
    from invariant_deterministic_gemm_bi_b200.sharding import max_over_ranks

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 1024 * 1024) or 126 * 1024 * 1024
    wbytes = N_DEC * K_DEC * 2
    n_copies = math.ceil(2 * l2 / wbytes) + 1

    # inputs resident in HBM before the timed region (rank-specific seeds: independent problems)
    seed = 2000 + 97 * rank
    Bs = [inputs.bf16_gaussian((N_DEC, K_DEC), seed=seed + 1 + i, std=K_DEC ** -0.5, device=dev)
          for i in range(n_copies)]
    Amax = inputs.bf16_gaussian((max(M_SWEEP), K_DEC), seed=seed, device=dev)
    As = {m: Amax[:m] for m in M_SWEEP}
    Cs = {m: torch.empty((m, N_DEC), dtype=torch.bfloat16, device=dev) for m in M_SWEEP}
    plan = weight_plan(N_DEC, K_DEC)
    stream = torch.cuda.Stream(device=dev)

    def run_step(phase):
        for i, m in enumerate(M_SWEEP):
            b = Bs[(phase * len(M_SWEEP) + i) % n_copies]
            bg.bi_gemm_run(plan, As[m], b, Cs[m], stream=stream)

    # one CUDA graph per rotation phase
    with torch.cuda.stream(stream):
        run_step(0)
        torch.cuda.synchronize()
        bg.bi_gemm_sync_status(plan, stream=stream)
        graphs = []
        for ph in range(n_copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                run_step(ph)
            graphs.append(g)
    torch.cuda.synchronize()

    for s in range(args.warmup):
        graphs[s % n_copies].replay()
    torch.cuda.synchronize()
    barrier()

    sampler = ClockSampler(local)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    torch.cuda.synchronize()
    barrier()
    sampler.start()
    with torch.cuda.stream(stream):
        ev[0].record(stream)
        for s in range(args.steps):
            graphs[s % n_copies].replay()
            ev[s + 1].record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    st = bg.bi_gemm_sync_status(plan, stream=stream, raise_on_error=False)
    if st != 0:
        raise RuntimeError(f"device status after the timed region: {bg.binding.STATUS_NAMES[st]}")
    total_ms = ev[0].elapsed_time(ev[-1])
    step_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = max_over_ranks(total_ms, device=dev)

    peaks = load_peaks()
    step_bytes = sweep_bytes()
    value = step_bytes * args.steps * world / (total_ms * 1e-3) / 1e9
    tflops = sweep_flops() * args.steps * world / (total_ms * 1e-3) / 1e12
    # roofline of the (only) kernel of the step: average launch duration from the per-step events
    launches = len(M_SWEEP)
    avg_launch_s = (sum(step_ms) / len(step_ms)) / launches * 1e-3
    achieved = step_bytes / launches / avg_launch_s / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                "peak_source": peaks["source"], "kernel": kernel_label(bg, plan),
                "note": "per-launch time = step time / 9 (graph gaps included)"}
    traffic = os.path.join(REPO, "profiles", "decode_bf16_traffic.json")
    if os.path.exists(traffic):
        with open(traffic) as f:
            tr = json.load(f)
        if tr.get("kernel_source_hash") == kernel_source_hash():
            roofline["traffic"] = tr["bytes_per_launch"]
            roofline["traffic_from"] = tr["kernel"]

    # row invariance on this workload: the M=256 rows against the same rows run at M=1
    row_diffs = 0
    with torch.cuda.stream(stream):
        C256 = torch.empty((256, N_DEC), dtype=torch.bfloat16, device=dev)
        bg.bi_gemm_run(plan, Amax, Bs[0], C256, stream=stream)
        for r in [0, 1, 63, 127, 128, 200, 255]:
            c1 = torch.empty((1, N_DEC), dtype=torch.bfloat16, device=dev)
            bg.bi_gemm_run(plan, Amax[r:r + 1], Bs[0], c1, stream=stream)
            stream.synchronize()
            row_diffs += int(not torch.equal(c1.view(torch.int16)[0], C256.view(torch.int16)[r]))
    torch.cuda.synchronize()

    e2e = measure_e2e(bg, plan, Bs, dev, stream, args, world, barrier)
    per_m = measure_per_m(bg, plan, As, Bs, Cs, dev, stream, n_copies, peaks)
    extras = None if args.no_extras else measure_extras(bg, inputs, dev, stream, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(15.0)
        cpu = {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample")}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "per_gpu": "independent sweep per rank",
                       "l2": f"{n_copies} rotating weight copies ({n_copies * wbytes / 2**20:.0f} MiB"
                             f" > 2 x {l2 / 2**20:.0f} MiB L2)",
                       "timing": "CUDA graph replay per step, CUDA events, max over ranks",
                       "weights": "resident (BI_PLAN_RESIDENT_WEIGHTS: B requested before the "
                                  "previous GEMM in the stream completes)",
                       "parallelism": f"replicas x{world} (M-sharded independent problems)"},
            "tflops": tflops,
            "roofline": roofline, "clocks": clocks, "e2e": e2e,
            "gpu_launches": launches * args.steps, "row_diffs": row_diffs,
            "per_m": per_m, "cpu_baseline": cpu, "extras": extras,
        }
        print(json.dumps(line), flush=True)
    del graphs
    if world > 1:
        dist.destroy_process_group()
    return 0


def profile_case(args):
    """Launch one workload a fixed number of times with rotating weights (no timing)."""
    import torch

    import invariant_deterministic_gemm_bi_b200 as bg
    from invariant_deterministic_gemm_bi_b200 import inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    M, L = args.profile_m, args.profile_launches
    calls = []
    if args.profile in ("decode", "prefill"):
        N, K = (N_DEC, K_DEC) if args.profile == "decode" else tuple(map(int, args.profile_nk.split("x")))
        plan = weight_plan(N, K)
        copies = 3 if args.profile == "decode" else 1
        Bs = [inputs.bf16_gaussian((N, K), seed=11 + i, std=K ** -0.5, device=dev) for i in range(copies)]
        A = inputs.bf16_gaussian((M, K), seed=10, device=dev)
        C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        calls = [lambda i=i: bg.bi_gemm_run(plan, A, Bs[i % copies], C) for i in range(L)]
    elif args.profile == "fp8":
        N = K = 7168
        KB = K // 128
        plan = weight_plan(N, K, bg.BI_DTYPE_E4M3_BLOCKSCALED)
        qbs = [inputs.e4m3_gaussian((N, K), seed=21 + i, device=dev) for i in range(3)]
        sb = inputs.scales_log_uniform((N // 128, KB), seed=22, device=dev)
        qa = inputs.e4m3_gaussian((M, K), seed=23, device=dev)
        sa = inputs.scales_log_uniform((KB, ((M + 3) // 4) * 4), seed=24, device=dev)[:, :M]
        C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        calls = [lambda i=i: bg.bi_gemm_run(plan, qa, qbs[i % 3], C, scale_a=sa, scale_b=sb)
                 for i in range(L)]
    elif args.profile == "w4a8":
        N = K = 7168
        KB = K // 128
        plan = weight_plan(N, K, bg.BI_DTYPE_E2M1_W4A8)
        qws = [inputs.e2m1_packed_uniform(N, K, seed=61 + i, device=dev) for i in range(6)]
        ws = inputs.channel_scales_pow2(N, seed=62, device=dev)
        wz = inputs.channel_zeros_fp16(ws, seed=63)
        qa = inputs.e4m3_gaussian((M, K), seed=64, device=dev)
        sa = inputs.scales_log_uniform((KB, ((M + 3) // 4) * 4), seed=65, device=dev)[:, :M]
        C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        work = torch.empty(bg.bi_gemm_w4a8_workspace_bytes(M) // 4, dtype=torch.float32, device=dev)
        calls = [lambda i=i: bg.bi_gemm_run_w4a8(plan, qa, sa, qws[i % 6], ws, C, w_zero=wz,
                                                 workspace=work) for i in range(L)]
    elif args.profile == "attention":
        # the attention_B{M}_L4096 workload of the extras: Hq = 32, Hkv = 8, D = 128
        import math
        Hq, Hkv, D, L4 = 32, 8, 128, 4096
        Q = inputs.bf16_gaussian((M, Hq, D), seed=8001, device=dev)
        Kc = inputs.bf16_gaussian((M, L4, Hkv, D), seed=8002, device=dev)
        Vc = inputs.bf16_gaussian((M, L4, Hkv, D), seed=8003, device=dev)
        lens = torch.full((M,), L4, dtype=torch.int32, device=dev)
        O = torch.empty((M, Hq, D), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(bg.bi_decode_attention_workspace_bytes(M, Hq, D, 4) // 4, dtype=torch.float32,
                         device=dev)
        for _ in range(L):
            bg.bi_decode_attention(Q, Kc, Vc, lens, O, 1.0 / math.sqrt(D), splits=args.profile_splits,
                                   workspace=ws)
        torch.cuda.synchronize()
        ok = not bool(torch.isnan(O.float()).any())
        print(json.dumps({"profile": "attention", "B": M, "splits": args.profile_splits, "launches": L,
                          "finite": ok}))
        return 0 if ok else 1
    else:
        E, N, K = 64, 2048, 7168
        plan = weight_plan(N, K, bg.BI_DTYPE_BF16, E)
        B = inputs.bf16_gaussian((E, N, K), seed=31, std=K ** -0.5, device=dev)
        A, off, _ = moe_routed_rows(bg, inputs, M, E, K, seed=32, dev=dev)
        C = torch.empty((A.shape[0], N), dtype=torch.bfloat16, device=dev)
        calls = [lambda: bg.bi_grouped_gemm_run(plan, A, B, C, off) for _ in range(L)]
    for f in calls:
        f()
    torch.cuda.synchronize()
    st = bg.bi_gemm_sync_status(plan, raise_on_error=False)
    print(json.dumps({"profile": args.profile, "M": M, "launches": L, "status": st}))
    return 0 if st == 0 else 1


def kernel_label(bg, plan) -> str:
    """The plan's kernel: its tile, instruction K order, and the full-height ring depths (each
    launch picks one of the plan's scheduling forms by M; the sweep runs five of them)."""
    i = bg.bi_gemm_plan_describe(plan)
    dt = {0: "bf16", 1: "e4m3", 2: "e2m1 x e4m3"}[i["dtype"]]
    order = {0: "ascending K", 1: "split-K", 2: "two K chains", 3: "four K chains"}[i["k_order_id"]]
    return (f"bi_gemm_kernel<BM={i['block_m']},BN={i['block_n']},{dt}>, {order},"
            f" every scheduling form of the plan (full-height rings A{i['stages_a']}/B{i['stages']})")


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("bi_kernels.cuh", "ptx_sm100.cuh", "bi_gemm.cu"):
        with open(os.path.join(REPO, "invariant_deterministic_gemm_bi_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def gpu_numa_node(dev) -> int | None:
    """NUMA node of the GPU's PCI device (sysfs), found through NVML by the device UUID."""
    try:
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        for i in range(pynvml.nvmlDeviceGetCount()):
            h = pynvml.nvmlDeviceGetHandleByIndex(i)
            u = pynvml.nvmlDeviceGetUUID(h)
            u = u.decode() if isinstance(u, bytes) else u
            if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                bus = pynvml.nvmlDeviceGetPciInfo(h).busId
                bus = bus.decode() if isinstance(bus, bytes) else bus
                dom, rest = bus.split(":", 1)
                path = f"/sys/bus/pci/devices/{int(dom, 16):04x}:{rest.lower()}/numa_node"
                with open(path) as f:
                    return int(f.read().strip())
    except Exception:
        return None
    return None


def node_cpus(node: int) -> set:
    try:
        with open(f"/sys/devices/system/node/node{node}/cpulist") as f:
            text = f.read().strip()
    except OSError:
        return set()
    cpus = set()
    for part in text.split(","):
        if "-" in part:
            a, b = part.split("-")
            cpus.update(range(int(a), int(b) + 1))
        elif part:
            cpus.add(int(part))
    return cpus


def measure_e2e(bg, plan, Bs, dev, stream, args, world, barrier):
    """The same sweep end to end through the library's host-buffer call.

    Each step is one bi_gemm_run_host_batch call with the sweep's nine GEMMs: pinned host A
    slices in, the kernels, pinned host C results out.  The slices of a step lie back to back in
    one pinned block for A and one for C, so the library moves each with one copy.  It runs the
    copy-ins on a copy-in stream, the kernels on the compute stream and the copy-outs on a
    copy-out stream, ordered by its own events over 3 staging regions (one per step in flight):
    a step's copy-in runs under the previous step's kernels and its copy-out under the kernels
    two steps later.  The host buffers are pinned on the GPU's NUMA node when it is known.  The
    record
    also holds the pinned copy bandwidth measured in this run (one 256 MiB cudaMemcpyAsync each
    way, then both at once on two streams) and the time of the step's own copy-in and copy-out
    run alone at once (copy_floor_ms_per_step), the bound the end-to-end step cannot beat."""
    import torch
    from invariant_deterministic_gemm_bi_b200 import inputs
    steps = max(2, min(args.steps, 400))
    node = gpu_numa_node(dev)
    affinity = None
    if node is not None and node >= 0 and hasattr(os, "sched_setaffinity"):
        here = os.sched_getaffinity(0)
        local = node_cpus(node) & here
        if local:
            affinity = here
            os.sched_setaffinity(0, local)   # pinned pages are placed on the allocating CPU's node
    rows = sum(M_SWEEP)
    offs = {}
    o = 0
    for m in M_SWEEP:
        offs[m] = o
        o += m
    try:
        # one step's activations and results, each laid out back to back in one pinned block (as
        # a serving loop's activation arena would be): the library moves each with one copy
        A_block = inputs.bf16_gaussian((rows, K_DEC), seed=77).pin_memory()
        C_block = torch.empty((rows, N_DEC), dtype=torch.bfloat16).pin_memory()
        probe_h = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
    finally:
        if affinity is not None:
            os.sched_setaffinity(0, affinity)
    probe_d = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def copy_gbs(dst, src):
        best = None
        with torch.cuda.stream(stream):
            for _ in range(3):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                dst.copy_(src, non_blocking=True)
                e1.record(stream)
                e1.synchronize()
                t = e0.elapsed_time(e1) * 1e-3
                best = t if best is None else min(best, t)
        return probe_h.numel() / best / 1e9
    h2d_gbs = copy_gbs(probe_d, probe_h)
    d2h_gbs = copy_gbs(probe_h, probe_d)
    # both directions at once, on two streams: whether the link carries them in parallel
    probe_d2 = torch.empty_like(probe_d)
    probe_h2 = torch.empty_like(probe_h).pin_memory()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    both = None
    for _ in range(3):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        with torch.cuda.stream(s_in):
            probe_d.copy_(probe_h, non_blocking=True)
        with torch.cuda.stream(s_out):
            probe_h2.copy_(probe_d2, non_blocking=True)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
        e1.record(stream)
        e1.synchronize()
        t = e0.elapsed_time(e1) * 1e-3
        both = t if both is None else min(both, t)
    duplex_gbs = 2 * probe_h.numel() / both / 1e9
    del probe_d, probe_h, probe_d2, probe_h2

    # the step's own copies alone (its activations in, its results out, on two streams at once):
    # the bound the end-to-end step cannot beat
    a_dev = torch.empty_like(A_block, device=dev)
    c_dev = torch.empty_like(C_block, device=dev)
    copies = None
    for _ in range(5):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        with torch.cuda.stream(s_in):
            a_dev.copy_(A_block, non_blocking=True)
        with torch.cuda.stream(s_out):
            C_block.copy_(c_dev, non_blocking=True)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
        e1.record(stream)
        e1.synchronize()
        t = e0.elapsed_time(e1)
        copies = t if copies is None else min(copies, t)
    del a_dev, c_dev

    # each block is one allocation: the library may move a step's slices with one copy each way
    bg.bi_gemm_plan_set_flags(plan, bg.BI_PLAN_RESIDENT_WEIGHTS | bg.BI_PLAN_HOST_ROW_BLOCKS)
    n_copies = len(Bs)
    arrays = [bg.host_gemm_array([(A_block[offs[m]:offs[m] + m], Bs[(ph * len(M_SWEEP) + i) % n_copies],
                                   C_block[offs[m]:offs[m] + m])
                                  for i, m in enumerate(M_SWEEP)]) for ph in range(n_copies)]
    # three steps' worth of staging regions: a step's copy-ins run while the previous step
    # computes, and its copy-outs two steps later
    staging = torch.empty(bg.bi_gemm_host_batch_staging_bytes(plan, arrays[0], 3),
                          dtype=torch.uint8, device=dev)
    cin, cout = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    cap = torch.cuda.Stream(device=dev)

    def batch(s, compute):
        bg.bi_gemm_run_host_batch(plan, arrays[s % n_copies], staging, copy_in=cin, compute=compute,
                                  copy_out=cout)

    # One CUDA graph holds 3 x n_copies consecutive steps (three turns of the weight rotation) and
    # a flush: inside it the library's events let the steps' copies overlap the neighbouring
    # steps' kernels; consecutive replays run in stream order.
    for s in range(n_copies):
        batch(s, stream)                      # outside capture: status words, kernel attributes
    bg.bi_gemm_host_batch_flush(plan, copy_in=cin, compute=stream, copy_out=cout)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    per_graph = 3 * n_copies
    with torch.cuda.graph(graph, stream=cap):
        for s in range(per_graph):
            batch(s, cap)
        bg.bi_gemm_host_batch_flush(plan, copy_in=cin, compute=cap, copy_out=cout)
    replays = max(1, steps // per_graph)
    steps = replays * per_graph

    def timed():
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(replays):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), device=dev)

    with torch.cuda.stream(stream):
        graph.replay()
    ms = timed()
    del graph
    # the last step's results, now in pinned host memory, against the same GEMMs run directly
    last = (steps - 1) % n_copies
    check_ok = True
    with torch.cuda.stream(stream):
        for i, m in enumerate(M_SWEEP):
            ref = torch.empty((m, N_DEC), dtype=torch.bfloat16, device=dev)
            bg.bi_gemm_run(plan, A_block[offs[m]:offs[m] + m].to(dev), Bs[(last * len(M_SWEEP) + i) % n_copies],
                           ref, stream=stream)
            torch.cuda.synchronize()
            check_ok &= bool(torch.equal(ref.cpu().view(torch.int16),
                                         C_block[offs[m]:offs[m] + m].view(torch.int16)))

    h2d = sum(m * K_DEC * 2 for m in M_SWEEP)
    d2h = sum(m * N_DEC * 2 for m in M_SWEEP)
    return {"value": sweep_bytes() * steps * world / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": ms / steps,
            "path": ("bi_gemm_run_host_batch, one call per step with the sweep's nine GEMMs, whose "
                     "activations and results lie back to back in one pinned block each: one "
                     "copy-in on a copy-in stream, the kernels on the compute stream, one copy-out "
                     "(two steps later) on a copy-out stream, ordered by the library's events over "
                     "3 staging regions; %d steps and a flush per captured CUDA graph, replayed "
                     "back to back" % per_graph),
            "copy_floor_ms_per_step": copies,
            "pinned_h2d_gbs": h2d_gbs, "pinned_d2h_gbs": d2h_gbs,
            "pinned_both_directions_gbs": duplex_gbs,
            "gpu_numa_node": node, "host_buffers_on_gpu_node": affinity is not None,
            "results_match_device_run": check_ok}


def graph_time_per_launch(fn_list, stream, reps=20):
    """Capture the launches in fn_list into one graph, replay it, return seconds per launch."""
    import torch
    with torch.cuda.stream(stream):
        for f in fn_list:
            f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for f in fn_list:
                f()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del g
    return ms * 1e-3 / (reps * len(fn_list))


def measure_per_m(bg, plan, As, Bs, Cs, dev, stream, n_copies, peaks):
    out = []
    for m in M_SWEEP:
        fns = [lambda i=i: bg.bi_gemm_run(plan, As[m], Bs[i % n_copies], Cs[m], stream=stream)
               for i in range(2 * n_copies)]
        t = graph_time_per_launch(fns, stream)
        b = N_DEC * K_DEC * 2 + m * K_DEC * 2 + m * N_DEC * 2
        gbs = b / t / 1e9
        out.append({"M": m, "us": t * 1e6, "GB/s": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                    "TFLOP/s": 2 * m * N_DEC * K_DEC / t / 1e12})
    return out


def measure_extras(bg, inputs, dev, stream, peaks):
    """The other workloads (small, prefill, FP8, W4A8, MoE and its layer steps, attention, the
    split-K variant): throughput and roofline fraction (not part of `value`)."""
    import time
    import torch
    res = {}
    bf16_peak = peaks["bf16_tflops"]
    fp8_peak = 2.0 * bf16_peak          # nominal dense fp8 : bf16 ratio
    hbm = peaks["hbm_gbs"]

    def settle():
        # a pause between workloads, so that one does not start under the power and clock state a
        # kilowatt-class predecessor (the prefill GEMMs) left behind
        torch.cuda.synchronize()
        time.sleep(1.0)
    # the small correctness shape N = 256, K = 512 (its 256 KB of weights stay in L2, so this is
    # launch latency, not HBM): per launch inside a graph
    plan = weight_plan(256, 512)
    B = inputs.bf16_gaussian((256, 512), seed=1001, device=dev)
    for M in [1, 3, 8, 17, 64]:
        A = inputs.bf16_gaussian((M, 512), seed=1002, device=dev)
        C = torch.empty((M, 256), dtype=torch.bfloat16, device=dev)
        t = graph_time_per_launch([lambda: bg.bi_gemm_run(plan, A, B, C, stream=stream)] * 16,
                                  stream, reps=8)
        b = 2 * (M * 512 + 256 * 512 + M * 256)
        res[f"small_N256_K512_M{M}"] = {"us": t * 1e6, "GB/s": b / t / 1e9,
                                        "TFLOP/s": 2 * M * 256 * 512 / t / 1e12}
        del A, C
    settle()
    # prefill, M = 16384 and 4096
    for (N, K) in [(7168, 2048), (2048, 7168)]:
        plan = weight_plan(N, K)
        B = inputs.bf16_gaussian((N, K), seed=3001, std=K ** -0.5, device=dev)
        for M in [1024, 4096, 16384]:
            A = inputs.bf16_gaussian((M, K), seed=3002, device=dev)
            C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            t = graph_time_per_launch([lambda: bg.bi_gemm_run(plan, A, B, C, stream=stream)] * 5,
                                      stream, reps=4)
            tf = 2 * M * N * K / t / 1e12
            res[f"prefill_N{N}_K{K}_M{M}"] = {"us": t * 1e6, "TFLOP/s": tf,
                                              "tensor_frac": tf / bf16_peak}
            del A, C
    settle()
    # FP8 N = K = 7168
    N = K = 7168
    KB = K // 128
    plan = weight_plan(N, K, bg.BI_DTYPE_E4M3_BLOCKSCALED)
    qbs = [inputs.e4m3_gaussian((N, K), seed=4001 + i, device=dev) for i in range(4)]
    sb = inputs.scales_log_uniform((N // 128, KB), seed=4002, device=dev)
    for M in [1, 4, 16, 64, 256, 1024, 4096]:
        qa = inputs.e4m3_gaussian((M, K), seed=4003, device=dev)
        sa = inputs.scales_log_uniform((KB, ((M + 3) // 4) * 4), seed=4004, device=dev)[:, :M]
        C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        fns = [lambda i=i: bg.bi_gemm_run(plan, qa, qbs[i % 4], C, scale_a=sa, scale_b=sb,
                                          stream=stream) for i in range(8)]
        t = graph_time_per_launch(fns, stream, reps=4)
        b = N * K + M * K + 2 * M * N + 4 * M * KB + 4 * (N // 128) * KB
        tf = 2 * M * N * K / t / 1e12
        res[f"fp8_M{M}"] = {"us": t * 1e6, "TFLOP/s": tf, "tensor_frac": tf / fp8_peak,
                            "GB/s": b / t / 1e9, "hbm_frac": b / t / 1e9 / hbm}
    del qbs
    settle()
    # e2m1 weights (per-channel 2^-j scale and fp16 zero point) x e4m3 activations, N = K = 7168;
    # 8 weight copies (205 MB) rotate so that every launch reads W from HBM
    plan = weight_plan(N, K, bg.BI_DTYPE_E2M1_W4A8)
    qws = [inputs.e2m1_packed_uniform(N, K, seed=6001 + i, device=dev) for i in range(8)]
    ws = inputs.channel_scales_pow2(N, seed=6002, device=dev)
    wz = inputs.channel_zeros_fp16(ws, seed=6003)
    for M in [1, 64, 4096]:
        qa = inputs.e4m3_gaussian((M, K), seed=6004, device=dev)
        sa = inputs.scales_log_uniform((KB, ((M + 3) // 4) * 4), seed=6005, device=dev)[:, :M]
        C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        work = torch.empty(bg.bi_gemm_w4a8_workspace_bytes(M) // 4, dtype=torch.float32, device=dev)
        fns = [lambda i=i: bg.bi_gemm_run_w4a8(plan, qa, sa, qws[i % 8], ws, C, w_zero=wz,
                                               workspace=work, stream=stream) for i in range(8)]
        t = graph_time_per_launch(fns, stream, reps=4)
        b = N * K // 2 + M * K + 2 * M * N + 4 * M * KB + 8 * N + 8 * M
        tf = 2 * M * N * K / t / 1e12
        res[f"w4a8_M{M}"] = {"us": t * 1e6, "TFLOP/s": tf, "tensor_frac": tf / fp8_peak,
                             "GB/s": b / t / 1e9, "hbm_frac": b / t / 1e9 / hbm}
        if M in (1, 4096):   # without zero points: no row-sum kernel, C = scale * acc
            fns = [lambda i=i: bg.bi_gemm_run_w4a8(plan, qa, sa, qws[i % 8], ws, C, stream=stream)
                   for i in range(8)]
            t = graph_time_per_launch(fns, stream, reps=4)
            b = N * K // 2 + M * K + 2 * M * N + 4 * M * KB + 4 * N
            res[f"w4a8_M{M}_no_zero"] = {"us": t * 1e6, "TFLOP/s": 2 * M * N * K / t / 1e12,
                                         "GB/s": b / t / 1e9, "hbm_frac": b / t / 1e9 / hbm}
    del qws
    # e2m1 quantisation of the bf16 weights of the same shape (a weight-preparation step)
    Wb = inputs.bf16_gaussian((N, K), seed=6006, std=0.01, device=dev)
    Qw = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    t = graph_time_per_launch([lambda: bg.bi_quantize_e2m1(Wb, ws, Qw, w_zero=wz, stream=stream)] * 4,
                              stream, reps=4)
    b = N * K * 2 + N * K // 2 + 8 * N
    res["quantize_e2m1_7168x7168"] = {"us": t * 1e6, "GB/s": b / t / 1e9, "hbm_frac": b / t / 1e9 / hbm}
    del Wb, Qw
    settle()
    # MoE: 64 experts, N = 2048, K = 7168, top-8
    E, N, K = 64, 2048, 7168
    plan = weight_plan(N, K, bg.BI_DTYPE_BF16, E)
    B = inputs.bf16_gaussian((E, N, K), seed=5001, std=K ** -0.5, device=dev)
    for T in [1, 64, 1024, 8192]:
        A, off, active = moe_routed_rows(bg, inputs, T, E, K, seed=5000 + T, dev=dev, stream=stream)
        C = torch.empty((A.shape[0], N), dtype=torch.bfloat16, device=dev)
        t = graph_time_per_launch([lambda: bg.bi_grouped_gemm_run(plan, A, B, C, off, stream=stream)] * 3,
                                  stream, reps=4)
        rows = A.shape[0]
        b = active * N * K * 2 + rows * K * 2 + rows * N * 2
        tf = 2 * rows * N * K / t / 1e12
        res[f"moe_T{T}"] = {"us": t * 1e6, "TFLOP/s": tf, "tensor_frac": tf / bf16_peak,
                            "GB/s": b / t / 1e9, "hbm_frac": b / t / 1e9 / hbm,
                            "active_experts": active}
    del B
    # The MoE layer around the grouped GEMM at T = 8192 and 64: route, dispatch, gather, combine
    # (each timed on its own; bytes are the algorithmic ones of each step)
    E, N, K, k = 64, 2048, 7168, 8
    for T in (64, 8192):
        g = inputs.generator(7000 + T, "cpu")
        logits = torch.randn(T, E, generator=g, dtype=torch.float32).to(dev)
        toks = inputs.bf16_gaussian((T, K), seed=7001, device=dev)
        R = T * k
        ex = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        tok = torch.empty(R, dtype=torch.int32, device=dev)
        ros = torch.empty(R, dtype=torch.int32, device=dev)
        A = torch.empty((R, K), dtype=torch.bfloat16, device=dev)
        Cp = inputs.bf16_gaussian((R, N), seed=7002, device=dev)
        Y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
        steps = {
            "route": (lambda: bg.bi_moe_route_topk(logits, k, ex, w, stream=stream), T * E * 4 + T * k * 8),
            "dispatch": (lambda: bg.bi_moe_dispatch(ex, E, off, tok, ros, stream=stream), R * 4 * 3 + (E + 1) * 4),
            # each token row is read from HBM once (its k copies hit L2): T rows in, R rows out
            "gather": (lambda: bg.bi_moe_gather_rows(toks, tok, A, stream=stream), T * K * 2 + R * K * 2 + R * 4),
            "combine": (lambda: bg.bi_moe_combine(Cp, ros, w, Y, stream=stream), R * N * 2 + T * N * 2 + R * 8),
        }
        bg.bi_moe_route_topk(logits, k, ex, w, stream=stream)
        bg.bi_moe_dispatch(ex, E, off, tok, ros, stream=stream)
        for name, (fn, b) in steps.items():
            t = graph_time_per_launch([fn] * 8, stream, reps=4)
            res[f"moe_layer_T{T}_{name}"] = {"us": t * 1e6, "GB/s": b / t / 1e9,
                                             "hbm_frac": b / t / 1e9 / hbm}
        del A, Cp, Y, toks
    settle()
    # Dual-kernel decode attention: Hq = 32, Hkv = 8, D = 128, bf16 KV cache, every sequence at
    # length L; no split vs split-KV (bitwise equal outputs).  Bytes: K and V once, Q and O.
    import math
    Hq, Hkv, D = 32, 8, 128
    for (Bsz, L) in ((16, 4096), (64, 4096), (16, 32768)):
        Q = inputs.bf16_gaussian((Bsz, Hq, D), seed=8001, device=dev)
        Kc = inputs.bf16_gaussian((Bsz, L, Hkv, D), seed=8002, device=dev)
        Vc = inputs.bf16_gaussian((Bsz, L, Hkv, D), seed=8003, device=dev)
        lens = torch.full((Bsz,), L, dtype=torch.int32, device=dev)
        O = torch.empty((Bsz, Hq, D), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(bg.bi_decode_attention_workspace_bytes(Bsz, Hq, D, 4) // 4,
                         dtype=torch.float32, device=dev)
        b = 2 * Bsz * L * Hkv * D * 2 + 2 * Bsz * Hq * D * 2
        outs = {}
        for splits in (1, 2, 4):
            fn = lambda splits=splits: bg.bi_decode_attention(Q, Kc, Vc, lens, O, 1.0 / math.sqrt(D),
                                                              splits=splits, workspace=ws, stream=stream)
            t = graph_time_per_launch([fn] * 4, stream, reps=4)
            torch.cuda.synchronize()
            outs[splits] = O.clone()
            res[f"attention_B{Bsz}_L{L}_splits{splits}"] = {"us": t * 1e6, "GB/s": b / t / 1e9,
                                                            "hbm_frac": b / t / 1e9 / hbm}
        res[f"attention_B{Bsz}_L{L}_splits{splits}"]["bitwise_equal_to_no_split"] = all(
            torch.equal(outs[1].view(torch.int16), o.view(torch.int16)) for o in outs.values())
        del Q, Kc, Vc, O, ws
    settle()
    # Fixed-split-K research variant on the decode shape (not the product path): what dropping
    # split-K costs at small M.  Bytes are the algorithmic ones (workspace traffic not counted).
    N, K = N_DEC, K_DEC
    Bs = [inputs.bf16_gaussian((N, K), seed=6001 + i, std=K ** -0.5, device=dev) for i in range(4)]
    for S in (2, 4, 8):
        plan = bg.bi_gemm_plan_splitk(N, K, S)
        for M in (1, 16, 64, 256):
            A = inputs.bf16_gaussian((M, K), seed=6002, device=dev)
            C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(bg.bi_gemm_splitk_workspace_bytes(plan, M) // 4, dtype=torch.float32,
                             device=dev)
            fns = [lambda i=i: bg.bi_gemm_run_splitk(plan, A, Bs[i % 4], C, ws, stream=stream)
                   for i in range(8)]
            t = graph_time_per_launch(fns, stream, reps=4)
            b = 2 * N * K + 2 * M * K + 2 * M * N
            res[f"splitk_S{S}_M{M}"] = {"us": t * 1e6, "GB/s": b / t / 1e9,
                                        "hbm_frac": b / t / 1e9 / hbm,
                                        "tile": f"128x{bg.bi_gemm_plan_describe(plan)['block_n']}"}
            del A, C, ws
    return res


if __name__ == "__main__":
    sys.exit(main())
