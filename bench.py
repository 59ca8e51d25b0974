"""Benchmark of the W4A16 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload llama3_8b_decode|decode_sweep|prefill|llama3_70b]

Default workload: Llama-3-8B-shaped decode layers at M = 1 (q_proj 4096x4096,
gate_proj and up_proj 14336x4096, down_proj 4096x14336; W ~ N(0, 0.02) with
1% of input channels x10, asymmetric zero points, g = 128). One step is one
layer's four GEMVs; the steps walk through 32 layer copies (3.3 GB of packed
weights), so no step finds its weights in L2 (126 MB). Steps are replayed
from CUDA graphs. The timed region is bracketed by a barrier and a device
synchronize on both sides and timed with CUDA events; with several GPUs each
rank runs its own replica and the time is the max over ranks.

Printed: one JSON line (rank 0) with the effective HBM GB/s of the whole job
(algorithmic bytes / time), the roofline object of the GEMV kernel (per-launch
durations from CUDA events captured inside the timed graphs), the oracle
timed on the host cores (cpu_baseline), the end-to-end number through the
public API with host buffers (e2e), SM clocks sampled during the timed region,
and the tensor-core GEMM measured on the prefill shape (M = 2048).

--impl reference times the CPU oracle (the only other implementation of this
method here) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import LLAMA3_8B_DECODE, WORKLOADS, make_weight  # noqa: E402

METRIC = "W4A16 GEMV/GEMM TFLOP/s and effective HBM GB/s (fraction of roofline), M=1..2048"
HBM_FALLBACK_GBS = 6650.0
TENSOR_FALLBACK_TFLOPS = 1590.0
GEMV_PROFILE = os.path.join(ROOT, "profiles", "awq_gemv_llama3_8b_decode_m1.md")
CHAIN_PROFILE = os.path.join(ROOT, "profiles", "awq_gemv_chain_llama3_8b_decode_m1.md")
GEMM_PROFILE = os.path.join(ROOT, "profiles", "awq_gemm_prefill_m2048.md")


# ----------------------------------------------------------------------------
# work accounting (per launch)
# ----------------------------------------------------------------------------
def algo_bytes(M: int, N: int, K: int, zp: bool = True) -> int:
    """Bytes a W4A16 product must move at least once: packed codes, scales,
    zero points (asymmetric), x and y."""
    G = K // 128
    return N * K // 2 + 2 * N * G + (2 * N * G if zp else 0) + 2 * M * K + 2 * M * N


def algo_flops(M: int, N: int, K: int) -> int:
    return 2 * M * N * K


# ----------------------------------------------------------------------------
# distributed plumbing (replicas only: the layer is independent per GPU)
# ----------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend: str):
    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    return dist if ws > 1 else None


def reduce_max(value: float, dist, device=None) -> float:
    """Max of a scalar over ranks (identity without a process group)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, dist, device=None) -> float:
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(units_local: float, seconds_local: float, dist, device=None):
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time. Returns (total_units, max_seconds)."""
    return reduce_sum(units_local, dist, device), reduce_max(seconds_local, dist, device)


# ----------------------------------------------------------------------------
# peaks, profiles, clocks
# ----------------------------------------------------------------------------
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, TENSOR_FALLBACK_TFLOPS, 0.0, "fallback"


COMMON_SRC = os.path.join(ROOT, "weight_only_int4_gemv_b200", "csrc", "awq_common.cuh")


def source_sha(path: str) -> str:
    """First 16 hex digits of the SHA-256 of a kernel's .cu file followed by
    the kernel body it includes (awq_gemm_body.cuh, for the GEMM) and the
    device helpers, so a profile goes stale when any of them changes."""
    h = hashlib.sha256()
    body = os.path.join(os.path.dirname(path), "awq_gemm_body.cuh")
    parts = (path, body, COMMON_SRC) if path.endswith("awq_gemm.cu") else (path, COMMON_SRC)
    for p in parts:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profile_traffic(profile_path: str, source_path: str):
    """Per-launch DRAM bytes from a committed ncu summary, or None when the
    summary is missing or the kernel source changed since it was taken."""
    try:
        text = open(profile_path).read()
    except OSError:
        return None
    m = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", text)
    t = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m or not t or m.group(1) != source_sha(source_path):
        return None
    return float(t.group(1))


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML while running."""

    REASONS = {
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, const in self.REASONS.items():
                    if r & getattr(nv, const, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# the CPU oracle on a bounded sample (baseline / reference arm)
# ----------------------------------------------------------------------------
def oracle_sample(shapes, M: int, rows: int, zp: bool = True, seed: int = 0):
    """Per shape: a sample of `rows` output channels quantized by the oracle,
    plus x. Returns [(x, qweight, scales, zeros, bytes)]."""
    from oracle import awq_oracle as O
    out = []
    rng = np.random.default_rng(seed)
    for sh in shapes:
        W = make_weight(rows, sh.K, 0.02, 0.01, seed=seed)
        qweight, scales, zeros = O.quantize_pack(W, 128, zp)
        x = rng.standard_normal((M, sh.K), dtype=np.float32).astype(np.float16)
        out.append((x, qweight, scales, zeros, algo_bytes(M, rows, sh.K, zp)))
    return out


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(sample, budget_s: float):
    """Run the oracle's layer (unpack, dequant, float64 matmul) over the sample
    until `budget_s` has passed; returns (bytes, seconds, passes)."""
    from oracle import awq_oracle as O
    done_bytes, passes = 0, 0
    t0 = time.perf_counter()
    while True:
        for x, q, s, z, b in sample:
            O.linear(x, q, s, z, 128)
            done_bytes += b
        passes += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return done_bytes, time.perf_counter() - t0, passes


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(shapes, M: int, budget_s: float = 10.0, rows: int = 1024):
    """The oracle on the host cores: all BLAS threads (the reported value),
    then BLAS pinned to one thread for a third of the budget."""
    sample = oracle_sample(shapes, M, rows)
    b, s, passes = time_oracle(sample, budget_s)
    single = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1, user_api="blas"):
            b1, s1, p1 = time_oracle(sample, budget_s / 3)
        single = {"value": round(b1 / s1 / 1e9, 4), "unit": "GB/s", "cores": 1, "passes": p1}
    except ImportError:
        pass
    return {"value": round(b / s / 1e9, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows} output channels of each of {len(shapes)} layer shapes, M={M}, "
                      f"{passes} passes in {s:.1f} s (numpy unpack/dequant single-threaded, "
                      f"float64 matmul on {blas_threads()} BLAS threads, {os.cpu_count()} host cores)",
            "single_thread": single, "cpu_model": cpu_model()}


# ----------------------------------------------------------------------------
# native arm
# ----------------------------------------------------------------------------
def chain_sources(shapes):
    """Per layer of a decode step, the earlier layer whose output is its input
    (-1: the step's input): the most recent earlier layer with as many output
    channels as this layer has input channels. For the Llama-3-8B layer:
    q_proj on the step's input, gate_proj and up_proj on q_proj's output,
    down_proj on up_proj's output."""
    src = []
    for i, sh in enumerate(shapes):
        j = next((j for j in range(i - 1, -1, -1) if shapes[j].N == sh.K), -1)
        src.append(j)
    return src


class DecodeModel:
    """n layer copies of the decode layer: packed weights of each shape and
    one output buffer per projection. Step s runs copy s % n; its first
    projection reads the last projection's output of the step before (copy
    (s - 1) % n), as a decode pass feeds each layer the previous one's
    output. Launches carry up to `per_launch` consecutive steps."""

    def __init__(self, awq, torch, packed, ys, shapes, M, per_launch):
        self.awq, self.torch = awq, torch
        self.packed, self.ys, self.shapes, self.M = packed, ys, shapes, M
        self.n = len(packed)
        self.per_launch = per_launch
        self.src = chain_sources(shapes)
        self._chains = {}

    def step_input(self, c):
        return self.ys[(c - 1) % self.n][-1]

    def chain(self, start, count):
        """The prepared awq_gemv_chain call of steps start .. start + count - 1."""
        key = (start % self.n, count)
        ch = self._chains.get(key)
        if ch is None:
            nl = len(self.shapes)
            specs = []
            for j in range(count):
                c = (start + j) % self.n
                for i, (q, s, z) in enumerate(self.packed[c]):
                    if i == 0:
                        xs = dict(x=self.step_input(c)) if j == 0 else dict(x_from=nl * (j - 1) + nl - 1)
                    else:
                        xs = dict(x_from=nl * j + self.src[i])
                    specs.append(dict(xs, qweight=q, scales=s, zeros=z, out=self.ys[c][i]))
            ch = self._chains[key] = self.awq.GemvChain(self.M, specs, weights_static=True)
        return ch

    def launches(self, first, count):
        """(start, count) of the launches that run steps first .. first + count - 1."""
        out, s = [], first
        while s < first + count:
            k = min(self.per_launch, first + count - s)
            out.append((s, k))
            s += k
        return out

    def run_steps_chain(self, first, count):
        for s, k in self.launches(first, count):
            self.chain(s, k)()

    def run_steps_per_gemv(self, first, count, workspaces):
        awq = self.awq
        for s in range(first, first + count):
            c = s % self.n
            for i, (q, sc, z) in enumerate(self.packed[c]):
                x = self.step_input(c) if i == 0 else self.ys[c][self.src[i]]
                awq.awq_gemv(x, q, sc, z, workspace=workspaces[i], out=self.ys[c][i], weights_static=True)


def build_decode(awq, torch, device, shapes, M: int, n_layers: int, zp: bool):
    """Quantize each shape on the GPU (recipe W, seed 0; the second, warm call
    is timed), then clone the packed tensors into n_layers copies at distinct
    addresses, each with its own output buffers (seeded N(0,1) values, so the
    first steps read finite inputs)."""
    base, quant_ms, quant_bytes = [], 0.0, 0
    for sh in shapes:
        W = torch.from_numpy(make_weight(sh.N, sh.K, 0.02, 0.01, seed=0)).to(device)
        # one untimed call first: the first call of a shape pays the output
        # allocations and module loading, not the quantizer
        awq.awq_pseudo_quantize_pack(W, zero_point=zp)
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        q, s, z = awq.awq_pseudo_quantize_pack(W, zero_point=zp)
        e1.record()
        torch.cuda.synchronize(device)
        quant_ms += e0.elapsed_time(e1)
        quant_bytes += 2 * sh.N * sh.K + algo_bytes(0, sh.N, sh.K, zp)
        base.append((q, s, z))
        del W
    if shapes[-1].N != shapes[0].K:
        raise SystemExit("a decode step's last projection must feed its first")
    rng = np.random.default_rng(1)
    packed, ys = [], []
    for _ in range(n_layers):
        packed.append([(q.clone(), s.clone(), z.clone() if z is not None else None) for q, s, z in base])
        ys.append([torch.from_numpy(rng.standard_normal((M, sh.N), dtype=np.float32).astype(np.float16)).to(device)
                   for sh in shapes])
    per_launch = max(1, awq.CHAIN_MAX_LAYERS // len(shapes))
    model = DecodeModel(awq, torch, packed, ys, shapes, M, per_launch)
    return model, {"ms": round(quant_ms, 4), "GB/s": round(quant_bytes / (quant_ms * 1e-3) / 1e9, 1)}


def run_native(args, dist):
    import torch
    import weight_only_int4_gemv_b200 as awq

    ws_, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    awq.lib()
    hbm_peak, tc_peak, tc_sust, peak_src = measured_peaks()
    wl = WORKLOADS[args.workload]
    zp = True
    if args.workload == "llama3_8b_decode":
        shapes, M = LLAMA3_8B_DECODE, 1
    else:
        shapes, M = wl.shapes, min(wl.Ms)
    if M > awq.GEMV_MAX_M:
        raise SystemExit("the decode bench runs the GEMV path; use --workload llama3_8b_decode or decode_sweep")

    model, quant = build_decode(awq, torch, device, shapes, M, args.layers, zp)
    step_bytes = sum(algo_bytes(M, sh.N, sh.K, zp) for sh in shapes)
    step_flops = sum(algo_flops(M, sh.N, sh.K) for sh in shapes)
    stream = torch.cuda.Stream(device)
    wss = [awq.alloc_workspace(M, sh.N, sh.K, zp, device=device) for sh in shapes]

    def run_steps(first, count):
        if args.per_gemv:
            model.run_steps_per_gemv(first, count, wss)
        else:
            model.run_steps_chain(first, count)

    def n_launches(first, count):
        return count * len(shapes) if args.per_gemv else len(model.launches(first, count))

    # The warm-up steps and the timed steps are each replayed from one CUDA
    # graph holding exactly those steps, so consecutive launches stay linked
    # by programmatic dependent launch whatever the number of steps (only the
    # first launch of the timed graph cannot overlap the launch before it).
    def capture(first, count):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run_steps(first, count)
        return g

    with torch.cuda.stream(stream):
        run_steps(0, args.warmup + args.steps)   # prepares every chain and plan outside capture
    torch.cuda.synchronize(device)
    g_warm = capture(0, args.warmup)
    g_timed = capture(args.warmup, args.steps)
    with torch.cuda.stream(stream):
        g_timed.replay()                           # untimed: first replay of the instantiated graph
    torch.cuda.synchronize(device)

    def barrier():
        if dist is not None:
            dist.barrier()

    with torch.cuda.stream(stream):
        g_warm.replay()
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier()
    torch.cuda.synchronize(device)
    with sampler:
        with torch.cuda.stream(stream):
            t0.record()
            g_timed.replay()
            t1.record()
        torch.cuda.synchronize(device)
    barrier()
    elapsed_s = t0.elapsed_time(t1) * 1e-3
    dev_err = awq.awq_device_error(device)
    del g_warm, g_timed

    # Every launch in the timed region is one of this library's products and
    # consecutive launches overlap (programmatic dependent launch), so the
    # kernel's average launch duration is the timed region over its launches.
    n_launch = n_launches(args.warmup, args.steps)
    mean_launch_s = elapsed_s / n_launch
    kernel_gbs = step_bytes * args.steps / elapsed_s / 1e9

    total_bytes, max_s = aggregate(step_bytes * args.steps, elapsed_s, dist, device)
    value = total_bytes / max_s / 1e9

    # end to end through the public API: pinned host x in, pinned host y out, every step
    e2e = run_e2e(awq, torch, device, stream, model, shapes, M, args, dist, step_bytes)

    gemm = None
    search = None
    if ws_ == 1 and not args.no_gemm:
        gemm = run_gemm_prefill(awq, torch, device, tc_peak, peak_src, args)
        search = run_scale_search(awq, torch, device)

    cpu = None
    if ws_ == 1 and rank == 0 and not args.no_cpu:
        cpu = cpu_baseline(shapes, M, budget_s=args.cpu_seconds)

    if rank == 0:
        src_file = "awq_gemv.cu" if args.per_gemv else "awq_gemv_chain.cu"
        kern_src = os.path.join(ROOT, "weight_only_int4_gemv_b200", "csrc", src_file)
        traffic = profile_traffic(GEMV_PROFILE if args.per_gemv else CHAIN_PROFILE, kern_src)
        deps = chain_sources(shapes)
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": ws_,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(max_s * 1e3 / args.steps, 6),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f16",
            "data": "synthetic (seeded N(0,0.02) weights, 1% salient input channels x10, N(0,1) x; no checkpoint)",
            "config": {
                "workload": f"{args.workload}_m{M}",
                "layers": [f"{sh.name} {sh.N}x{sh.K}" + (f" (x = {shapes[d].name} output)" if d >= 0 else " (x = step input)")
                           for sh, d in zip(shapes, deps)],
                "M": M, "group_size": 128, "zero_point": zp,
                "weights_static": "AWQ_FLAG_WEIGHTS_STATIC set: weights are loaded once, so a launch may "
                                  "start streaming them before the previous kernel on the stream finishes",
                "step": "one layer: the listed projections, each reading its input only after the projection "
                        "it comes from is complete; a step's first projection reads the previous step's last "
                        "output",
                "launch": ("one awq_gemv launch per projection" if args.per_gemv else
                           f"one awq_gemv_chain launch per {model.per_launch} consecutive steps "
                           f"({model.per_launch * len(shapes)} projections; a shorter last launch when the step "
                           "count is not a multiple)"),
                "graphs": "the warm-up steps and the timed steps are each replayed from one CUDA graph "
                          "holding exactly those steps (the timed graph is replayed once untimed first)",
                "l2": f"inputs larger than L2: steps rotate over {args.layers} layer copies "
                      f"({args.layers * step_bytes / 1e9:.2f} GB of packed weights)",
                "parallelism": f"replicas x{ws_}",
            },
            "tflops": round(reduce_sum(step_flops * args.steps, dist, device) / max_s / 1e12, 4),
            "roofline": {
                "bound": "hbm", "achieved": round(kernel_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(kernel_gbs / hbm_peak, 4),
                "traffic": traffic, "peak_source": peak_src,
                "kernel": ("awq_gemv (gemv_kernel, M tile 1, asymmetric)" if args.per_gemv else
                           "awq_gemv_chain (chain_kernel<1, 1>: M = 1, fp16 zero points)"),
                "launches_timed": n_launch,
                "algorithmic_bytes_per_launch": round(step_bytes * args.steps / n_launch),
                "mean_launch_us": round(1e6 * mean_launch_s, 3),
                "duration_source": "CUDA events around the timed steps on the launch stream / launches",
                "frac_of_nominal_8TBs": round(kernel_gbs / 8000.0, 4),
            },
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": n_launch,
            "clocks": sampler.summary(),
            "device_error": dev_err,
            "quantize": quant,
        }
        if gemm is not None:
            line["prefill_gemm"] = gemm
        if search is not None:
            line["scale_search"] = search
        print(json.dumps(line), flush=True)


def run_e2e(awq, torch, device, stream, model, shapes, M, args, dist, step_bytes):
    """Same metric through the Python API with host buffers: every step copies
    its input x from pinned host memory to the device, runs the layer (one
    prepared chain call of that step), reads the layer's result (the last
    projection's output) back into pinned host memory, then synchronizes.
    By default the three operations of a step are replayed from one CUDA
    graph per layer copy (as a serving loop would run them); --e2e-eager
    issues them one by one."""
    steps = max(1, min(args.steps, args.e2e_steps))
    hx = torch.empty_like(model.step_input(0), device="cpu").pin_memory()
    hy = torch.empty_like(model.ys[0][-1], device="cpu").pin_memory()
    hx.copy_(model.step_input(0).cpu())
    h2d = hx.numel() * 2
    d2h = hy.numel() * 2
    wss = [awq.alloc_workspace(M, sh.N, sh.K, True, device=device) for sh in shapes]

    def step(s):
        c = s % model.n
        model.step_input(c).copy_(hx, non_blocking=True)
        if args.per_gemv:
            model.run_steps_per_gemv(s, 1, wss)
        else:
            model.chain(s, 1)()
        hy.copy_(model.ys[c][-1], non_blocking=True)
        torch.cuda.current_stream(device).synchronize()

    graphs = []
    with torch.cuda.stream(stream):
        for s in range(max(min(args.warmup, 20), model.n)):   # every layer copy's chain is prepared
            step(s)
        if not args.e2e_eager and not args.per_gemv:
            for c in range(model.n):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    model.step_input(c).copy_(hx, non_blocking=True)
                    model.chain(c, 1)()
                    hy.copy_(model.ys[c][-1], non_blocking=True)
                graphs.append(g)

            def step(s):   # noqa: F811 (the graph form of the same step)
                graphs[s % model.n].replay()
                torch.cuda.current_stream(device).synchronize()

            for s in range(model.n):
                step(s)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(device)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for s in range(steps):
            step(s)
        t1.record()
        torch.cuda.synchronize(device)
    sec = t0.elapsed_time(t1) * 1e-3
    total, max_s = aggregate(step_bytes * steps, sec, dist, device)
    return {"value": round(total / max_s / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "note": "effective HBM GB/s of the same algorithmic bytes, time includes the copies and a "
                    "host synchronize per step (one launch per step" +
                    (", issued one by one)" if args.e2e_eager or args.per_gemv else
                     "; copy in, launch and copy out replayed from one CUDA graph per step)")}


def run_scale_search(awq, torch, device):
    """awq_search_scale on gate_proj 14336x4096 with 512 calibration tokens
    (the pages' max_calib_seq_len) of synthetic activations whose 1 % salient
    channels are 10x larger, a 20-point grid: one warm call, device time."""
    N, K, Ms, n_grid = 14336, 4096, 512, 20
    W = torch.from_numpy(make_weight(N, K, 0.02, 0.0, seed=0)).to(device)
    rng = np.random.default_rng(2)
    X = rng.standard_normal((Ms, K), dtype=np.float32)
    X[:, rng.choice(K, K // 100, replace=False)] *= 10.0
    X = torch.from_numpy(X.astype(np.float16)).to(device)
    awq.awq_search_scale(W, X, n_grid=n_grid)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    _, losses = awq.awq_search_scale(W, X, n_grid=n_grid)
    e1.record()
    torch.cuda.synchronize(device)
    losses = losses.cpu().numpy().astype(np.float64)
    best = int(np.argmin(losses))
    return {"workload": "gate_proj 14336x4096, 512 calibration tokens, 20 grid points", "ms": round(e0.elapsed_time(e1), 3),
            "best_alpha": best / n_grid, "loss_best_over_alpha0": round(float(losses[best] / losses[0]), 4)}


def run_gemm_prefill(awq, torch, device, tc_peak, peak_src, args):
    """awq_gemm at M = 2048 on gate_proj 14336x4096 (the prefill shape), four
    weight/activation copies in rotation (180 MB > L2), events per launch."""
    M, N, K = 2048, 14336, 4096
    W = torch.from_numpy(make_weight(N, K, 0.02, 0.0, seed=0)).to(device)
    q, s, z = awq.awq_pseudo_quantize_pack(W, zero_point=True)
    del W
    rng = np.random.default_rng(2)
    copies = []
    for _ in range(4):
        x = torch.from_numpy(rng.standard_normal((M, K), dtype=np.float32).astype(np.float16)).to(device)
        copies.append((x, q.clone(), s.clone(), z.clone(), torch.empty((M, N), dtype=torch.float16, device=device)))
    reps = max(8, min(args.gemm_steps, 400))
    for i in range(4):
        x, qq, ss, zz, y = copies[i]
        awq.awq_gemm(x, qq, ss, zz, out=y)
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    sampler = ClockSampler(device.index if device.index is not None else 0)
    with sampler:
        for r in range(reps):
            x, qq, ss, zz, y = copies[r % 4]
            evs[r][0].record()
            awq.awq_gemm(x, qq, ss, zz, out=y)
            evs[r][1].record()
        torch.cuda.synchronize(device)
    ms = [a.elapsed_time(b) for a, b in evs]
    mean_ms = sum(ms) / len(ms)
    tflops = algo_flops(M, N, K) / (mean_ms * 1e-3) / 1e12
    err = awq.awq_device_error(device)
    gemm_src = os.path.join(ROOT, "weight_only_int4_gemv_b200", "csrc", "awq_gemm.cu")
    return {"workload": f"prefill_m{M} gate_proj {N}x{K}", "launches": reps,
            "mean_launch_us": round(mean_ms * 1e3, 2), "min_launch_us": round(min(ms) * 1e3, 2),
            "tflops": round(tflops, 1),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": tc_peak, "unit": "TFLOP/s",
                         "frac": round(tflops / tc_peak, 4), "peak_source": f"{peak_src} (bf16 burst; fp16 same rate)",
                         "traffic": profile_traffic(GEMM_PROFILE, gemm_src)},
            "clocks": sampler.summary(), "device_error": err}


# ----------------------------------------------------------------------------
# reference arm: the CPU oracle
# ----------------------------------------------------------------------------
def run_reference(args, dist):
    ws_, rank, _ = dist_env()
    if rank != 0:
        return
    if args.workload == "llama3_8b_decode":
        shapes, M = LLAMA3_8B_DECODE, 1
    else:
        wl = WORKLOADS[args.workload]
        shapes, M = wl.shapes, min(wl.Ms)
    rows = args.ref_rows
    sample = oracle_sample(shapes, M, rows)
    for _ in range(args.warmup):
        time_oracle(sample, 0.0)
    b, s, passes = 0, 0.0, 0
    for _ in range(args.steps):
        bb, ss, _p = time_oracle(sample, 0.0)
        b += bb
        s += ss
        passes += 1
    value = b / s / 1e9
    desc = (f"each step: the oracle layer on {rows} output channels of each of {len(shapes)} shapes "
            f"({', '.join(f'{sh.name} {sh.N}x{sh.K}' for sh in shapes)}), M={M}")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": ws_,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(s * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": f"{args.workload}_m{M}", "sample": desc},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "kind": "oracle", "cores": blas_threads(),
                         "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_table(args):
    """Per (shape, M) device time of awq_gemv and awq_gemm: one JSON line per
    measurement. Weights come from make_packed_random (every code value in
    every slot, which the kernels' time does not depend on); each shape gets
    enough weight copies that one round of launches exceeds L2, and the
    launches of a round are replayed back to back from a CUDA graph, as a
    decode loop runs them (cold: `us`). For the GEMV rows of layers up to
    half of L2, `hot_us` repeats the round on the first copy only, whose
    weights then stay in L2."""
    import torch
    import weight_only_int4_gemv_b200 as awq
    from workloads import make_packed_random

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    hbm_peak, tc_peak, _, peak_src = measured_peaks()
    # (N, K), batch sizes, fused gate/up (AWQ_FLAG_SILU_MUL: N = gate + up rows, y has N / 2 columns),
    # packed zero points (AWQ_FLAG_PACKED_ZEROS, GEMV only), zero points (False: symmetric)
    mid = (16, 24, 32, 48, 64, 96, 128)   # around the GEMV / GEMM crossover
    cases = [((4096, 4096), (1, 2, 4, 8, 16, 128, 512, 2048), False, False, True),
             ((14336, 4096), (1, 2, 4, 8, 16, 128, 512, 2048), False, False, True),
             ((4096, 4096), mid[1:], False, False, True), ((14336, 4096), mid[1:], False, False, True),
             ((28672, 4096), (1, 4, 16, 128, 2048), True, False, True),
             ((6144, 4096), (1, 4, 16), False, False, True),     # q, k, v of Llama-3-8B concatenated
             ((1024, 4096), (1, 4, 16), False, False, True),     # k or v alone
             ((4096, 14336), (1, 2, 4, 8, 16), False, False, True),
             ((14336, 4096), (1, 2, 4, 8, 16), False, False, False),   # symmetric
             ((4096, 14336), (1, 2, 4, 8, 16), False, False, False),
             ((8192, 8192), (1, 8, 2048), False, False, True), ((28672, 8192), (1, 8, 2048), False, False, True),
             ((8192, 28672), (1, 8, 2048), False, False, True),
             ((4096, 4096), (1, 4, 16), False, True, True), ((14336, 4096), (1, 4, 16), False, True, True),
             ((4096, 14336), (1, 4, 16), False, True, True), ((28672, 4096), (1, 4, 16), True, True, True)]
    only = os.environ.get("AWQ_TABLE_CASES")   # optional comma-separated case indices
    if only:
        cases = [cases[int(i)] for i in only.split(",")]
    l2_bytes = 126 << 20
    rng = np.random.default_rng(3)
    for (N, K), Ms, silu, packed, zp in cases:
        q, s, z = [torch.from_numpy(a).to(device) if a is not None else None
                   for a in make_packed_random(N, K, 128, zp, seed=1)]
        if packed:
            z = awq.awq_pack_zeros(z)
        wbytes = N * K // 2 + (4 if zp else 2) * N * (K // 128)
        copies = max(2, -(-2 * l2_bytes // wbytes))
        packs = [(q.clone(), s.clone(), z.clone() if z is not None else None) for _ in range(copies)]
        del q, s, z
        for M in Ms:
            x = torch.from_numpy(rng.standard_normal((M, K), dtype=np.float32).astype(np.float16)).to(device)
            y = torch.empty((M, N // 2 if silu else N), dtype=torch.float16, device=device)
            entry = (("awq_gemv" if M <= awq.GEMV_MAX_M else "awq_gemm") + (" silu_mul" if silu else "") +
                     (" packed_zeros" if packed else "") + ("" if zp else " symmetric"))
            fn = awq.awq_gemv if M <= awq.GEMV_MAX_M else awq.awq_gemm
            kw = {"weights_static": True} if M <= awq.GEMV_MAX_M else {}
            if silu:
                kw["silu_mul"] = True
            ws = awq.alloc_workspace(M, N, K, zp, device=device, silu_mul=silu, packed_zeros=packed)
            stream = torch.cuda.Stream(device)
            with torch.cuda.stream(stream):
                for qq, ss, zz in packs:
                    fn(x, qq, ss, zz, workspace=ws, out=y, **kw)
                torch.cuda.synchronize(device)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for qq, ss, zz in packs:
                        fn(x, qq, ss, zz, workspace=ws, out=y, **kw)
                reps = max(3, min(200, int(2e6 / (copies * max(1.0, M / 8)))))
                for _ in range(3):
                    g.replay()
                torch.cuda.synchronize(device)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(reps):
                    g.replay()
                e1.record()
                torch.cuda.synchronize(device)
                cold_ms = e0.elapsed_time(e1)
                hot_us = None
                if M <= awq.GEMV_MAX_M and wbytes <= l2_bytes // 2:
                    # hot: the same number of launches, all on the first copy,
                    # whose weights then stay in L2 between launches
                    gh = torch.cuda.CUDAGraph()
                    qq, ss, zz = packs[0]
                    with torch.cuda.graph(gh, stream=stream):
                        for _ in packs:
                            fn(x, qq, ss, zz, workspace=ws, out=y, **kw)
                    for _ in range(3):
                        gh.replay()
                    torch.cuda.synchronize(device)
                    e0.record()
                    for _ in range(reps):
                        gh.replay()
                    e1.record()
                    torch.cuda.synchronize(device)
                    hot_us = e0.elapsed_time(e1) * 1e3 / (reps * copies)
                    del gh
            us = cold_ms * 1e3 / (reps * copies)
            # y: N/2 columns with silu_mul; packed zero points: 4 bits instead of 16 per (row, group)
            nbytes = algo_bytes(M, N, K, zp) - (M * N if silu else 0) - (3 * N * (K // 128) // 2 if packed else 0)
            gbs = nbytes / (us * 1e-6) / 1e9
            tfl = algo_flops(M, N, K) / (us * 1e-6) / 1e12
            print(json.dumps({"entry": entry, "N": N, "K": K, "M": M, "us": round(us, 3), "GB/s": round(gbs, 1),
                              "frac_hbm": round(gbs / hbm_peak, 4), "TFLOP/s": round(tfl, 2),
                              "frac_tensor": round(tfl / tc_peak, 4), "peaks": peak_src,
                              "weight_copies": copies,
                              "hot_us": None if hot_us is None else round(hot_us, 3),
                              "hot_GB/s": None if hot_us is None else round(nbytes / (hot_us * 1e-6) / 1e9, 1)}),
                  flush=True)
            del g
        del packs
        torch.cuda.empty_cache()
    if not only:
        run_table_chain(awq, torch, device, hbm_peak, peak_src)


def run_table_chain(awq, torch, device, hbm_peak, peak_src):
    """The Llama-3-8B decode step (the bench's data flow: gate/up on q's
    output, down on up's, the next q on down's) through awq_gemv_chain at
    M = 1 .. 16, asymmetric and symmetric: 8 steps per launch over 8 layer
    copies (0.8 GB of packed weights), 64 steps replayed from one CUDA graph.
    One JSON line per (M, variant) with the time per step."""
    from workloads import make_packed_random
    shapes = LLAMA3_8B_DECODE
    stream = torch.cuda.Stream(device)
    for zp in (True, False):
        base = [[torch.from_numpy(a).to(device) if a is not None else None
                 for a in make_packed_random(sh.N, sh.K, 128, zp, seed=1)] for sh in shapes]
        n = 8
        packed = [[tuple(t.clone() if t is not None else None for t in b) for b in base] for _ in range(n)]
        for M in (1, 2, 4, 8, 16):
            rng = np.random.default_rng(M)
            ys = [[torch.from_numpy(rng.standard_normal((M, sh.N), dtype=np.float32).astype(np.float16) * 0.01)
                   .to(device) for sh in shapes] for _ in range(n)]
            model = DecodeModel(awq, torch, packed, ys, shapes, M, awq.CHAIN_MAX_LAYERS // len(shapes))
            steps = 64
            with torch.cuda.stream(stream):
                model.run_steps_chain(0, steps)
            torch.cuda.synchronize(device)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                model.run_steps_chain(0, steps)
            ts = []
            for _ in range(4):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                with torch.cuda.stream(stream):
                    g.replay()
                e1.record(stream)
                torch.cuda.synchronize(device)
                ts.append(e0.elapsed_time(e1) * 1e3 / steps)
            us = float(np.median(ts[1:]))
            nbytes = sum(algo_bytes(M, sh.N, sh.K, zp) for sh in shapes)
            gbs = nbytes / (us * 1e-6) / 1e9
            print(json.dumps({"entry": "awq_gemv_chain llama3_8b step" + ("" if zp else " symmetric"), "M": M,
                              "us_per_step": round(us, 3), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm_peak, 4),
                              "peaks": peak_src, "device_error": awq.awq_device_error()}), flush=True)
            del g, model
        del packed, base
        torch.cuda.empty_cache()


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=64)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=["llama3_8b_decode", "decode_sweep"], default="llama3_8b_decode")
    ap.add_argument("--layers", type=int, default=32, help="layer copies the steps rotate over")
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--e2e-eager", action="store_true",
                    help="e2e: issue each step's copies and launch one by one instead of replaying a graph")
    ap.add_argument("--gemm-steps", type=int, default=100)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-rows", type=int, default=256)
    ap.add_argument("--no-gemm", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--per-gemv", action="store_true",
                    help="run each projection as its own awq_gemv launch instead of one awq_gemv_chain per step")
    ap.add_argument("--table", action="store_true",
                    help="instead of the bench line: per (shape, M) GEMV / GEMM times, one JSON line each")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.steps < 1:
        ap.error("--steps must be >= 1")
    return a


def main(argv=None):
    args = parse_args(argv)
    ws_, _, _ = dist_env()
    if args.impl == "reference":
        run_reference(args, None)
        return 0
    if args.table:
        run_table(args)
        return 0
    dist = init_dist("nccl")
    try:
        run_native(args, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
