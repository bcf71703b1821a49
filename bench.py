"""Benchmark of the sign-weight linear layers on B200 (one JSON line on rank 0).

Workload (default): OneBit decode GEMV -- X M x 4096 bf16 ~N(0,1) for M in
{1, 4, 16}, W 4096 x 4096 ~N(0, 0.02) packed to 2 MiB of signs, a, b fp32 from
SVID.  One step = one decode token through a pool of L distinct 4096 x 4096
OneBit layers at each batch size (for M in {1,4,16}: for each layer: ob_linear),
so every call reads its weights from HBM: the pool (L x 2.1 MB) is larger than
three times the L2 cache.  Each batch size's pass is captured once as a CUDA
graph (a decode step runs all layers at one M) and the three are replayed per
step; inputs are resident in HBM when the timed region starts.

  value     HBM GB/s of the step: algorithmic bytes (packed signs + a + b + X + Y
            per call) / device time, summed over ranks, time = max over ranks.
  roofline  the decode kernel: algorithmic bytes per launch / average launch
            time, against the measured HBM copy bandwidth.
  e2e       the same metric through the C-ABI with host buffers: pinned X is
            copied to the device and Y back inside the timed region.
  extra     prefill (M=2048, 4096 -> 11008, tensor-core TFLOP/s) and DBF
            (K=N=4096, r=2048, M in {1, 512}) measured in the same run.

``--impl reference`` times the fp64 CPU oracle (the reference arm of this
build) on a bounded sample of the same workload and metric.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ob_linear/dbf_linear TFLOP/s-equiv & weight GB/s at M=1/16/2048, % of roofline"
N_DIM = K_DIM = 4096
DECODE_MS = (1, 4, 16)
LAYERS = 192          # 192 x 2.13 MB = 409 MB of weights per pass > 3 x 126 MB L2
SEED = 1


def decode_call_bytes(M: int, N: int = N_DIM, K: int = K_DIM) -> int:
    """Algorithmic HBM bytes of one OneBit call: packed signs, a, b, X (bf16), Y (bf16)."""
    return N * K // 8 + 4 * N + 4 * K + 2 * M * K + 2 * M * N


def step_bytes(layers: int) -> int:
    return layers * sum(decode_call_bytes(m) for m in DECODE_MS)


def step_flops(layers: int) -> int:
    return layers * sum(2 * m * N_DIM * K_DIM for m in DECODE_MS)


# ------------------------------------------------------------------ distributed plumbing

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        import torch
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, interval_ms: int = 50):
        self.dev = device_index
        self.interval = interval_ms
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", str(self.interval)], stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self) -> dict:
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.file.flush()
        with open(self.file.name) as f:
            rows = [r.split(",") for r in f.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ helpers

def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def prefill_kernel_name() -> str:
    """The tcgen05 GEMM AUTO runs on the prefill workload (bf16 Y, M >= 512): the CTA-pair kernel."""
    return "sign_gemm_tc2_kernel"


def prefill_kernel_source():
    return ("linear_tc2.cu",)


def ncu_traffic(kernel_file: str, key: str):
    """DRAM bytes per launch from a committed ncu summary, or None if the kernel changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    import hashlib
    with open(path) as f:
        table = json.load(f)
    entry = table.get(key)
    if not entry:
        return None
    with open(os.path.join(ROOT, "binary_weight_gemm_b200", "csrc", kernel_file), "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()[:16]
    return entry["bytes_per_launch"] if entry.get("source_sha") == digest else None


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ reference arm (the oracle on the host)

def oracle_step_sample(budget_s: float, steps: int | None = None, warmup: int = 0):
    """Time the oracle's direct form on one 4096 x 4096 layer at M = 1, 4, 16 (one layer per step)."""
    import oracle
    from binary_weight_gemm_b200 import synth
    W = synth.weights(SEED, N_DIM, K_DIM)
    # The oracle's SVID (full SVD) is the conversion step; it is timed once, outside the linear sample.
    t0 = time.perf_counter()
    a, b, _ = oracle.svid_rank1(W)
    svd_s = time.perf_counter() - t0
    a, b = a.astype(np.float32), b.astype(np.float32)
    S = oracle.sign_pm1(W)
    xs = {m: synth.activations(SEED, m, K_DIM)[1] for m in DECODE_MS}

    def one():
        for m in DECODE_MS:
            oracle.onebit_linear(xs[m], S, a, b)

    for _ in range(warmup):
        one()
    n, t0 = 0, time.perf_counter()
    while True:
        one()
        n += 1
        el = time.perf_counter() - t0
        if (steps is not None and n >= steps) or (steps is None and el >= budget_s):
            break
    return n, el, svd_s


def run_reference(args, world, rank):
    if rank != 0:
        return
    steps = max(1, args.steps)
    n, el, svd_s = oracle_step_sample(0.0, steps=steps, warmup=args.warmup)
    bytes_per = step_bytes(1)
    value = bytes_per * n / el / 1e9
    cores = cpu_cores()
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
        "steps": n, "warmup": args.warmup, "ms_per_step": 1e3 * el / n, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "onebit_decode_4096x4096_M1_4_16", "layers_per_step": 1,
                   "M": list(DECODE_MS), "N": N_DIM, "K": K_DIM, "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n} steps x (M=1,4,16) on one 4096x4096 layer, direct form "
                                   f"(W_hat materialised each call); SVID full SVD once: {svd_s:.1f} s"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def run_ours(args, world, rank, local):
    import torch
    from binary_weight_gemm_b200 import build, synth
    build.build()
    from binary_weight_gemm_b200 import ops

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    peaks = load_peaks()
    L = args.layers

    # Weights: one seeded 4096 x 4096 matrix, converted by the library (pack + SVID, timed once).
    W = torch.from_numpy(synth.weights(SEED, N_DIM, K_DIM)).to(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ops.ob_pack_signs(W, stream=stream)  # first launch loads the module; not timed
        stream.synchronize()
        ev0.record(stream)
        P0 = ops.ob_pack_signs(W, stream=stream)
        ev1.record(stream)
        stream.synchronize()
        pack_ms = ev0.elapsed_time(ev1)
        t0 = time.perf_counter()
        a0, b0, _, svid_iters, _ = ops.ob_svid_rank1(W, stream=stream)
        svid_ms = 1e3 * (time.perf_counter() - t0)
    del W
    # Pool of L distinct weight buffers (same values, different addresses) so each call misses L2.
    pool = [(P0.clone(), a0.clone(), b0.clone()) for _ in range(L)]
    xs = {m: torch.from_numpy(synth.activations(SEED, m, K_DIM)[0].view(np.int16)).to(dev).view(torch.bfloat16)
          for m in DECODE_MS}
    ys = {m: torch.empty((m, N_DIM), dtype=torch.bfloat16, device=dev) for m in DECODE_MS}
    torch.cuda.synchronize()

    # The weights are loaded once and reused by every step, so the calls say so
    # (OB_FLAG_STATIC_WEIGHTS: the one-token kernel then reads its sign words before the
    # previous call has finished); the plain AUTO call is timed beside it.
    decode_path = ops.OB_PATH_AUTO | ops.OB_FLAG_STATIC_WEIGHTS

    def step(s, ms=DECODE_MS):
        for m in ms:
            for (P, a, b) in pool:
                ops.ob_linear(xs[m], P, a, b, out=ys[m], stream=s, path=decode_path)

    # One CUDA graph per M (calls are stream-ordered; no allocation inside): a decode
    # step applies every layer at one batch size, and graphs that mix the kernels of
    # different M lose the programmatic-launch overlap (their shared-memory footprints
    # differ), which no real decode step would see.  A step replays the three graphs.
    graphs = {}
    with torch.cuda.stream(stream):
        step(stream)  # warm: first calls set kernel attributes
        stream.synchronize()
        for m in DECODE_MS:
            graphs[m] = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graphs[m], stream=stream):
                step(stream, ms=(m,))
    launches_per_step = L * len(DECODE_MS)

    def replay_step():
        for m in DECODE_MS:
            graphs[m].replay()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            replay_step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        start.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                replay_step()
        end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = start.elapsed_time(end)
    ms_max = max_over_ranks(ms, world)
    value = world * step_bytes(L) * args.steps / (ms_max * 1e-3) / 1e9
    tflops = world * step_flops(L) * args.steps / (ms_max * 1e-3) / 1e12

    # Per-M breakdown (same graph technique, one M at a time).
    per_m = {}
    for m in DECODE_MS:
        with torch.cuda.stream(stream):
            g = graphs[m]
            g.replay()
            stream.synchronize()
            reps = max(3, args.steps // 4)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
            stream.synchronize()
        t_call = e0.elapsed_time(e1) * 1e-3 / (reps * L)
        per_m[str(m)] = {"us_per_call": t_call * 1e6, "hbm_gbs": decode_call_bytes(m) / t_call / 1e9,
                         "weight_gbs": (N_DIM * K_DIM // 8 + 4 * (N_DIM + K_DIM)) / t_call / 1e9,
                         "tflops_equiv": 2 * m * N_DIM * K_DIM / t_call / 1e12,
                         "frac_hbm": decode_call_bytes(m) / t_call / 1e9 / peaks["hbm_gbs"]}

    # Kernels forced by path, for comparison with the ones AUTO picks (same pool, same graphs).
    def time_forced(m, path):
        with torch.cuda.stream(stream):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for (P, a, b) in pool:
                    ops.ob_linear(xs[m], P, a, b, out=ys[m], path=path, stream=stream)
            g.replay()
            stream.synchronize()
            reps = max(3, args.steps // 4)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
            stream.synchronize()
        del g
        t = e0.elapsed_time(e1) * 1e-3 / (reps * L)
        return {"us_per_call": t * 1e6, "hbm_gbs": decode_call_bytes(m) / t / 1e9,
                "frac_hbm": decode_call_bytes(m) / t / 1e9 / peaks["hbm_gbs"]}

    for name, code in (("mma", ops.OB_PATH_MMA_DECODE), ("i8", ops.OB_PATH_I8), ("lut", ops.OB_PATH_SIMT),
                       ("auto_plain", ops.OB_PATH_AUTO)):
        for m in DECODE_MS:
            if name in ("lut", "auto_plain") and m > 1:
                continue
            per_m[f"{m}_{name}_forced"] = time_forced(m, code)

    # Dominant kernel of the step: the warp-level MMA decode kernel, which serves the M = 4 and
    # M = 16 calls (one launch each); its achieved bandwidth is its algorithmic bytes over its own
    # measured launch times (the M = 1 calls run the table-driven CUDA-core kernel).
    mma_ms = [m for m in DECODE_MS if m > 1]
    t_mma = sum(per_m[str(m)]["us_per_call"] for m in mma_ms) * 1e-6
    achieved = sum(decode_call_bytes(m) for m in mma_ms) / t_mma / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"],
                "kernel": "sign_gemm_mma_decode_kernel",
                "traffic": ncu_traffic("linear_mma_decode.cu", "decode_4096x4096")}

    # End to end through the C-ABI with host buffers: pinned X in, Y out, inside the timed region.
    hx = {m: xs[m].cpu().pin_memory() for m in DECODE_MS}
    hy = {m: torch.empty((m, N_DIM), dtype=torch.bfloat16).pin_memory() for m in DECODE_MS}
    e2e_layers = min(L, 48)

    def e2e_step():
        for m in DECODE_MS:
            for (P, a, b) in pool[:e2e_layers]:
                xs[m].copy_(hx[m], non_blocking=True)
                ops.ob_linear(xs[m], P, a, b, out=ys[m], stream=stream)
                hy[m].copy_(ys[m], non_blocking=True)

    e2e_steps = max(2, args.steps // 10)
    with torch.cuda.stream(stream):
        e2e_step()
        stream.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = world * step_bytes(e2e_layers) * e2e_steps / (e2e_ms * 1e-3) / 1e9
    h2d = e2e_layers * sum(2 * m * K_DIM for m in DECODE_MS)
    d2h = e2e_layers * sum(2 * m * N_DIM for m in DECODE_MS)

    extra = run_extra(ops, dev, stream, peaks) if (args.extra and world == 1) else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, el, svd_s = oracle_step_sample(args.cpu_seconds)
        cpu = {"value": step_bytes(1) * n / el / 1e9, "unit": "GB/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": f"{n} steps x (M=1,4,16) on one 4096x4096 layer in {el:.1f} s, fp64 direct form "
                         f"(W_hat materialised per call); oracle SVID (full SVD) {svd_s:.1f} s once"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "onebit_decode_4096x4096_M1_4_16", "M": list(DECODE_MS), "N": N_DIM,
                       "K": K_DIM, "layers_per_step": L,
                       "l2": f"inputs larger than L2: rotating pool of {L} weight sets "
                             f"({L * decode_call_bytes(0) / 1e6:.0f} MB) per pass",
                       "graph": "one CUDA graph per M (192 calls each), replayed M=1,4,16 per step; programmatic dependent launch between calls",
                       "path": "OB_PATH_AUTO | OB_FLAG_STATIC_WEIGHTS (weights loaded once, reused every step); per_m['1_auto_plain_forced'] times plain AUTO",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "tflops_equiv": tflops,
            "per_m": per_m,
            "roofline": roofline,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "layers_per_step": e2e_layers},
            "gpu_launches": args.steps * launches_per_step,
            "clocks": clocks.summary(),
            "offline": {"pack_ms": pack_ms, "svid_ms": svid_ms, "svid_iters": svid_iters,
                        "pack_gbs": (N_DIM * K_DIM * 4 + N_DIM * K_DIM // 8) / (pack_ms * 1e-3) / 1e9},
            "cpu_baseline": cpu,
            "extra": extra,
        }
        print(json.dumps(line), flush=True)
    graphs.clear()



def _timed(step_fn, args, world, stream, local):
    """Warm up, then time args.steps calls of step_fn on `stream` (barrier + sync on both sides)."""
    import torch
    for _ in range(args.warmup):
        step_fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                step_fn()
            e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1), world), e0.elapsed_time(e1), clocks.summary()


def run_prefill(args, world, rank, local):
    """OneBit prefill: X 2048 x 4096 bf16, W 11008 x 4096 -> Y 2048 x 11008 (tensor-core path)."""
    import torch
    from binary_weight_gemm_b200 import build, synth
    build.build()
    from binary_weight_gemm_b200 import ops
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    peaks = load_peaks()
    M, K, N = 2048, 4096, 11008
    W = torch.from_numpy(synth.weights(2, N, K)).to(dev)
    P = ops.ob_pack_signs(W, stream=stream)
    a, b, _, _, _ = ops.ob_svid_rank1(W, stream=stream)
    del W
    # Three (X, W_packed, Y) sets, 3 x 67 MB > L2, rotated call to call.
    sets = [(torch.from_numpy(synth.activations(2 + i, M, K)[0].view(np.int16)).to(dev).view(torch.bfloat16),
             P.clone(), a.clone(), b.clone(), torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for i in range(3)]
    it = [0]

    def step():
        X, Pp, aa, bb, Y = sets[it[0] % 3]
        it[0] += 1
        ops.ob_linear(X, Pp, aa, bb, out=Y, stream=stream)

    ms_max, ms, clocks = _timed(step, args, world, stream, local)
    flops = 2 * M * N * K
    t = ms * 1e-3 / args.steps
    value = world * flops * args.steps / (ms_max * 1e-3) / 1e12
    # e2e: pinned X in, Y out, per call.
    hx = sets[0][0].cpu().pin_memory()
    hy = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()

    def e2e_step():
        X, Pp, aa, bb, Y = sets[0]
        X.copy_(hx, non_blocking=True)
        ops.ob_linear(X, Pp, aa, bb, out=Y, stream=stream)
        hy.copy_(Y, non_blocking=True)

    e2e_steps = max(3, args.steps // 4)
    with torch.cuda.stream(stream):
        e2e_step()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        Wn = synth.weights(2, N, K)
        an, bn = a.cpu().numpy(), b.cpu().numpy()
        xs = synth.activations(2, 64, K)[1]
        S = oracle.sign_pm1(Wn)
        n, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < args.cpu_seconds:
            oracle.onebit_linear(xs[:16], S, an, bn)
            n += 1
        el = time.perf_counter() - t0
        cpu = {"value": n * 2 * 16 * N * K / el / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": f"{n} calls of 16 token rows x (4096 -> 11008), fp64 direct form, in {el:.1f} s"}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "onebit_prefill_M2048_4096x11008", "M": M, "N": N, "K": K,
                       "l2": "inputs larger than L2: three rotating (X, W, Y) sets, 200 MB",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "roofline": {"bound": "tensor", "achieved": flops / t / 1e12, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": flops / t / 1e12 / peaks["bf16_tflops"],
                         "frac_sustained": flops / t / 1e12 / (peaks["bf16_tflops_sustained"] or peaks["bf16_tflops"]),
                         "peak_source": peaks["source"], "kernel": prefill_kernel_name(),
                         "traffic": ncu_traffic(*prefill_kernel_source(), "prefill_2048x4096x11008")},
            "e2e": {"value": world * flops * e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": 2 * M * K, "d2h_bytes_per_step": 2 * M * N},
            "gpu_launches": args.steps, "clocks": clocks, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)

def factorize_flops(N, K, r, sweeps, admm_iters, cg_iters, refit_rounds):
    """fp32 multiply-add work (2 flops each) of one dbf_factorize run, as its GEMMs count it."""
    gemm = lambda m, n, k: 2 * m * n * k  # noqa: E731
    cg = lambda rows, iters: gemm(rows, r, r) * (iters + 1)  # noqa: E731
    start = gemm(N, r, K) + gemm(r, r, N) + gemm(K, r, N) + cg(K, 4 * cg_iters) + gemm(N, K, r)
    step_a = gemm(r, r, K) + gemm(N, r, K) + cg(N, cg_iters)
    step_b = gemm(r, r, N) + gemm(K, r, N) + cg(K, cg_iters)
    sweep = admm_iters * (step_a + step_b) + gemm(N, K, r)
    refit = 3 * gemm(N, K, r) + gemm(r, r, N) + gemm(r, r, K) + gemm(K, r, N)
    return start + sweeps * sweep + refit_rounds * refit + gemm(N, K, r)


def run_factorize(args, world, rank, local):
    """DBF factorisation of one 4096 x 4096 weight at r = 2048 (the bits of OneBit), offline.

    Times whole dbf_factorize calls (synchronous: the error is read back after every
    sweep) after one untimed call with a single sweep.  Reports seconds per weight, the
    fp32 GEMM work done per second, and the relative error of the result.
    """
    import torch
    from binary_weight_gemm_b200 import build, synth
    build.build()
    from binary_weight_gemm_b200 import ops
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    N = K = 4096
    r = 2048
    sweeps, admm_iters, cg_iters, refit_rounds = 20, 3, 5, 2
    W = torch.from_numpy(synth.weights(1, N, K)).to(dev)
    omega = torch.from_numpy((np.random.default_rng(11).standard_normal((K, r)) / np.sqrt(K)).astype(np.float32)).to(dev)
    ws = torch.empty(ops.dbf_factorize_workspace_size(N, K, r), dtype=torch.uint8, device=dev)
    ops.dbf_factorize(W, r, omega, sweeps=1, workspace=ws)
    reps = max(1, min(args.steps, 2))
    torch.cuda.synchronize()
    barrier(world)
    with ClockSampler(local) as clocks:
        t0 = time.perf_counter()
        for _ in range(reps):
            res = ops.dbf_factorize(W, r, omega, sweeps=sweeps, admm_iters=admm_iters, cg_iters=cg_iters,
                                    refit_rounds=refit_rounds, workspace=ws)
        el = time.perf_counter() - t0
    el = max_over_ranks(el * 1e3, world) * 1e-3
    assert ops.ob_last_device_error() == 0
    flops = factorize_flops(N, K, r, sweeps, admm_iters, cg_iters, refit_rounds)
    nW = float(torch.linalg.vector_norm(W).item())
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # The fp64 oracle (exact r x r solves) on a bounded sample: 2 sweeps of a 1024 x 1024
        # weight at r = 512, scaled to the full problem by the counted GEMM work.
        import oracle.dbf_factorize as F
        ns, rs = 1024, 512
        Ws = synth.weights(1, ns, ns).astype(np.float64)
        oms = np.random.default_rng(11).standard_normal((ns, rs)) / np.sqrt(ns)
        t0 = time.perf_counter()
        F.dbf_factorize(Ws, rs, sweeps=2, omega=oms)
        t_s = time.perf_counter() - t0
        f_s = factorize_flops(ns, ns, rs, 2, admm_iters, cg_iters, refit_rounds)
        cpu = {"value": t_s * flops / f_s, "unit": "s", "cores": cpu_cores(), "kind": "oracle",
               "sample": f"2 sweeps of a {ns}x{ns} weight at r={rs} in {t_s:.1f} s, scaled by counted GEMM work "
                         "to the full factorisation"}
    if rank == 0:
        line = {
            "metric": "dbf_factorize seconds per 4096x4096 weight (r=2048)", "value": el / reps, "unit": "s",
            "n_gpus": world, "steps": reps, "warmup": 1, "ms_per_step": el / reps * 1e3,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "dbf_factorize_4096x4096_r2048", "N": N, "K": K, "r": r, "sweeps": sweeps,
                       "admm_iters": admm_iters, "cg_iters": cg_iters, "refit_rounds": refit_rounds,
                       "timing": "host wall clock around synchronous calls (the call reads its error back "
                                 "after every sweep)"},
            "gemm_tflops": flops * reps / el / 1e12,
            "relative_error": res["error"] / nW, "relative_error_best_iterate": res["best"] / nW,
            "history": [h / nW for h in res["history"]],
            "gpu_launches": None, "clocks": clocks.summary(), "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


STACK_SHAPES = {"q": (4096, 4096), "k": (4096, 4096), "v": (4096, 4096), "o": (4096, 4096),
                "gate": (4096, 11008), "up": (4096, 11008), "down": (11008, 4096)}  # name: (K, N)


def run_stack(args, world, rank, local):
    """Decode through a stack of 7B-shaped OneBit linear layers, one token (batch M) at a time.

    Per block: q, k, v, o (4096 -> 4096), gate, up (4096 -> 11008), down (11008 -> 4096),
    chained through their outputs (q, k, v read the block input; o reads q's output;
    gate and up read o's; down reads gate's; the next block reads down's).  Attention,
    the gated activation and the norms are not part of this library, so a layer's output
    feeds the next layer directly.  32 blocks = 224 distinct packed weight buffers (819 MB,
    6.5 x L2).  Timed: one ob_linear_stack per token (one persistent launch, grid barriers
    where a layer reads an earlier output), captured as a CUDA graph per batch size; the
    same token as 224 ob_linear calls in a graph is timed beside it.
    """
    import torch
    from binary_weight_gemm_b200 import build, synth
    build.build()
    from binary_weight_gemm_b200 import ops
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    peaks = load_peaks()
    blocks = args.blocks
    ms_list = (1, 2, 16)
    lin_path = ops.OB_PATH_AUTO | ops.OB_FLAG_STATIC_WEIGHTS  # the weights are written once, before timing
    # One seeded matrix per shape, packed and SVID'd by the library, cloned into every block.
    base = {}
    for K, N in sorted(set(STACK_SHAPES.values())):
        W = torch.from_numpy(synth.weights(7 + K % 97 + N % 89, N, K)).to(dev)
        P = ops.ob_pack_signs(W, stream=stream)
        a, b, _, _, _ = ops.ob_svid_rank1(W, stream=stream)
        base[(K, N)] = (P, a, b)
        del W
    layers = [{name: tuple(t.clone() for t in base[STACK_SHAPES[name]]) for name in STACK_SHAPES}
              for _ in range(blocks)]
    wbytes = sum(N * K // 8 + 4 * (N + K) for K, N in STACK_SHAPES.values()) * blocks
    acts = {}
    for m in ms_list:
        x0 = torch.from_numpy(synth.activations(7, m, 4096)[0].view(np.int16)).to(dev).view(torch.bfloat16)
        buf = {name: torch.empty((m, N), dtype=torch.bfloat16, device=dev) for name, (K, N) in STACK_SHAPES.items()}
        acts[m] = (x0, buf)

    def token(m, s):
        x0, buf = acts[m]
        x = x0
        for L in layers:
            for name in ("q", "k", "v"):
                P, a, b = L[name]
                ops.ob_linear(x, P, a, b, out=buf[name], stream=s, path=lin_path)
            P, a, b = L["o"]
            ops.ob_linear(buf["q"], P, a, b, out=buf["o"], stream=s, path=lin_path)
            for name in ("gate", "up"):
                P, a, b = L[name]
                ops.ob_linear(buf["o"], P, a, b, out=buf[name], stream=s, path=lin_path)
            P, a, b = L["down"]
            ops.ob_linear(buf["gate"], P, a, b, out=buf["down"], stream=s, path=lin_path)
            x = buf["down"]

    def spec(m):
        """The same token as ob_linear_stack descriptors (after_previous where a layer reads an
        output of the block it is in, or of the previous block)."""
        x0, buf = acts[m]
        out, x = [], x0
        for bi, L in enumerate(layers):
            for name in ("q", "k", "v"):
                P, a, b = L[name]
                out.append((x, P, a, b, buf[name], bi > 0 and name == "q"))
            P, a, b = L["o"]
            out.append((buf["q"], P, a, b, buf["o"], True))
            for name in ("gate", "up"):
                P, a, b = L[name]
                out.append((buf["o"], P, a, b, buf[name], name == "gate"))
            P, a, b = L["down"]
            out.append((buf["gate"], P, a, b, buf["down"], True))
            x = buf["down"]
        return out

    specs = {m: spec(m) for m in ms_list}
    ws = torch.zeros(ops.ob_stack_workspace_size(), dtype=torch.uint8, device=dev)

    # The dataflow form (int8, one token): every layer of every block writes its own buffer, so
    # the list qualifies; consumers poll their producers' tagged outputs, no grid barriers.
    df_ms = [m for m in ms_list if m == 1]

    def spec_df(m):
        x0, _ = acts[m]
        out, x = [], x0
        for bi, L in enumerate(layers):
            bb = {name: torch.empty((m, N), dtype=torch.bfloat16, device=dev) for name, (K, N) in STACK_SHAPES.items()}
            for name in ("q", "k", "v"):
                P, a, b = L[name]
                out.append((x, P, a, b, bb[name], bi > 0 and name == "q"))
            P, a, b = L["o"]
            out.append((bb["q"], P, a, b, bb["o"], True))
            for name in ("gate", "up"):
                P, a, b = L[name]
                out.append((bb["o"], P, a, b, bb[name], name == "gate"))
            P, a, b = L["down"]
            out.append((bb["gate"], P, a, b, bb["down"], True))
            x = bb["down"]
        return out

    dspecs = {m: spec_df(m) for m in df_ms}
    dws = {m: torch.zeros(ops.ob_linear_stack_workspace_size(dspecs[m], m), dtype=torch.uint8, device=dev)
           for m in df_ms}
    graphs, pgraphs = {}, {}
    with torch.cuda.stream(stream):
        for m in ms_list:
            token(m, stream)
            ops.ob_linear_stack(specs[m], m, workspace=ws, stream=stream)
        stream.synchronize()
        for m in ms_list:
            graphs[m] = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graphs[m], stream=stream):
                token(m, stream)
            pgraphs[m] = torch.cuda.CUDAGraph()
            with torch.cuda.graph(pgraphs[m], stream=stream):
                ops.ob_linear_stack(specs[m], m, workspace=ws, stream=stream)
        dgraphs = {}
        for m in df_ms:
            ops.ob_linear_stack(dspecs[m], m, workspace=dws[m], stream=stream)
            stream.synchronize()
            dgraphs[m] = torch.cuda.CUDAGraph()
            with torch.cuda.graph(dgraphs[m], stream=stream):
                ops.ob_linear_stack(dspecs[m], m, workspace=dws[m], stream=stream)
        # The bf16 warp-MMA stack form forced at one token, beside the int8 form AUTO takes.
        mgraphs = {}
        ops.ob_linear_stack(specs[1], 1, workspace=ws, stream=stream, path=ops.OB_PATH_MMA_DECODE)
        stream.synchronize()
        mgraphs[1] = torch.cuda.CUDAGraph()
        with torch.cuda.graph(mgraphs[1], stream=stream):
            ops.ob_linear_stack(specs[1], 1, workspace=ws, stream=stream, path=ops.OB_PATH_MMA_DECODE)
    calls = 7 * blocks

    def step():
        for m in ms_list:
            pgraphs[m].replay()

    ms_max, ms, clocks = _timed(step, args, world, stream, local)
    per_m = {}
    for mode, gs in (("persistent", pgraphs), ("per_call", graphs), ("persistent_bf16mma", mgraphs),
                     ("persistent_dataflow", dgraphs)):
        for m in gs:
            reps = max(3, args.steps // 2)
            with torch.cuda.stream(stream):
                gs[m].replay()
                stream.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(reps):
                    gs[m].replay()
                e1.record(stream)
                stream.synchronize()
            t_tok = e0.elapsed_time(e1) * 1e-3 / reps
            abytes = sum(2 * m * (K + N) for K, N in STACK_SHAPES.values()) * blocks
            per_m[f"{mode}_M{m}"] = {"us_per_token": t_tok * 1e6, "tokens_per_s": m / t_tok,
                                     "weight_gbs": wbytes / t_tok / 1e9, "hbm_gbs": (wbytes + abytes) / t_tok / 1e9,
                                     "frac_hbm": (wbytes + abytes) / t_tok / 1e9 / peaks["hbm_gbs"],
                                     "us_per_layer": t_tok * 1e6 / calls}
    assert ops.ob_last_device_error() == 0
    step_bytes_total = sum(wbytes + sum(2 * m * (K + N) for K, N in STACK_SHAPES.values()) * blocks
                           for m in ms_list)
    value = world * step_bytes_total * args.steps / (ms_max * 1e-3) / 1e9
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"onebit_decode_stack_7b_{blocks}blocks", "M": list(ms_list),
                       "layers_per_token": calls, "weights_mb": wbytes / 1e6,
                       "l2": f"inputs larger than L2: {blocks * 7} distinct weight buffers ({wbytes / 1e6:.0f} MB)",
                       "graph": "one CUDA graph per token and M holding one ob_linear_stack (persistent, "
                                "grid barriers between dependent layers; AUTO: int8 form at M=1 and 2, bf16 "
                                "warp-MMA form at M=16; persistent_bf16mma_M1 forces the bf16 form); per_call_* "
                                "times one ob_linear per layer (AUTO | OB_FLAG_STATIC_WEIGHTS) in a graph with "
                                "programmatic dependent launch; persistent_dataflow_* gives every layer its own "
                                "output buffer and the workspace of ob_linear_stack_workspace_size (tagged outputs "
                                "polled by their consumers instead of grid barriers)",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "per_m": per_m,
            "gpu_launches": args.steps * len(ms_list), "clocks": clocks, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    graphs.clear()
    pgraphs.clear()
    mgraphs.clear()


SWEEP_SHAPES = ((4096, 4096), (4096, 11008), (11008, 4096))  # (K, N): the 7B-shaped outlier sweep
SWEEP_MS = (1, 16, 256, 4096)


def run_sweep(args, world, rank, local):
    """The 7B-shaped layer sweep with outlier activations: K -> N in {4096 -> 4096,
    4096 -> 11008, 11008 -> 4096} x M in {1, 16, 256, 4096}, through ob_linear (AUTO).

    X ~ N(0, 1) bf16 with 6 fixed channels scaled x60 (the LLM.int8() page's outlier
    features); W ~ N(0, 0.02) packed and SVID'd by the library.  M <= 16: one CUDA graph over
    a pool of distinct weight copies larger than 3 x L2 (HBM-bound calls); M >= 256: rotating
    input / output sets larger than L2.  Reports per (shape, M) the time per call, the HBM
    fraction (packed weights + scales + X + Y bytes) and the dense bf16 fraction (2 M N K)."""
    import torch
    from binary_weight_gemm_b200 import build, synth
    build.build()
    from binary_weight_gemm_b200 import ops
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    peaks = load_peaks()
    rows = {}
    for si, (K, N) in enumerate(SWEEP_SHAPES):
        W = torch.from_numpy(synth.weights(4 + si, N, K)).to(dev)
        P = ops.ob_pack_signs(W, stream=stream)
        a, b, _, _, _ = ops.ob_svid_rank1(W, stream=stream)
        del W
        wbytes = N * K // 8 + 4 * (N + K)
        for M in SWEEP_MS:
            X = torch.from_numpy(synth.activations(4 + si, M, K, outliers=True)[0].view(np.int16)).to(dev)
            X = X.view(torch.bfloat16)
            call_bytes = wbytes + 2 * M * K + 2 * M * N
            if M <= 16:
                nset = max(8, -(-3 * 126 * 2**20 // wbytes))
                pool = [P.clone() for _ in range(nset)]
                Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
                t = _time_graph(lambda i: ops.ob_linear(X, pool[i % nset], a, b, out=Y, stream=stream), stream, nset)
                del pool
            else:
                nset = max(2, -(-2 * 126 * 2**20 // (2 * M * (K + N))))
                sets = [(X.clone(), torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for _ in range(nset)]
                # ob_linear_ws: few-tile problems split over K through this workspace.
                wsb = ops.ob_linear_workspace_size(M, N, K)
                ws = torch.empty(wsb, dtype=torch.uint8, device=dev) if wsb else None
                t = _time_calls(lambda i: ops.ob_linear(sets[i % nset][0], P, a, b, out=sets[i % nset][1],
                                                        stream=stream, workspace=ws), stream, max(10, 3 * nset))
                del sets
            fl = 2 * M * N * K
            rows[f"{K}x{N}_M{M}"] = {"us_per_call": t * 1e6, "hbm_gbs": call_bytes / t / 1e9,
                                     "frac_hbm": call_bytes / t / 1e9 / peaks["hbm_gbs"],
                                     "tflops": fl / t / 1e12, "frac_bf16_burst": fl / t / 1e12 / peaks["bf16_tflops"]}
    if rank == 0:
        tot_t = sum(r["us_per_call"] for r in rows.values()) * 1e-6
        tot_fl = sum(2 * M * N * K for (K, N) in SWEEP_SHAPES for M in SWEEP_MS)
        line = {
            "metric": METRIC, "value": tot_fl / tot_t / 1e12, "unit": "TFLOP/s", "n_gpus": world, "steps": 1,
            "warmup": 1, "ms_per_step": tot_t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "onebit_sweep_7b_outliers", "shapes_KxN": [list(x) for x in SWEEP_SHAPES],
                       "M": list(SWEEP_MS), "outliers": "6 channels x60",
                       "l2": "M<=16: weight pool > 3x L2 in one CUDA graph; M>=256: rotating sets > L2",
                       "api": "ob_linear (AUTO); M>=256 with the workspace of ob_linear_workspace_size (split over K "
                              "where few output tiles)"},
            "per_case": rows, "peak_source": peaks["source"], "gpu_launches": None, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)


def _time_calls(fn, stream, reps):
    import torch
    with torch.cuda.stream(stream):
        fn(0)
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(reps):
            fn(i)
        e1.record(stream)
        stream.synchronize()
    return e0.elapsed_time(e1) * 1e-3 / reps


def _time_graph(fn, stream, reps, replays=5):
    """Per-call time of fn(0 .. reps-1) captured in one CUDA graph (the deployed form: no host
    launch overhead, programmatic dependent launch between kernels where the library uses it)."""
    import torch
    with torch.cuda.stream(stream):
        fn(0)  # warm: kernel attributes, module load
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(reps):
                fn(i)
        g.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(replays):
            g.replay()
        e1.record(stream)
        stream.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e-3 / (reps * replays)


def run_extra(ops, dev, stream, peaks):
    """Prefill and DBF workloads, measured briefly in the same run (rotating buffers > L2)."""
    import torch
    from binary_weight_gemm_b200 import synth
    out = {}
    # Prefill: X 2048 x 4096, W 11008 x 4096 (5.6 MB packed), Y 2048 x 11008.
    M, K, N = 2048, 4096, 11008
    W = torch.from_numpy(synth.weights(2, N, K)).to(dev)
    P = ops.ob_pack_signs(W, stream=stream)
    a, b, _, _, _ = ops.ob_svid_rank1(W, stream=stream)
    del W
    sets = [(torch.from_numpy(synth.activations(2 + i, M, K)[0].view(np.int16)).to(dev).view(torch.bfloat16),
             P.clone(), torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for i in range(3)]
    t = _time_calls(lambda i: ops.ob_linear(sets[i % 3][0], sets[i % 3][1], a, b, out=sets[i % 3][2],
                                            stream=stream), stream, 30)
    fl = 2 * M * N * K
    out["prefill_2048x4096x11008"] = {"us_per_call": t * 1e6, "tflops": fl / t / 1e12,
                                      "frac_bf16_burst": fl / t / 1e12 / peaks["bf16_tflops"],
                                      "frac_bf16_sustained": fl / t / 1e12 / (peaks["bf16_tflops_sustained"] or 1),
                                      "kernel": prefill_kernel_name()}
    # The same prefill followed by LayerNorm over each token's outputs (ob_linear_ln).
    t_ln = _time_calls(lambda i: ops.ob_linear_ln(sets[i % 3][0], sets[i % 3][1], a, b, out=sets[i % 3][2],
                                                  stream=stream), stream, 30)
    out["prefill_ln_2048x4096x11008"] = {"us_per_call": t_ln * 1e6, "tflops": fl / t_ln / 1e12,
                                         "ln_us": (t_ln - t) * 1e6,
                                         "kernels": prefill_kernel_name() + " + layernorm_rows_kernel"}
    del sets
    # OneBit decode 4096 x 4096 followed by LayerNorm, M = 1 and 16 (pool of weight sets > L2).
    W = torch.from_numpy(synth.weights(1, 4096, 4096)).to(dev)
    P1 = ops.ob_pack_signs(W, stream=stream)
    a1, b1, _, _, _ = ops.ob_svid_rank1(W, stream=stream)
    del W
    pool = [P1.clone() for _ in range(192)]
    for M in (1, 16):
        X = torch.from_numpy(synth.activations(1, M, 4096)[0].view(np.int16)).to(dev).view(torch.bfloat16)
        Y = torch.empty((M, 4096), dtype=torch.bfloat16, device=dev)
        t0 = _time_graph(lambda i: ops.ob_linear(X, pool[i % 192], a1, b1, out=Y, stream=stream), stream, 192)
        t1 = _time_graph(lambda i: ops.ob_linear_ln(X, pool[i % 192], a1, b1, out=Y, stream=stream), stream, 192)
        out[f"decode_ln_M{M}"] = {"us_per_call": t1 * 1e6, "linear_only_us": t0 * 1e6, "ln_us": (t1 - t0) * 1e6,
                                  "hbm_gbs": decode_call_bytes(M) / t1 / 1e9}
    del pool
    # DBF: K = N = 4096, r = 2048 (the configured workload) and the middle dimensions of
    # about 0.5, 1.5 and 2.3 bits per weight (non-uniform r per layer).
    for r in (2048, 1056, 3072, 4704):
        f = synth.dbf_factors(3, 4096, r, 4096)
        SB = ops.ob_pack_signs(torch.from_numpy(f["S_B"].astype(np.float32)).to(dev), stream=stream)
        SA = ops.ob_pack_signs(torch.from_numpy(f["S_A"].astype(np.float32)).to(dev), stream=stream)
        vec = {k: torch.from_numpy(f[k]).to(dev) for k in ("a", "m", "b")}
        wbytes = r * 4096 // 8 * 2
        for M in (1, 512):
            nset = max(8, -(-3 * 126 * 2**20 // (wbytes + 2 * M * 4096 * 2)))  # > 3x L2 in total
            pool = [(SB.clone(), SA.clone()) for _ in range(nset)]
            X = torch.from_numpy(synth.activations(3, M, 4096)[0].view(np.int16)).to(dev).view(torch.bfloat16)
            Y = torch.empty((M, 4096), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(ops.dbf_workspace_size(M, r), dtype=torch.uint8, device=dev)
            timer = _time_graph  # the deployed form at every M (no host launch cost between calls)
            # Weights are static here (written once, before the timing): decode-size calls say so.
            dpath = ops.OB_PATH_AUTO | (ops.OB_FLAG_STATIC_WEIGHTS if M <= 16 else 0)
            t = timer(lambda i: ops.dbf_linear(X, pool[i % nset][0], vec["m"], pool[i % nset][1], vec["a"],
                                               vec["b"], out=Y, workspace=ws, stream=stream, path=dpath), stream,
                      max(50, 2 * nset))
            fl = 2 * M * r * (4096 + 4096)
            byts = wbytes + 4 * (4096 * 2 + r) + 2 * M * 4096 * 2
            key = f"dbf_M{M}" if r == 2048 else f"dbf_r{r}_M{M}"
            out[key] = {"us_per_call": t * 1e6, "r": r, "bits_per_weight": r * 8192 / 4096**2,
                        "tflops_equiv": 2 * M * 4096 * 4096 / t / 1e12, "tflops_alg": fl / t / 1e12,
                        "hbm_gbs": byts / t / 1e9, "frac_hbm": byts / t / 1e9 / peaks["hbm_gbs"],
                        "frac_bf16_burst": fl / t / 1e12 / peaks["bf16_tflops"]}
            if M == 1 and r == 2048:
                # Beside AUTO with static weights (two per-call kernels): plain AUTO, and both
                # products in one persistent launch (OB_PATH_STACK).
                for name, pth in (("dbf_M1_plain", ops.OB_PATH_AUTO), ("dbf_M1_one_launch", ops.OB_PATH_STACK)):
                    t2 = timer(lambda i: ops.dbf_linear(X, pool[i % nset][0], vec["m"], pool[i % nset][1],
                                                        vec["a"], vec["b"], out=Y, workspace=ws, stream=stream,
                                                        path=pth), stream, max(50, 2 * nset))
                    out[name] = {"us_per_call": t2 * 1e6, "hbm_gbs": byts / t2 / 1e9,
                                 "frac_hbm": byts / t2 / 1e9 / peaks["hbm_gbs"]}
            del pool
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["decode", "prefill", "stack", "factorize", "sweep"], default="decode",
                    help="decode: OneBit 4096x4096 at M=1,4,16 (default); prefill: M=2048, 4096 -> 11008; "
                         "stack: one token through 32 blocks of 7B-shaped OneBit layers at M=1 and 16; "
                         "factorize: DBF factorisation of a 4096x4096 weight at r=2048; "
                         "sweep: the 7B-shaped layer sweep with outlier activations")
    ap.add_argument("--blocks", type=int, default=32, help="blocks of the stack workload")
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--no-extra", dest="extra", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_init()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.workload == "prefill":
            run_prefill(args, world, rank, local)
        elif args.workload == "stack":
            run_stack(args, world, rank, local)
        elif args.workload == "factorize":
            run_factorize(args, world, rank, local)
        elif args.workload == "sweep":
            run_sweep(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
