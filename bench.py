"""Benchmark: dense NHWC convolution (bf16, N=32, 56x56, 64->64, K=3) on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-extras]

A step is one forward dense convolution over one batch of 32 images (the hot path: tensor
maps, TMA im2col gather, tcgen05 mainloop, epilogue) with inputs resident in HBM. Inputs and
outputs rotate over enough buffer sets that their total exceeds twice the L2 size, so every
step reads cold data. The steps are replayed from CUDA graphs captured around the C-ABI call
and timed with CUDA events on the launching stream, bracketed by a barrier and a device
synchronisation; the reported time is the maximum over ranks. Under torchrun every rank
runs its own batch (weak scaling, no collective on the data path).

Also reported: "e2e" -- the same metric through the public Python API with the inputs copied
from pinned host memory and the output copied back inside the timed region; "roofline" for
the dense kernel; "cpu_baseline" -- the CPU oracle timed on a bounded sample of the same
workload (rank 0, N=1); and, unless --no-extras, the other configurations (pointwise, large
dense, the depthwise sweep in both modes) as secondary measurements.

--impl reference times the CPU oracle itself on the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "dense conv TFLOP/s (% bf16 TC peak); depthwise GB/s (% HBM) on 1 B200"
L2_BYTES = 126 * 1024 * 1024
CASE = workloads.DENSE_3X3
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "cnn_convolution_nhwc_b200", "csrc")
    for name in sorted(os.listdir(d)):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on these sources."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(kernel, {}).get(workload)
    if not rec or rec.get("source_hash") != source_hash():
        return None
    return rec.get("bytes_per_launch")


# ------------------------------------------------------------------------------------------
# Clock sampling (NVML) during the timed region
# ------------------------------------------------------------------------------------------
REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # reading clocks is best effort; the line says so
            self._nv = None
            self.error = f"{type(e).__name__}: {e}"

    def _run(self):
        nv = self._nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self._h))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": getattr(self, "error", "")}
        reasons = [name for bit, name in REASON_BITS.items() if self.reasons & bit and name != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------
# Distributed plumbing
# ------------------------------------------------------------------------------------------
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend: str):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            if self.pg.get_backend() == "nccl":
                import torch
                self.pg.barrier(device_ids=[torch.cuda.current_device()])
            else:
                self.pg.barrier()

    def max(self, v: float) -> float:
        if self.pg is None:
            return v
        import torch
        dev = torch.device("cuda", torch.cuda.current_device()) if self.pg.get_backend() == "nccl" else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ------------------------------------------------------------------------------------------
# Timing helpers
# ------------------------------------------------------------------------------------------
def rotating_sets(set_bytes: int) -> int:
    """Buffer sets so that their total is at least twice the L2 (1 when one set already is)."""
    return max(1, math.ceil(2 * L2_BYTES / max(1, set_bytes)))


def capture(fn_list):
    """One CUDA graph per callable plus one graph running them all in order."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for fn in fn_list:   # eager warm-up off the capture
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    singles = []
    for fn in fn_list:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        singles.append(g)
    cycle = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cycle):
        for fn in fn_list:
            fn()
    torch.cuda.synchronize()
    return singles, cycle


def replay(singles, cycle, steps: int):
    R = len(singles)
    q, r = divmod(steps, R)
    for _ in range(q):
        cycle.replay()
    for i in range(r):
        singles[i].replay()


def time_graph_steps(singles, cycle, steps: int, warmup: int, dist=None, sampler=None):
    """Replays `steps` steps; returns elapsed ms on the launching stream (max over ranks)."""
    import torch
    replay(singles, cycle, warmup)
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.start()
    start.record(stream)
    replay(singles, cycle, steps)
    end.record(stream)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.stop()
    if dist is not None:
        dist.barrier()
    ms = start.elapsed_time(end)
    return dist.max(ms) if dist is not None else ms


# ------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------
def dense_bench(cb, torch, case, X0, F0, steps, warmup, dist=None, sampler=None):
    set_bytes = case.bytes
    R = rotating_sets(set_bytes)
    Xs = [X0.clone() for _ in range(R)]
    Fs = [F0.clone() for _ in range(R)]
    Ys = [torch.empty((case.N, case.Ho, case.Wo, case.Cout), dtype=X0.dtype, device=X0.device) for _ in range(R)]
    fns = [(lambda i=i: cb.conv2d_nhwc_fwd(Xs[i], Fs[i], Ys[i])) for i in range(R)]
    singles, cycle = capture(fns)
    ms = time_graph_steps(singles, cycle, steps, warmup, dist, sampler)
    del singles, cycle
    return ms, R


def depthwise_bench(cb, torch, case, mode, steps):
    g = torch.Generator(device="cuda").manual_seed(case.seed)
    co = case.C * case.mult
    x0 = torch.rand((case.N, case.C, case.H, case.W), device="cuda", generator=g) * 2 - 1
    w0 = torch.randn((co, case.KH, case.KW), device="cuda", generator=g) / math.sqrt(case.KH * case.KW)
    b0 = torch.randn((co,), device="cuda", generator=g) * math.sqrt(0.1)
    R = rotating_sets(case.bytes)
    xs = [x0.clone() for _ in range(R)]
    ys = [torch.empty((case.N, co, case.Ho, case.Wo), device="cuda") for _ in range(R)]
    fns = [(lambda i=i: cb.depthwise_fwd(xs[i], w0, b0, ys[i], case.stride, case.pad, case.dil, mode))
           for i in range(R)]
    singles, cycle = capture(fns)
    ms = time_graph_steps(singles, cycle, steps, max(3, steps // 10))
    return ms / steps, R


def dense_extra(cb, torch, case, steps):
    g = torch.Generator(device="cuda").manual_seed(case.seed)
    X = torch.randn((case.N, case.H, case.W, case.Cin), device="cuda", generator=g).to(torch.bfloat16)
    F = (torch.randn((case.K, case.K, case.Cin, case.Cout), device="cuda", generator=g)
         / math.sqrt(case.K * case.K * case.Cin)).to(torch.bfloat16)
    ms, R = dense_bench(cb, torch, case, X, F, steps, max(3, steps // 10))
    return ms / steps, R


def e2e_bench(cb, torch, case, Xh, Fh, steps, warmup):
    """Public API end to end: pinned host inputs -> device, convolution, output -> pinned host."""
    X = torch.empty(Xh.shape, dtype=Xh.dtype, device="cuda")
    F = torch.empty(Fh.shape, dtype=Fh.dtype, device="cuda")
    Y = torch.empty((case.N, case.Ho, case.Wo, case.Cout), dtype=Xh.dtype, device="cuda")
    Yh = torch.empty(Y.shape, dtype=Y.dtype, pin_memory=True)

    def step():
        X.copy_(Xh, non_blocking=True)
        F.copy_(Fh, non_blocking=True)
        cb.conv2d_nhwc_fwd(X, F, Y)
        Yh.copy_(Y, non_blocking=True)

    for _ in range(warmup):
        step()
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    h2d = Xh.numel() * Xh.element_size() + Fh.numel() * Fh.element_size()
    d2h = Yh.numel() * Yh.element_size()
    return ms, h2d, d2h


def cpu_baseline_dense(case, Xb, Fb, budget_s=12.0):
    """The oracle as it stands on this host: whole images until about budget_s of work."""
    import oracle
    X = workloads.bf16_to_f32(Xb)
    F = workloads.bf16_to_f32(Fb)
    per_image = case.flops / case.N
    done = 0
    t0 = time.perf_counter()
    n = 0
    while n < case.N and (time.perf_counter() - t0) < budget_s:
        oracle.conv2d_nhwc(X[n:n + 1], F)
        done += per_image
        n += 1
    dt = time.perf_counter() - t0
    return {"value": done / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} of {case.N} images of the workload, float64 seven-loop oracle, {dt:.1f} s"}


def run_ours(args, dist):
    import torch
    import cnn_convolution_nhwc_b200 as cb

    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    peaks, peaks_src = load_peaks()
    case = workloads.DenseCase(CASE.name, CASE.N, CASE.H, CASE.W, CASE.Cin, CASE.Cout, CASE.K, "bf16",
                               "normal", seed=dist.rank)
    Xb, Fb = workloads.dense_inputs(case)
    Xh = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).pin_memory()
    Fh = torch.from_numpy(Fb.view(np.int16)).view(torch.bfloat16).pin_memory()
    X0 = Xh.to(dev)
    F0 = Fh.to(dev)

    sampler = ClockSampler(dist.local_rank)
    ms, R = dense_bench(cb, torch, case, X0, F0, args.steps, args.warmup, dist, sampler)
    ms_step = ms / args.steps
    value = dist.world * case.flops * args.steps / (ms * 1e-3) / 1e12
    achieved = case.flops / (ms_step * 1e-3) / 1e12
    e2e_steps = max(10, min(200, args.steps // 10))
    e2e_ms, h2d, d2h = e2e_bench(cb, torch, case, Xh, Fh, e2e_steps, 3)
    e2e_ms = dist.max(e2e_ms)
    e2e_value = dist.world * case.flops / (e2e_ms * 1e-3) / 1e12
    status = cb.conv_device_status()

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 / Box-Muller: X~N(0,1), F~N(0,1/(K*K*Cin)), rounded to bf16)",
        "config": {"workload": CASE.name, "N_per_gpu": case.N, "H": case.H, "W": case.W, "Cin": case.Cin,
                   "Cout": case.Cout, "K": case.K, "flop_per_step": case.flops, "bytes_per_step": case.bytes,
                   "l2": f"inputs larger than L2: {R} rotating X/F/Y sets of {case.bytes / 1e6:.2f} MB",
                   "launch": "CUDA graph replay of the C-ABI call", "parallelism": f"replicas x{dist.world}"},
        "roofline": {"kernel": "dense_tc_kernel (BN=64)", "bound": "tensor", "achieved": round(achieved, 3),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "traffic": traffic_for("dense_tc_kernel", CASE.name),
                     "algorithmic_bytes": case.bytes,
                     "hbm_frac": round(case.bytes / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                     "peak_source": f"{peaks_src} (bf16 burst; HBM copy {peaks['hbm_gbs']} GB/s)"},
        "e2e": {"value": round(e2e_value, 4), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4), "path": "python binding -> C ABI, pinned host copies in the timed region"},
        "gpu_launches": args.steps,
        "clocks": sampler.summary(),
        "device_status": cb.conv_status_string(status),
    }
    if dist.world == 1 and not args.no_extras:
        line["extras"] = extras(cb, torch, peaks)
    if dist.rank == 0 and dist.world == 1:
        line["cpu_baseline"] = cpu_baseline_dense(case, Xb, Fb)
    return line


def extras(cb, torch, peaks):
    out = {"dense": [], "depthwise": []}
    for case in (workloads.DENSE_1X1, workloads.DENSE_LARGE):
        steps = 200 if case.flops < 1e11 else 40
        ms, R = dense_extra(cb, torch, case, steps)
        tf = case.flops / (ms * 1e-3) / 1e12
        out["dense"].append({"workload": case.name, "ms": round(ms, 5), "TFLOP/s": round(tf, 2),
                             "frac_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
                             "GB/s": round(case.bytes / (ms * 1e-3) / 1e9, 1),
                             "frac_hbm": round(case.bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                             "rotating_sets": R})
    for case in workloads.DW_SWEEP:
        for mode, name in ((0, "exact"), (1, "fast")):
            ms, R = depthwise_bench(cb, torch, case, mode, 200)
            gbs = case.bytes / (ms * 1e-3) / 1e9
            out["depthwise"].append({"workload": case.name, "mode": name, "ms": round(ms, 5),
                                     "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                     "GFLOP/s": round(case.flops / (ms * 1e-3) / 1e9, 1), "rotating_sets": R})
    return out


# ------------------------------------------------------------------------------------------
# Reference arm: the CPU oracle
# ------------------------------------------------------------------------------------------
def run_reference(args, dist):
    import oracle
    case = CASE
    Xb, Fb = workloads.dense_inputs(case)
    X = workloads.bf16_to_f32(Xb)
    F = workloads.bf16_to_f32(Fb)
    total = case.N * case.Ho * case.Wo * case.Cout
    flop_per_out = 2 * case.K * case.K * case.Cin
    # calibrate: points per second of the oracle's per-output routine
    idx = (workloads.splitmix64(1, 4096) % np.uint64(total)).astype(np.int64)
    t0 = time.perf_counter()
    oracle.conv2d_nhwc_points(X, F, idx)
    rate = 4096 / max(1e-6, time.perf_counter() - t0)
    per_step = int(min(total, max(64, rate * 90.0 / max(1, args.steps + args.warmup))))
    samples = [(workloads.splitmix64(100 + s, per_step) % np.uint64(total)).astype(np.int64)
               for s in range(min(8, args.steps + args.warmup))]
    for s in range(args.warmup):
        oracle.conv2d_nhwc_points(X, F, samples[s % len(samples)])
    t0 = time.perf_counter()
    for s in range(args.steps):
        oracle.conv2d_nhwc_points(X, F, samples[s % len(samples)])
    dt = time.perf_counter() - t0
    ms = dt * 1e3 / args.steps
    value = per_step * flop_per_out / (dt / args.steps) / 1e12
    cores = oracle.num_threads()
    sample = (f"{per_step} sampled outputs of the workload per step (of {total}), float64 oracle, "
              f"OpenMP over outputs")
    return {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs as the GPU arm)",
        "config": {"workload": case.name, "N_per_gpu": case.N, "H": case.H, "W": case.W, "Cin": case.Cin,
                   "Cout": case.Cout, "K": case.K},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50000)
    ap.add_argument("--warmup", type=int, default=500)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    dist = Dist()
    if args.impl == "reference":
        if dist.rank != 0:
            return 0
        print(json.dumps(run_reference(args, dist)), flush=True)
        return 0
    import torch
    torch.cuda.set_device(dist.local_rank)
    dist.init("nccl")
    try:
        line = run_ours(args, dist)
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
