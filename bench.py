"""Benchmark: dense NHWC convolution (bf16, N=64, 112x112, 128->128, K=5) on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-extras]
                    [--workload NAME]

A step is one forward dense convolution over one batch of 64 images (the hot path: tensor
maps, TMA patch gather, tcgen05 mainloop, epilogue) with inputs resident in HBM; the default
workload is the largest dense configuration. Inputs and outputs rotate over enough buffer sets
that their total exceeds twice the L2 size, so every step reads cold data. The W warm-up steps
and then the K timed steps each run from CUDA graphs captured around the C-ABI call that hold
the steps back to back (one graph launch per 1000 steps), timed with CUDA events on the
launching stream, bracketed by a barrier and a device synchronisation; the reported time is
the maximum over ranks. Under torchrun every rank runs its own batch (weak scaling, no
collective on the data path).

Also reported: "e2e" -- the same metric through the public Python API with the inputs copied
from pinned host memory and the output copied back inside the timed region; "roofline" for
the timed kernel; "cpu_baseline" -- the CPU oracle timed on a bounded sample of the same
workload (rank 0, N=1); and, unless --no-extras, every other configuration (the dense 3x3 and
pointwise layers, the general-geometry, grouped and Conv1D layers, the depthwise sweep in both
modes, the fused depthwise-pointwise blocks) as one compact "extras" table at the end of the line.

--impl reference times the CPU oracle itself on the same workload (rank 0 only).
--workload selects another single configuration (for timing or profiling one kernel alone):
"dense3x3", "pointwise", ... or "dw-C<C>-K<K>-s<stride>-H<H>-exact|fast" from the depthwise sweep.
"""
from __future__ import annotations

import argparse
import dataclasses
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
DEFAULT_WORKLOAD = "dense-large"


def workload_table():
    """Name -> (kind, case, mode). The default headline is the large dense configuration; the
    others exist so any single kernel can be timed or profiled alone."""
    t = {"dense3x3": ("dense", workloads.DENSE_3X3, None),
         "pointwise": ("dense", workloads.DENSE_1X1, None),
         "dense-large": ("dense", workloads.DENSE_LARGE, None),
         "dense-s2": ("dense", workloads.DENSE_S2, None),
         "grouped": ("dense", workloads.DENSE_GROUPED, None),
         "conv1d-stem1": ("dense", workloads.CONV1D_STEM1, None),
         "conv1d-stem2": ("dense", workloads.CONV1D_STEM2, None),
         "conv1d-causal": ("dense", workloads.CONV1D_CAUSAL, None),
         # comparison path: explicit patch matrix + one cuBLAS GEMM, packing inside the timing
         "dense3x3-explicit-im2col": ("dense", workloads.DENSE_3X3, "im2col")}
    for c in workloads.DWPW_BLOCKS:
        for mode, name in ((0, "exact"), (1, "fast")):
            t[f"dwpw-C{c.C}-K{c.K}-H{c.H}-Cout{c.Cout}-{name}"] = ("dwpw", c, mode)
    for c in workloads.DW_SWEEP:
        for mode, name in ((0, "exact"), (1, "fast")):
            t[f"dw-C{c.C}-K{c.KH}-s{c.stride}-H{c.H}-{name}"] = ("depthwise", c, mode)
    return t


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        for k, v in FALLBACK_PEAKS.items():
            d.setdefault(k, v)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "dense_fold_kernel": ("dense_fold.cuh", "dense_halo.cuh", "dense_tc.cuh", "depthwise.cuh", "ptx.cuh"),
    "dense_halo_kernel": ("dense_halo.cuh", "ptx.cuh"),
    "dense_tc_kernel": ("dense_tc.cuh", "ptx.cuh"),
    "dense_stream_kernel": ("dense_stream.cuh", "dense_halo.cuh", "ptx.cuh"),
    "dense_halo_pad_kernel": ("dense_halo_pad.cuh", "dense_halo.cuh", "ptx.cuh"),
    "dense_direct_kernel": ("dense_direct.cuh",),
    "depthwise_tma_kernel": ("depthwise_tma.cuh", "depthwise.cuh", "ptx.cuh"),
    "depthwise_reg_kernel": ("depthwise_reg.cuh", "depthwise.cuh"),
    "depthwise_kernel": ("depthwise.cuh",),
    "dwpw_kernel": ("dwpw.cuh", "dense_tc.cuh", "depthwise.cuh", "ptx.cuh"),
    "dwpw_staged_kernel": ("dwpw.cuh", "dense_tc.cuh", "depthwise.cuh", "ptx.cuh"),
    "dwpw_gemm_kernel": ("dwpw_gemm.cuh", "depthwise_tma.cuh", "depthwise_plane.cuh", "depthwise.cuh", "dense_halo.cuh",
                         "ptx.cuh"),
    "depthwise_plane_kernel": ("depthwise_plane.cuh", "depthwise_tma.cuh", "depthwise.cuh", "ptx.cuh"),
}


def source_hash(kernel: str) -> str:
    """Hash of the source files that define a kernel (its DRAM counters go stale with them)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "cnn_convolution_nhwc_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current sources:
    (read + write, read, write during the launch, note) or Nones."""
    none = (None, None, None, None)
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p) or kernel not in KERNEL_SOURCES:
        return none
    with open(p) as f:
        d = json.load(f)
    rec = d.get(kernel, {}).get(workload)
    if not rec or rec.get("source_hash") != source_hash(kernel):
        return none
    return rec.get("bytes_per_launch"), rec.get("read"), rec.get("write"), rec.get("note")


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


CHUNK = 1000   # launches per captured graph (longer runs replay it; one graph launch per CHUNK steps)


class StepGraphs:
    """CUDA graphs that launch exactly `n` C-ABI calls back to back on the current stream,
    cycling over the rotating buffer sets: one graph of `chunk` calls (a multiple of the number
    of sets, at most CHUNK) replayed n // chunk times, then one graph of the remaining calls.
    The calls inside a graph follow each other with no host gap."""

    def __init__(self, fns, n):
        import torch
        R = len(fns)
        chunk = min(n, CHUNK)
        if chunk >= R:
            chunk -= chunk % R
        self.q, r = divmod(n, chunk) if chunk else (0, 0)
        self.main = self._graph(torch, fns, chunk) if chunk else None
        self.tail = self._graph(torch, fns, r) if r else None

    @staticmethod
    def _graph(torch, fns, count):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(count):
                fns[i % len(fns)]()
        return g

    def replay(self):
        for _ in range(self.q):
            self.main.replay()
        if self.tail is not None:
            self.tail.replay()


def eager_first_calls(fns):
    """Each call once, eagerly and off any capture: the first call of a kernel sets its
    shared-memory attribute and may query cluster occupancy, which stream capture forbids."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for fn in fns:
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()


def time_graph_steps(fns, steps: int, warmup: int, dist=None, sampler=None):
    """Runs `warmup` untimed steps, then exactly `steps` timed steps from one captured graph
    (see StepGraphs); returns the elapsed ms on the launching stream (max over ranks)."""
    import torch
    eager_first_calls(fns)
    warm = StepGraphs(fns, warmup)
    timed = StepGraphs(fns, steps)
    torch.cuda.synchronize()
    warm.replay()
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.start()
    start.record(stream)
    timed.replay()
    end.record(stream)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.stop()
    if dist is not None:
        dist.barrier()
    ms = start.elapsed_time(end)
    del warm, timed
    return dist.max(ms) if dist is not None else ms


# ------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------
def dense_device_inputs(torch, case, seed):
    """Seeded bf16 X, F (and the float32 bias, if the case has one) generated on the device
    (for the secondary measurements)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    X = torch.randn((case.N, case.H, case.W, case.Cin), device="cuda", generator=g).to(torch.bfloat16)
    F = (torch.randn(case.f_shape, device="cuda", generator=g)
         / math.sqrt(case.kh * case.kw * case.cin_g)).to(torch.bfloat16)
    b = torch.randn((case.Cout,), device="cuda", generator=g) * math.sqrt(0.1) if case.bias else None
    return X, F, b


def dense_plain(case):
    return case.square and case.stride == 1 and case.pad == 0 and case.dil == 1 and not case.bias


def dense_call(cb, case, X, F, b, Y, mode=None, ws=None):
    """The public entry a user calls for this case: the plain one, the one with stride,
    padding, dilation and bias, or (mode "im2col") the explicit-im2col comparison path."""
    if mode == "im2col":
        return cb.conv2d_nhwc_fwd_im2col(X, F, Y, workspace=ws)
    if dense_plain(case):
        return cb.conv2d_nhwc_fwd(X, F, Y)
    if case.square:
        return cb.conv2d_nhwc_fwd_ex(X, F, b, Y, case.stride, case.pad, case.dil)
    return cb.conv2d_nhwc_fwd_grouped(X, F, b, Y, (case.stride, case.sw), case.pads, (case.dil, case.dw),
                                      case.groups)


def oracle_dense(oracle, case, X, F, b):
    """The oracle entry for a dense case (whole images of X)."""
    if dense_plain(case):
        return oracle.conv2d_nhwc(X, F)
    if case.square:
        return oracle.conv2d_nhwc_ex(X, F, b, case.stride, case.pad, case.dil)
    return oracle.conv2d_grouped(X, F, b, (case.stride, case.sw), case.pads, (case.dil, case.dw), case.groups)


def im2col_workspace(cb, torch, case, mode):
    if mode != "im2col":
        return None
    return torch.empty(cb.lib.conv2d_nhwc_im2col_workspace(case.N, case.H, case.W, case.Cin, case.K),
                       dtype=torch.uint8, device="cuda")


def dw_device_inputs(torch, case, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    co = case.C * case.mult
    x = torch.rand((case.N, case.C, case.H, case.W), device="cuda", generator=g) * 2 - 1
    w = torch.randn((co, case.KH, case.KW), device="cuda", generator=g) / math.sqrt(case.KH * case.KW)
    b = torch.randn((co,), device="cuda", generator=g) * math.sqrt(0.1)
    return x, w, b


def dwpw_device_inputs(torch, case, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.rand((case.N, case.C, case.H, case.W), device="cuda", generator=g) * 2 - 1
    w = torch.randn((case.C, case.K, case.K), device="cuda", generator=g) / case.K
    F = (torch.randn((case.C, case.Cout), device="cuda", generator=g) / math.sqrt(case.C)).to(torch.bfloat16)
    bd = torch.randn((case.C,), device="cuda", generator=g) * math.sqrt(0.1) if case.bias else None
    bp = torch.randn((case.Cout,), device="cuda", generator=g) * math.sqrt(0.1) if case.bias else None
    return x, w, bd, F, bp


def device_inputs(torch, kind, case, seed):
    if kind == "dense":
        return dense_device_inputs(torch, case, seed)
    if kind == "dwpw":
        return dwpw_device_inputs(torch, case, seed)
    return dw_device_inputs(torch, case, seed)


def out_shape(kind, case):
    if kind == "dense":
        return (case.N, case.Ho, case.Wo, case.Cout)
    if kind == "dwpw":
        return (case.N, case.Cout, case.Ho, case.Wo)
    return (case.N, case.C * case.mult, case.Ho, case.Wo)


def dwpw_call(cb, case, x, w, bd, F, bp, y, mode):
    return cb.dwpw_fwd(x, w, bd, F, bp, y, case.stride, case.pad, case.dil, mode)


def steps_fns(cb, torch, kind, case, mode, inputs):
    """R rotating buffer sets (total at least twice the L2) and one C-ABI call per set."""
    R = rotating_sets(case.bytes)
    if kind == "dense":
        X0, F0, b0 = inputs
        Xs = [X0.clone() for _ in range(R)]
        Fs = [F0.clone() for _ in range(R)]
        Ys = [torch.empty((case.N, case.Ho, case.Wo, case.Cout), dtype=X0.dtype, device=X0.device)
              for _ in range(R)]
        ws = im2col_workspace(cb, torch, case, mode)
        fns = [(lambda i=i: dense_call(cb, case, Xs[i], Fs[i], b0, Ys[i], mode, ws)) for i in range(R)]
        keep = (Xs, Fs, Ys, b0, ws)
    elif kind == "dwpw":
        x0, w0, bd0, F0, bp0 = inputs
        xs = [x0.clone() for _ in range(R)]
        ys = [torch.empty(out_shape(kind, case), device=x0.device) for _ in range(R)]
        fns = [(lambda i=i: dwpw_call(cb, case, xs[i], w0, bd0, F0, bp0, ys[i], mode)) for i in range(R)]
        keep = (xs, ys)
    else:
        x0, w0, b0 = inputs
        xs = [x0.clone() for _ in range(R)]
        ys = [torch.empty((case.N, case.C * case.mult, case.Ho, case.Wo), device=x0.device) for _ in range(R)]
        fns = [(lambda i=i: cb.depthwise_fwd(xs[i], w0, b0, ys[i], case.stride, case.pad, case.dil, mode))
               for i in range(R)]
        keep = (xs, ys)
    return fns, R, keep


def time_case(cb, torch, kind, case, mode, inputs, steps, warmup, dist=None, sampler=None):
    fns, R, keep = steps_fns(cb, torch, kind, case, mode, inputs)
    ms = time_graph_steps(fns, steps, warmup, dist, sampler)
    kernel = cb.conv_last_kernel()      # the dispatcher's choice for this workload
    del keep
    return ms, R, kernel


E2E_SETS = 2   # device buffer sets of the end-to-end pipeline


def e2e_bench(cb, torch, kind, case, mode, host, steps, warmup):
    """Public API end to end: every step copies its inputs from pinned host memory to the
    device, runs the convolution and copies its output back to pinned host memory. The copies
    in and out and the convolution run on three streams over E2E_SETS device buffer sets,
    ordered by events (a set's inputs are rewritten only after the convolution that read them,
    its output only after the copy that read it), so step i+1's upload overlaps step i's
    download as in a serving loop; the timed region spans the first upload to the last
    download."""
    def dev_set():
        d = [torch.empty(h.shape, dtype=h.dtype, device="cuda") if h is not None else None for h in host]
        if kind == "dense":
            o = torch.empty(out_shape(kind, case), dtype=host[0].dtype, device="cuda")
        else:
            o = torch.empty(out_shape(kind, case), device="cuda")
        w = im2col_workspace(cb, torch, case, mode) if kind == "dense" else None
        return d, o, w

    sets = [dev_set() for _ in range(E2E_SETS)]
    out_h = torch.empty(sets[0][1].shape, dtype=sets[0][1].dtype, pin_memory=True)
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: [torch.cuda.Event() for _ in range(E2E_SETS)]   # noqa: E731
    ev_in, ev_cmp, ev_out = ev(), ev(), ev()

    def step(i):
        k = i % E2E_SETS
        dev, out, ws = sets[k]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[k])          # the convolution that read this set is done
            for d, h in zip(dev, host):
                if h is not None:
                    d.copy_(h, non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[k])
            s_cmp.wait_event(ev_out[k])         # this set's previous output has been copied out
            if kind == "dense":
                dense_call(cb, case, dev[0], dev[1], dev[2], out, mode, ws)
            elif kind == "dwpw":
                dwpw_call(cb, case, dev[0], dev[1], dev[2], dev[3], dev[4], out, mode)
            else:
                cb.depthwise_fwd(dev[0], dev[1], dev[2], out, case.stride, case.pad, case.dil, mode)
            ev_cmp[k].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[k])
            out_h.copy_(out, non_blocking=True)
            ev_out[k].record(s_out)

    main = torch.cuda.current_stream()
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(main)
    for st in (s_in, s_cmp, s_out):
        st.wait_stream(main)
    for i in range(steps):
        step(i)
    for st in (s_in, s_cmp, s_out):
        main.wait_stream(st)
    end.record(main)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    h2d = sum(h.numel() * h.element_size() for h in host if h is not None)
    d2h = out_h.numel() * out_h.element_size()
    return ms, h2d, d2h


def cpu_baseline(kind, case, mode, host_np, budget_s=10.0):
    """The oracle as it stands on this host: whole images, cycling through the batch, until
    about budget_s of work."""
    import oracle
    done = 0.0
    n = 0
    t0 = time.perf_counter()
    while (time.perf_counter() - t0) < budget_s:
        i = n % case.N
        if kind == "dense":
            X, F, b = host_np
            oracle_dense(oracle, case, X[i:i + 1], F, b)
            done += case.flops / case.N
        elif kind == "dwpw":
            x, w, bd, F, bp = host_np
            oracle.dwpw(x[i:i + 1], w, bd, F, bp, case.stride, case.pad, case.dil, mode)
            done += case.bytes / case.N
        else:
            x, w, b = host_np
            oracle.depthwise(x[i:i + 1], w, b, mult=case.mult, stride=case.stride, pad=case.pad, dil=case.dil,
                             mode=mode)
            done += case.bytes / case.N
        n += 1
    dt = time.perf_counter() - t0
    unit = "TFLOP/s" if kind == "dense" else "GB/s"
    scale = 1e12 if kind == "dense" else 1e9
    if kind == "dense":
        what = "float64 seven-loop oracle"
    elif kind == "dwpw":
        what = f"float32 depthwise oracle ({'exact' if mode == 0 else 'fast'} mode) + float64 pointwise"
    else:
        what = f"float32 per-output oracle, {'exact' if mode == 0 else 'fast'} mode"
    return {"value": done / dt / scale, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} single-image calls cycling over the {case.N} images of the workload, {what}, {dt:.1f} s"}


def host_inputs(torch, kind, case, seed):
    """Seeded host inputs from the workloads generators, as numpy (oracle view) and pinned torch."""
    if kind == "dense":
        c = dataclasses.replace(case, seed=seed)
        Xb, Fb = workloads.dense_inputs(c)
        b = workloads.dense_bias(c)
        host = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in (Xb, Fb)]
        host.append(None if b is None else torch.from_numpy(b).pin_memory())
        return (workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb), b), host
    if kind == "dwpw":
        x, w, bd, F, bp = workloads.dwpw_inputs(dataclasses.replace(case, seed=seed))
        host = [torch.from_numpy(x).pin_memory(), torch.from_numpy(w).pin_memory(),
                None if bd is None else torch.from_numpy(bd).pin_memory(),
                torch.from_numpy(F.view(np.int16)).view(torch.bfloat16).pin_memory(),
                None if bp is None else torch.from_numpy(bp).pin_memory()]
        return (x, w, bd, workloads.bf16_to_f32(F), bp), host
    c = workloads.DepthwiseCase(case.name, case.N, case.C, case.mult, case.H, case.W, case.KH, case.KW, case.stride,
                                case.pad, case.dil, case.bias, seed)
    x, w, b = workloads.depthwise_inputs(c)
    host = [torch.from_numpy(a).pin_memory() for a in (x, w, b)]
    return (x, w, b), host


def run_ours(args, dist):
    import torch
    import cnn_convolution_nhwc_b200 as cb

    kind, case, mode = workload_table()[args.workload]
    torch.cuda.set_device(dist.local_rank)
    peaks, peaks_src = load_peaks()
    host_np, host = host_inputs(torch, kind, case, seed=dist.rank)
    dev_inputs = tuple(None if h is None else h.to("cuda") for h in host)

    sampler = ClockSampler(dist.local_rank)
    ms, R, kernel = time_case(cb, torch, kind, case, mode, dev_inputs, args.steps, args.warmup, dist, sampler)
    ms_step = ms / args.steps
    e2e_steps = max(10, min(200, args.steps // 10))
    e2e_ms, h2d, d2h = e2e_bench(cb, torch, kind, case, mode, host, e2e_steps, 3)
    e2e_ms = dist.max(e2e_ms)
    status = cb.conv_device_status()

    if kind == "dense":
        unit, work, scale = "TFLOP/s", case.flops, 1e12
        achieved = case.flops / (ms_step * 1e-3) / 1e12
        roof = {"kernel": kernel, "bound": "tensor", "achieved": round(achieved, 3), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                **traffic_fields(kernel, args.workload), "algorithmic_bytes": case.bytes,
                "algorithmic_flops": case.flops,
                "hbm_frac": round(case.bytes / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                # a timed region of ~100 ms of back-to-back dense launches can reach the 1 kW power
                # cap (sw_power_cap in "clocks"): the fraction of the sustained GEMM figure too
                "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                "peak_source": f"{peaks_src}: frac of the bf16 burst figure ({peaks['bf16_tflops']}), "
                               f"frac_of_sustained of the seconds-long figure ({peaks['bf16_tflops_sustained']}); "
                               f"HBM copy {peaks['hbm_gbs']} GB/s"}
        dtype = "bf16"
        data = "synthetic (seeded SplitMix64 / Box-Muller: X~N(0,1), F~N(0,1/(K*K*Cin)), rounded to bf16)"
        cfg = {"workload": case.name, "N_per_gpu": case.N, "H": case.H, "W": case.W, "Cin": case.Cin,
               "Cout": case.Cout, "K": case.K, "stride": case.stride, "pad": case.pad, "dil": case.dil,
               "bias": case.bias, "flop_per_step": case.flops, "bytes_per_step": case.bytes}
        if not case.square:
            cfg.update({"KH": case.kh, "KW": case.kw, "stride_w": case.sw, "pad_w": case.pw, "pad_w_end": case.pwe,
                        "dil_w": case.dw,
                        "groups": case.groups})
        # the explicit patch matrix the implicit kernels never build (N*Ho*Wo rows by
        # KH*KW*Cin/groups bf16 columns per group) and its size over the input's
        patch = 2 * case.N * case.Ho * case.Wo * case.kh * case.kw * case.Cin
        cfg["patch_matrix_bytes_avoided"] = patch if mode != "im2col" else 0
        cfg["patch_matrix_expansion"] = round(patch / (2 * case.N * case.H * case.W * case.Cin), 3)
        if mode == "im2col":
            cfg["path"] = "explicit patch matrix in a workspace + one cuBLAS GEMM (comparison path)"
    else:
        unit, work, scale = "GB/s", case.bytes, 1e9
        achieved = case.bytes / (ms_step * 1e-3) / 1e9
        roof = {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                **traffic_fields(kernel, args.workload), "algorithmic_bytes": case.bytes,
                "GFLOP/s": round(case.flops / (ms_step * 1e-3) / 1e9, 1),
                "peak_source": f"{peaks_src}: HBM copy"}
        dtype = "f32"
        data = "synthetic (seeded SplitMix64 / Box-Muller: x~U(-1,1), w~N(0,1/K^2), bias~N(0,0.1))"
        if kind == "dwpw":
            data = ("synthetic (seeded SplitMix64 / Box-Muller: x~U(-1,1), w~N(0,1/K^2), F~N(0,1/C) rounded to bf16, "
                    "biases~N(0,0.1))")
            cfg = {"workload": case.name + (" exact" if mode == 0 else " fast"), "N_per_gpu": case.N, "C": case.C,
                   "H": case.H, "W": case.W, "K": case.K, "stride": case.stride, "pad": case.pad, "dil": case.dil,
                   "Cout": case.Cout, "flop_per_step": case.flops, "bytes_per_step": case.bytes,
                   "intermediate": "depthwise output rounded to bf16 in shared memory, never in HBM"}
        else:
            cfg = {"workload": case.name + (" exact" if mode == 0 else " fast"), "N_per_gpu": case.N, "C": case.C,
                   "mult": case.mult, "H": case.H, "W": case.W, "K": case.KH, "stride": case.stride,
                   "pad": case.pad, "dil": case.dil, "flop_per_step": case.flops, "bytes_per_step": case.bytes}
    cfg.update({"l2": f"inputs larger than L2: {R} rotating buffer sets of {case.bytes / 1e6:.2f} MB",
                "launch": "CUDA graphs of the C-ABI call, the timed steps back to back (one graph launch per "
                          f"{CHUNK} steps)", "parallelism": f"replicas x{dist.world}"})
    value = dist.world * work * args.steps / (ms * 1e-3) / scale
    e2e_value = dist.world * work / (e2e_ms * 1e-3) / scale
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": unit, "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": data,
        "config": cfg, "roofline": roof,
        "e2e": {"value": round(e2e_value, 4), "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4),
                "path": "python binding -> C ABI, pinned host copies in the timed region; uploads, "
                        f"convolutions and downloads on three streams over {E2E_SETS} device buffer sets "
                        "(step i+1's upload overlaps step i's download)"},
        "gpu_launches": args.steps,   # one library kernel per step (the comparison path adds a cuBLAS GEMM)
        "clocks": sampler.summary(),
        "device_status": cb.conv_status_string(status),
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(kind, case, mode, host_np)
    if dist.world == 1 and not args.no_extras:
        # last, so that the end of the line (what a log tail keeps) holds every row
        line["extras_format"] = ("workload: [kernel, us per launch, fraction of the bound's measured peak "
                                 "(dense: bf16 burst TFLOP/s; depthwise and fused blocks: HBM GB/s), "
                                 "dense only: fraction of HBM]")
        line["extras"] = extras(cb, torch, peaks, skip=args.workload)
    return line


def traffic_fields(kernel, workload):
    """roofline.traffic (DRAM read + write of one launch, from the committed ncu summary taken on
    the current sources, else null) and its parts. Output lines still in L2 when the kernel ends
    are written to DRAM after it, so the write part can be below the output's size."""
    total, read, write, note = traffic_for(kernel, workload)
    out = {"traffic": total, "traffic_dram_read": read, "traffic_dram_write_in_launch": write}
    if note:
        out["traffic_note"] = note
    return out


def extras(cb, torch, peaks, skip):
    """Every other workload, timed like the headline; one short row each (see extras_format)."""
    out = {}
    for name, (kind, case, mode) in workload_table().items():
        if name == skip:
            continue
        steps = 200 if case.flops < 1e11 else 40
        inputs = dense_device_inputs(torch, case, 0) if kind == "dense" else device_inputs(torch, kind, case, 0)
        ms, R, kernel = time_case(cb, torch, kind, case, mode, inputs, steps, 10)
        ms /= steps
        short = kernel.replace("_kernel", "")
        gbs = case.bytes / (ms * 1e-3) / 1e9
        if kind == "dense":
            tf = case.flops / (ms * 1e-3) / 1e12
            out[name] = [short, round(ms * 1e3, 2), round(tf / peaks["bf16_tflops"], 3), round(gbs / peaks["hbm_gbs"], 3)]
        else:
            out[name] = [short, round(ms * 1e3, 2), round(gbs / peaks["hbm_gbs"], 3)]
    return out


# ------------------------------------------------------------------------------------------
# Reference arm: the CPU oracle, as it stands, on the host cores
# ------------------------------------------------------------------------------------------
def run_reference(args, dist):
    import oracle
    kind, case, mode = workload_table()[args.workload]
    if kind == "dense":
        Xb, Fb = workloads.dense_inputs(case)
        X, F = workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb)
        b = workloads.dense_bias(case)
        total = case.N * case.Ho * case.Wo * case.Cout
        work_per_out, unit, scale = 2 * case.kh * case.kw * case.cin_g, "TFLOP/s", 1e12

        def run(idx):
            if dense_plain(case):
                oracle.conv2d_nhwc_points(X, F, idx)
            elif case.square:
                oracle.conv2d_nhwc_ex_points(X, F, idx, b, case.stride, case.pad, case.dil)
            else:
                oracle.conv2d_grouped_points(X, F, idx, b, (case.stride, case.sw), case.pads, (case.dil, case.dw),
                                             case.groups)
    elif kind == "dwpw":
        x, w, bd, Fb, bp = workloads.dwpw_inputs(case)
        F = workloads.bf16_to_f32(Fb)
        total = case.N * case.Cout * case.Ho * case.Wo
        work_per_out, unit, scale = case.bytes / total, "GB/s", 1e9

        def run(idx):
            oracle.dwpw_points(x, w, bd, F, bp, idx, case.stride, case.pad, case.dil, mode)
    else:
        x, w, b = workloads.depthwise_inputs(case)
        total = case.N * case.C * case.mult * case.Ho * case.Wo
        work_per_out, unit, scale = case.bytes / total, "GB/s", 1e9

        def run(idx):
            oracle.depthwise_points(x, w, b, idx, mult=case.mult, stride=case.stride, pad=case.pad, dil=case.dil,
                                    mode=mode)
    idx = (workloads.splitmix64(1, 4096) % np.uint64(total)).astype(np.int64)
    t0 = time.perf_counter()
    run(idx)
    rate = 4096 / max(1e-6, time.perf_counter() - t0)
    per_step = int(min(total, max(64, rate * 90.0 / max(1, args.steps + args.warmup))))
    samples = [(workloads.splitmix64(100 + s, per_step) % np.uint64(total)).astype(np.int64) for s in range(8)]
    for s in range(args.warmup):
        run(samples[s % 8])
    t0 = time.perf_counter()
    for s in range(args.steps):
        run(samples[s % 8])
    dt = time.perf_counter() - t0
    value = per_step * work_per_out / (dt / args.steps) / scale
    sample = f"{per_step} sampled outputs of the workload per step (of {total}), oracle per-output routine"
    return {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64" if kind == "dense" else "f32",
        "data": "synthetic (same seeded inputs as the GPU arm)",
        "config": {"workload": case.name if kind == "dense" else args.workload},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workload_table()))
    ap.add_argument("--no-extras", action="store_true")
    # profiling runs (ncu captures of one workload) skip the seconds-long CPU oracle sample
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
