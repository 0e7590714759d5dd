"""Benchmark of the B200 ConvTranspose library: one JSON line on rank 0.

A step is one ``ct_run`` of the headline workload (2-D decoder upsample,
fp16, X[8,256,64,64] * W[256,128,4,4], stride 2, pads 1 -> Y[8,128,128,128])
with X resident in HBM: plan, output-size resolution and the weight pre-pack
happen once, before timing, as they do for a deployed layer.  The metric is
effective TFLOP/s = 2*N*C*(M/group)*prod(in)*prod(k) / time, summed over
ranks.  Steps are CUDA-graph launches of one ct_run each, rotating over
enough X/Y buffer sets that consecutive steps do not hit L2 (more bytes than
the L2 holds between reuses).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank takes its own workload-sized slice of the global
batch (weak scaling: images are independent, no collective on the data
path); the reported time is the max over ranks.  ``--impl reference`` times the fp64
CPU oracle on a bounded sample of the same workload instead.
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from transposed_convolution_02_b200 import ct  # noqa: E402
from transposed_convolution_02_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

HEADLINE = 2
METRIC = "ConvTranspose effective TFLOP/s per config at 1 B200; % of tensor/HBM roofline"


# ---------------------------------------------------------------------------
# workload arithmetic used for reporting

def workload_numbers(wl):
    """Effective FLOP per pass and algorithmic bytes (X + W + bias + Y once)."""
    n, c = wl.x_shape[0], wl.x_shape[1]
    mg = wl.w_shape[1]
    flop = 2 * n * c * mg * math.prod(wl.x_shape[2:]) * math.prod(wl.w_shape[2:])
    eb = torch.finfo(wl.dtype).bits // 8
    m = mg * wl.group
    nbytes = eb * (math.prod(wl.x_shape) + math.prod(wl.w_shape) + (m if wl.bias else 0)
                   + math.prod(wl.y_shape))
    return flop, nbytes


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return dict(hbm_gbs=pk["hbm_gbs"], tc_tflops=pk["bf16_tflops"],
                    tc_tflops_sustained=pk.get("bf16_tflops_sustained"),
                    sm_max_mhz=pk.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, tc_tflops=1590.0, tc_tflops_sustained=1400.0,
                sm_max_mhz=1965.0, source="fallback")


# Nominal dense TF32 : BF16 tensor rates of a B200 (1.1 : 2.25 PFLOP/s): the
# TF32 peak is the measured BF16 peak times this ratio.
TF32_PER_BF16 = 1.1 / 2.25


def roofline_for(wl, seconds_per_launch, peaks, sms, kernel=None):
    """Bound and achieved rate of the workload's dominant kernel."""
    flop, nbytes = workload_numbers(wl)
    if wl.dtype == torch.float32 and kernel == "dense_tc_pair":
        # 3xTF32 on the tensor cores: three TF32 MMAs per fp32 product, so the
        # algorithmic fp32 rate is bounded by a third of the TF32 peak
        peak = peaks["tc_tflops"] * TF32_PER_BF16 / 3
        a = flop / seconds_per_launch / 1e12
        return dict(bound="tensor", achieved=a, peak=peak, unit="TFLOP/s", frac=a / peak,
                    peak_note="3xTF32: measured bf16 peak x %.3f (nominal TF32/BF16) / 3" % TF32_PER_BF16)
    if wl.dtype == torch.float32:
        # FP32 FFMA peak: SMs x 128 lanes x 2 flop x max SM clock
        peak = sms * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
        return dict(bound="alu", achieved=flop / seconds_per_launch / 1e12, peak=peak,
                    unit="TFLOP/s", frac=(flop / seconds_per_launch / 1e12) / peak)
    t_tc = flop / (peaks["tc_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    # both fractions, whichever bounds: the fp16 targets are stated against
    # the tensor peak even where HBM is the binding resource
    both = dict(tensor_frac=flop / seconds_per_launch / 1e12 / peaks["tc_tflops"],
                hbm_frac=nbytes / seconds_per_launch / 1e9 / peaks["hbm_gbs"])
    if t_tc >= t_hbm:
        a = flop / seconds_per_launch / 1e12
        return dict(bound="tensor", achieved=a, peak=peaks["tc_tflops"], unit="TFLOP/s",
                    frac=a / peaks["tc_tflops"], **both)
    a = nbytes / seconds_per_launch / 1e9
    return dict(bound="hbm", achieved=a, peak=peaks["hbm_gbs"], unit="GB/s",
                frac=a / peaks["hbm_gbs"], **both)


def profile_record(wid, kernel):
    """The committed ncu record of the workload's dominant kernel (DRAM bytes
    per launch, its share of one call), if that kernel's source is unchanged
    since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(str(wid))
    if not rec or rec.get("kernel") != kernel:
        return None
    src = os.path.join(ROOT, "transposed_convolution_02_b200", "csrc", rec["source"])
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return rec if h == rec["sha256_16"] else None


def traffic_for(wid, kernel):
    rec = profile_record(wid, kernel)
    return rec["bytes_per_launch"] if rec else None


def annotate_roofline(roof, wid, kernel, launches, call_seconds=None, flop=None, nbytes=None):
    """Scope and provenance of the roofline figures.  `achieved` and `frac`
    are the dominant kernel's, timed alone (CUDA events over launches of that
    kernel only); the whole call (all of its launches) is given beside it.
    `traffic` is DRAM read + write bytes of one steady-state launch from the
    committed ncu record, while the kernel source still matches it."""
    rec = profile_record(wid, kernel)
    roof["traffic"] = rec["bytes_per_launch"] if rec else None
    if rec:
        roof["traffic_detail"] = {k: rec[k] for k in ("dram_read", "dram_write", "l2_write_from_sm",
                                                       "capture") if k in rec}
        if nbytes:
            roof["traffic_over_algorithmic"] = rec["bytes_per_launch"] / nbytes
    roof["kernel"] = kernel
    roof["scope"] = ("dominant kernel alone, CUDA events; the call is %d launch%s"
                     % (launches, "" if launches == 1 else "es"))
    if call_seconds is not None:
        roof["call_us"] = call_seconds * 1e6
        roof["call_frac"] = roof["frac"] * roof["kernel_us"] / roof["call_us"] \
            if roof.get("kernel_us") else None
    return roof


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)

class ClockSampler:
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = device_index
            if vis:
                ids = [v for v in vis.split(",") if v.strip()]
                if device_index < len(ids) and ids[device_index].strip().isdigit():
                    idx = int(ids[device_index])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# our arm

def build_op(wl, device):
    x, w, b = make_inputs(wl)
    op = ct.ConvTranspose(w.to(device), list(x.shape), b.to(device) if b is not None else None,
                          strides=wl.strides, dilations=wl.dilations, pads=wl.pads,
                          output_padding=wl.output_padding, auto_pad=wl.auto_pad,
                          group=wl.group)
    return op, x


def _graph_set(op, xs, ys, parts):
    """One CUDA graph per buffer set, each holding one call restricted to `parts`."""
    graphs = []
    for i in range(len(xs)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            op.run_part(xs[i], ys[i], parts)
        graphs.append(g)
    return graphs


def _replay_ms(graphs, steps, first, sampler=None):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        start.record()
        for j in range(steps):
            graphs[(first + j) % len(graphs)].replay()
        end.record()
        torch.cuda.synchronize()
    return start.elapsed_time(end)


def time_device(wl, device, steps, warmup, l2_bytes, dist_max=None, sampler=None, kernel_steps=None):
    """Device time of `steps` ct_runs (CUDA graphs, rotating buffer sets),
    then of `kernel_steps` launches of the call's main kernel alone (the
    preparation launches replayed once before, so its workspace is in place)
    and of the preparation alone.  Returns (ms for `steps` calls, info)."""
    op, x_cpu = build_op(wl, device)
    xb = x_cpu.numel() * x_cpu.element_size()
    yb = math.prod(op.y_shape) * x_cpu.element_size()
    nsets = max(2, min(8, math.ceil(2 * l2_bytes / (xb + yb)) + 1))
    free, _ = torch.cuda.mem_get_info(device)
    while nsets > 1 and nsets * (xb + yb) > 0.6 * free:
        nsets -= 1
    xs = [x_cpu.to(device) for _ in range(nsets)]
    ys = [torch.empty(op.y_shape, dtype=wl.dtype, device=device) for _ in range(nsets)]
    s = torch.cuda.Stream(device)
    s.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(s):
        for i in range(nsets):       # warm the launch path before capture
            op(xs[i], out=ys[i])
    torch.cuda.current_stream(device).wait_stream(s)
    torch.cuda.synchronize(device)
    graphs = _graph_set(op, xs, ys, ct.PART_ALL)
    for j in range(warmup):
        graphs[j % nsets].replay()
    if dist_max is not None:
        dist_max("barrier")
    torch.cuda.synchronize(device)
    ms = _replay_ms(graphs, steps, warmup, sampler)
    if dist_max is not None:
        dist_max("barrier")
    info = dict(kernel=op.kernel, launches_per_step=op.launches, sets=nsets,
                set_bytes=xb + yb)
    del graphs
    # the main kernel alone, and the preparation alone (rank-local timings:
    # every rank runs the same steps, no collective in between)
    ksteps = kernel_steps if kernel_steps is not None else min(steps, 400)
    main = _graph_set(op, xs, ys, ct.PART_MAIN)
    for j in range(max(3, warmup // 4)):
        main[j % nsets].replay()
    torch.cuda.synchronize(device)
    info["kernel_ms_per_launch"] = _replay_ms(main, ksteps, 0) / ksteps
    del main
    if op.launches > 1:
        prep = _graph_set(op, xs, ys, ct.PART_PREPARE)
        for j in range(3):
            prep[j % nsets].replay()
        torch.cuda.synchronize(device)
        info["prepare_ms_per_call"] = _replay_ms(prep, ksteps, 0) / ksteps
        del prep
    else:
        info["prepare_ms_per_call"] = 0.0
    # leave Y as the full call writes it (the parts runs above overwrote it)
    for i in range(nsets):
        op(xs[i], out=ys[i])
    torch.cuda.synchronize(device)
    return ms, info


def kernel_roofline(wl, wid, info, call_seconds, peaks, sms):
    """The roofline object of a workload: the dominant (main) kernel timed
    alone against its bound, with the whole call beside it."""
    flop, nbytes = workload_numbers(wl)
    ksec = info["kernel_ms_per_launch"] / 1e3
    roof = roofline_for(wl, ksec, peaks, sms, info["kernel"])
    roof["peak_source"] = peaks["source"] + " (burst)"
    roof["kernel_us"] = ksec * 1e6
    roof["prepare_us"] = info["prepare_ms_per_call"] * 1e3
    call = roofline_for(wl, call_seconds, peaks, sms, info["kernel"])
    roof["call"] = {"us": call_seconds * 1e6, "achieved": call["achieved"], "frac": call["frac"],
                    "tensor_frac": call.get("tensor_frac"), "hbm_frac": call.get("hbm_frac")}
    roof["algorithmic"] = {"flop": flop, "bytes": nbytes}
    return annotate_roofline(roof, wid, info["kernel"], info["launches_per_step"], nbytes=nbytes)


def make_dist_max(dist, device=None):
    """Collective helpers over the default process group: a barrier, and the
    maximum of one float over all ranks (every rank takes the same steps)."""
    def dist_max(what, value=None):
        if what == "barrier":
            dist.barrier()
            return None
        t = torch.tensor([float(value)], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return dist_max


def aggregate(flop_per_replica, ms_local, steps, world, dist_max=None):
    """Whole-job rate of `world` independent replicas: every rank processed
    one replica per step, the job took the slowest rank's time.  Returns
    (ms for `steps` steps, TFLOP/s over all ranks)."""
    ms = dist_max("max", ms_local) if dist_max is not None else ms_local
    sec_per_step = ms / 1e3 / steps
    return ms, flop_per_replica * max(world, 1) / sec_per_step / 1e12


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def time_e2e(wl, device, steps, warmup):
    """Through the public API with host buffers: pinned X -> device, ct_run,
    Y -> pinned host, all inside the timed region every step.  Steps are
    pipelined the way a caller streaming batches would run them: copy-in,
    compute and copy-out each on their own stream with two buffer sets, so
    step i's input copy overlaps step i-1's compute and step i-2's output
    copy (PCIe carries both directions at once)."""
    op, x_cpu = build_op(wl, device)
    xh = x_cpu.pin_memory()
    yh = [torch.empty(op.y_shape, dtype=wl.dtype).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x_cpu, device=device) for _ in range(2)]
    yd = [torch.empty(op.y_shape, dtype=wl.dtype, device=device) for _ in range(2)]
    s_in, s_run, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def step(i):
        b = i & 1
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev_run[b])   # the compute that read xd[b] is done
            xd[b].copy_(xh, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[b])
            if used[b]:
                s_run.wait_event(ev_out[b])  # yd[b] has been copied out
            op(xd[b], out=yd[b], stream=s_run)
            ev_run[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[b])
            yh[b].copy_(yd[b], non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    main = torch.cuda.current_stream(device)
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(device)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(main)
    for st in (s_in, s_run, s_out):
        st.wait_event(start)
    for i in range(steps):
        step(warmup + i)
    for st in (s_in, s_run, s_out):
        main.wait_stream(st)
    end.record(main)
    torch.cuda.synchronize(device)
    return start.elapsed_time(end), xh.numel() * xh.element_size(), yh[0].numel() * yh[0].element_size()


# ---------------------------------------------------------------------------
# the oracle on the host cores (reported baseline / reference arm)

def oracle_sample(wl, target_s=12.0):
    """Time the fp64 oracle on a bounded sample of the workload.

    The sample is batch image 0, the first m' output channels of every group
    (m' = as many as there are cores, at most M/group: the oracle's threads
    split the work by output plane) and the first h' positions of the first
    spatial axis of X, h' sized from a one-row calibration run so the sample
    takes about ``target_s``.  Returns (TFLOP/s, cores, description, seconds).
    """
    from oracle import Attrs, conv_transpose_ref
    x, w, b = make_inputs(wl)
    x = x[:1].double().numpy()
    w = w.double().numpy()
    b = b.double().numpy() if b is not None else None
    g = wl.group
    mg_full = wl.w_shape[1]
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    mg = max(1, min(mg_full, math.ceil(cores / g)))
    ws = np.ascontiguousarray(w[:, :mg])
    bs = None
    if b is not None:
        bs = np.ascontiguousarray(b.reshape(g, mg_full)[:, :mg].reshape(-1))
    attrs = Attrs(strides=wl.strides, dilations=wl.dilations, pads=wl.pads,
                  output_padding=wl.output_padding, auto_pad=wl.auto_pad, group=g)
    rows = x.shape[2]

    def run(h):
        xs = np.ascontiguousarray(x[:, :, :h])
        t0 = time.perf_counter()
        conv_transpose_ref(xs, ws, bs, attrs)
        dt = time.perf_counter() - t0
        flop = 2 * xs.shape[1] * mg * math.prod(xs.shape[2:]) * math.prod(w.shape[2:])
        return dt, flop

    dt, flop = run(1)
    h = int(max(1, min(rows, round(target_s / max(dt, 1e-4)))))
    if h > 1:
        dt, flop = run(h)
    desc = ("batch image 0 of %d, %d of %d output channels per group, first %d of %d "
            "positions on the first spatial axis (%.3f GFLOP), %d OpenMP threads"
            % (wl.x_shape[0], mg, mg_full, h, rows, flop / 1e9, cores))
    return flop / dt / 1e12, cores, desc, dt


# ---------------------------------------------------------------------------

# Shapes beyond the five workloads: the stride-1 implicit GEMM (a 3x3
# convolution with tap-reversed weights), the 1x1 stride-1 GEMM, channels-last
# input, more than 256 output channels, 3 input channels, fp32 in 2-D.
GENERAL_SHAPES = [
    ("stride-1 3x3 fp16 X[8,256,64,64] W[256,256,3,3] p1", [8, 256, 64, 64], [256, 256, 3, 3],
     torch.float16, "nchw", dict(strides=[1, 1], pads=[1, 1, 1, 1])),
    ("1x1 stride-1 fp16 X[8,512,64,64] W[512,256,1,1]", [8, 512, 64, 64], [512, 256, 1, 1],
     torch.float16, "nchw", dict(strides=[1, 1])),
    ("channels-last decoder fp16 X[8,64,64,256] W[256,4,4,128] s2 p1", [8, 256, 64, 64], [256, 128, 4, 4],
     torch.float16, "nhwc", dict(strides=[2, 2], pads=[1, 1, 1, 1])),
    ("512-channel decoder fp16 X[8,256,32,32] W[256,512,4,4] s2 p1", [8, 256, 32, 32], [256, 512, 4, 4],
     torch.float16, "nchw", dict(strides=[2, 2], pads=[1, 1, 1, 1])),
    ("3-channel input fp16 X[16,3,128,128] W[3,64,4,4] s2 p1", [16, 3, 128, 128], [3, 64, 4, 4],
     torch.float16, "nchw", dict(strides=[2, 2], pads=[1, 1, 1, 1])),
    ("2-D fp32 decoder X[8,256,64,64] W[256,128,4,4] s2 p1", [8, 256, 64, 64], [256, 128, 4, 4],
     torch.float32, "nchw", dict(strides=[2, 2], pads=[1, 1, 1, 1])),
]


def general_shapes(device, peaks, runs=50, algos=("auto", "dense_tc", "dense_tc_pertap",
                                                  "dense_tc_pair", "generic"), only=None,
                   quiet=False):
    """Device time per call of each general shape under each algorithm that
    accepts it (CUDA events around a batch of calls, inputs rotated so the
    outputs exceed L2): kernel, effective TFLOP/s and the roofline of the
    binding resource (tensor peak for the dtype, 3xTF32 for fp32, or HBM for
    the algorithmic bytes X + W + bias + Y)."""
    torch.cuda.set_device(device)
    results = []
    for si, (name, xs, ws, dt, layout, kw) in enumerate(GENERAL_SHAPES):
        if only is not None and si != only:
            continue
        g = torch.Generator(device="cpu").manual_seed(7)
        x = torch.randn(xs, generator=g).to(dt)
        w = (torch.randn(ws, generator=g) / math.sqrt(ws[0] * math.prod(ws[2:]))).to(dt)
        b = (torch.randn(ws[1], generator=g) * 0.1).to(dt)
        if layout == "nhwc":
            x = x.movedim(1, -1).contiguous()
            w = w.movedim(1, -1).contiguous()
        flop = 2 * xs[0] * xs[1] * ws[1] * math.prod(xs[2:]) * math.prod(ws[2:])
        for algo in algos:
            try:
                op = ct.ConvTranspose(w.to(device), list(x.shape), b.to(device), layout=layout,
                                      algo=algo, **kw)
            except ct.CtError:
                continue
            if algo != "auto" and op.kernel != algo:
                continue
            esz = x.element_size()
            ybytes = math.prod(op.y_shape) * esz
            nbytes = (x.numel() + w.numel() + b.numel()) * esz + ybytes
            sets = max(2, min(8, int(2 * 126 * 2 ** 20 // max(1, ybytes)) + 1))
            xd = [x.to(device) for _ in range(sets)]
            yd = [torch.empty(op.y_shape, dtype=dt, device=device) for _ in range(sets)]
            for i in range(5):
                op(xd[i % sets], out=yd[i % sets])
            torch.cuda.synchronize(device)
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record()
            for i in range(runs):
                op(xd[i % sets], out=yd[i % sets])
            s1.record()
            torch.cuda.synchronize(device)
            us = s0.elapsed_time(s1) * 1e3 / runs
            tc_peak = peaks["tc_tflops"] * (TF32_PER_BF16 / 3 if dt == torch.float32 else 1.0)
            t_tc = flop / (tc_peak * 1e12)
            t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
            bound = "tensor" if t_tc >= t_hbm else "hbm"
            frac = max(t_tc, t_hbm) / (us * 1e-6)
            rec = {"shape": name, "algo": algo, "kernel": op.kernel,
                   "us_per_call": round(us, 2), "tflops": round(flop / us / 1e6, 1),
                   "gbs": round(nbytes / us / 1e3, 1), "bound": bound,
                   "frac": round(frac, 3)}
            results.append(rec)
            if not quiet:
                print(json.dumps(rec), flush=True)
            del op, xd, yd
    return results


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=HEADLINE)
    ap.add_argument("--no-others", action="store_true",
                    help="skip the secondary per-workload measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--plain", action="store_true",
                    help="profiling mode: eager ct_run launches of one workload, nothing else")
    ap.add_argument("--sets", type=int, default=1,
                    help="with --plain: X/Y buffer sets to rotate over (default 1)")
    ap.add_argument("--general", action="store_true",
                    help="time a set of general shapes (stride 1, 1x1, channels-last, many or few "
                         "channels) and print one JSON line per shape")
    ap.add_argument("--shape", type=int, default=None,
                    help="with --general: time only this entry of the general shape list")
    ap.add_argument("--algo", default=None, help="with --general: time only this algorithm")
    ap.add_argument("--runs", type=int, default=50, help="with --general: timed calls per shape")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = WORKLOADS[args.workload]
    flop, nbytes = workload_numbers(wl)
    config = {"workload": wl.name, "x": list(wl.x_shape), "w": list(wl.w_shape),
              "y": list(wl.y_shape), "global_batch": wl.x_shape[0] * max(world, 1),
              "parallelism": "dp%d (batch sharded: each GPU one workload-sized slice, "
                             "no data-path collective)" % max(world, 1)}

    if args.impl == "reference":
        if rank != 0:
            return
        per_step = []
        info = None
        budget = min(12.0, 150.0 / (args.steps + args.warmup))
        for _ in range(args.warmup):
            oracle_sample(wl, target_s=budget)
        for _ in range(args.steps):
            v, cores, desc, dt = oracle_sample(wl, target_s=budget)
            per_step.append((v, dt))
            info = (cores, desc)
        v = statistics.median([p[0] for p in per_step])
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
                "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * statistics.median([p[1] for p in per_step]),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic (seeded, workload distributions)",
                "config": config,
                "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": info[0],
                                 "kind": "oracle", "sample": info[1]},
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if args.general:
        kw = dict(runs=args.runs, only=args.shape)
        if args.algo:
            kw["algos"] = (args.algo,)
        general_shapes(torch.device("cuda", local), load_peaks(), **kw)
        return

    if args.plain:
        device = torch.device("cuda", local)
        torch.cuda.set_device(device)
        op, x_cpu = build_op(wl, device)
        # --sets K > 1 rotates K X/Y buffer sets, so that a workload smaller
        # than L2 still moves its data through DRAM as in the timed steps
        xs = [x_cpu.to(device) for _ in range(args.sets)]
        ys = [torch.empty(op.y_shape, dtype=wl.dtype, device=device) for _ in range(args.sets)]
        for i in range(args.warmup + args.steps):
            op(xs[i % args.sets], out=ys[i % args.sets])
        torch.cuda.synchronize(device)
        print(json.dumps({"plain": wl.name, "kernel": op.kernel, "launches": op.launches,
                          "runs": args.warmup + args.steps, "sets": args.sets}), flush=True)
        return

    dist_max = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist_max = make_dist_max(dist, device=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    peaks = load_peaks()

    sampler = ClockSampler(local)
    ms, info = time_device(wl, device, args.steps, args.warmup, l2, dist_max, sampler)
    ms, value = aggregate(flop, ms, args.steps, world, dist_max)
    sec_per_step = ms / 1e3 / args.steps
    roof = kernel_roofline(wl, args.workload, info, sec_per_step, peaks, props.multi_processor_count)

    e2e_steps = max(3, min(args.steps, 50))
    ems, hb, db = time_e2e(wl, device, e2e_steps, 3)
    ems, e2e_value = aggregate(flop, ems, e2e_steps, world, dist_max)

    others = {}
    if not args.no_others:
        for wid in sorted(WORKLOADS):
            if wid == args.workload:
                continue
            owl = WORKLOADS[wid]
            ofl, _ = workload_numbers(owl)
            osteps = 20 if owl.dtype == torch.float32 and wid == 4 else 200
            oms, oinfo = time_device(owl, device, osteps, 5, l2, dist_max)
            if dist_max is not None:
                oms = dist_max("max", oms)
            osec = oms / 1e3 / osteps
            oroof = kernel_roofline(owl, wid, oinfo, osec, peaks, props.multi_processor_count)
            others[str(wid)] = {"workload": owl.name, "kernel": oinfo["kernel"],
                                "us_per_step": osec * 1e6, "tflops": ofl / osec / 1e12,
                                "roofline": oroof}
        if world == 1:
            others["general"] = general_shapes(device, peaks, runs=50, algos=("auto",),
                                               quiet=True)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, desc, dt = oracle_sample(wl)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        clocks = sampler.summary()
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": max(world, 1),
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f16" if wl.dtype == torch.float16 else "f32",
                "data": "synthetic (seeded; X~N(0,1), W~N(0,1/32), bias~N(0,0.1))",
                "config": dict(config, l2="rotating %d X/Y buffer sets of %.1f MB (> L2 %d MB "
                               "between reuses)" % (info["sets"], info["set_bytes"] / 1e6,
                                                    l2 // 2 ** 20),
                               kernel=info["kernel"], launch="CUDA graph per step"),
                "roofline": roof,
                "cpu_baseline": cpu,
                "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": hb,
                        "d2h_bytes_per_step": db},
                "gpu_launches": args.steps * info["launches_per_step"],
                "clocks": clocks,
                "others": others}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
