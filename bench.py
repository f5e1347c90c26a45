#!/usr/bin/env python
"""Benchmark of the additive 2D Gaussian-splatting renderer, fwd + bwd.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the fp64 CPU oracle on host cores

One step = one pass of the whole hot path over one batch: tile binning, the
forward render and the backward pass (dL/dI is a fixed synthetic N(0, 1)
field, as in training after the loss) -- two library calls, pdr_render_fwd
(which bins) and pdr_render_bwd (which reuses the bins), replayed from a CUDA
graph with a timing event on each side.  L2 is flushed (a 256 MiB write)
between timed steps, outside the timed events.  Per-kernel times come from
separate graphs with events between the calls, timed after the timed region.
Each rank renders its own frames (weak scaling, no collective on the data
path); the time is the max over ranks.

Metric: Gaussian-pixel evaluations per second -- in-grid (Gaussian, window
pixel) pairs of one pass, counted once per fwd + bwd step -- and frames/s.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from differentiable_gaussian_splatting_pdr_b200.inputs import (  # noqa: E402
    WORKLOADS, WORKLOAD_ORDER, make_inputs, rank_seed)

METRIC = "Gaussian-pixel evals/s and frames/s (fwd+bwd, 1 B200), % of roofline"
UNIT = "evals/s"
# The largest single-GPU workload: 8 frames, C=3, 512x512, N=65536/frame, k=15.
DEFAULT_WORKLOAD = "stress512"
SM_COUNT = 148
FP32_LANES_PER_SM = 128
L2_FLUSH_BYTES = 256 << 20


def fp32_ops_per_eval(C: int):
    """Algorithmic FP32 instructions per in-window (Gaussian, pixel) pair:
    forward 7 + C (offsets, quadratic form, C accumulations), backward 15 + 2C
    (recompute 7, G = sum_c g_c a_c, v, C amplitude sums, five moments)."""
    return 7 + C, 15 + 2 * C


def in_grid_evals(params: np.ndarray, H: int, W: int, k: int) -> int:
    """Number of in-grid (Gaussian, window pixel) pairs: the work unit."""
    r = (k - 1) // 2
    mu = params[..., :2].astype(np.float64)
    ok = np.isfinite(mu).all(axis=-1)
    c = np.floor(np.where(np.isfinite(mu), mu, 0.0) + 0.5)
    nx = np.clip(np.minimum(c[..., 0] + r, W - 1) - np.maximum(c[..., 0] - r, 0) + 1, 0, None)
    ny = np.clip(np.minimum(c[..., 1] + r, H - 1) - np.maximum(c[..., 1] - r, 0) + 1, 0, None)
    return int((nx * ny * ok).sum())


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f)
    except OSError:
        return {}


def source_hash(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "differentiable_gaussian_splatting_pdr_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {"k_fwd": ("render_fwd.cu", "common.cuh"),
                  "k_fwd_cluster": ("render_fwd.cu", "common.cuh"),
                  "k_bwd": ("render_bwd.cu", "common.cuh"),
                  "k_loss_coef": ("loss.cu", "common.cuh"),
                  "k_loss_grad": ("loss.cu", "common.cuh")}
CLUSTER_MAX_TILES = 16       # frames of at most this many tiles ...
CLUSTER_MAX_BLOCKS = 4 * 148  # ... in launches of at most this many blocks: k_fwd_cluster


def forward_kernel(w) -> str:
    """The forward kernel the library launches for workload w: small launches
    of frames of at most 16 tiles are binned and rendered by one clustered
    launch; everything else is binned first and rendered by k_fwd."""
    tiles = -(-w.H // 16) * -(-w.W // 16)
    fused = tiles <= CLUSTER_MAX_TILES and w.B * tiles <= CLUSTER_MAX_BLOCKS
    return "k_fwd_cluster" if fused else "k_fwd"


def aggregate_over_ranks(torch, dist, world, device, evals, step_ms, extra_ms=()):
    """Whole-job figures from per-rank ones: the evals of all ranks summed
    (every rank renders its own frames, drawn with its own seed), and each time
    the max over ranks.  Every rank takes the same two collectives."""
    e = torch.tensor([float(evals)], dtype=torch.float64, device=device)
    t = torch.tensor([float(step_ms)] + [float(x) for x in extra_ms], dtype=torch.float64,
                     device=device)
    if world > 1:
        dist.all_reduce(e, op=dist.ReduceOp.SUM)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return int(round(float(e.item()))), [float(x) for x in t.tolist()]


def throughput(evals_all, steps, max_ms):
    """Units of all ranks per second over the max-over-ranks timed region."""
    return evals_all * steps / (max_ms * 1e-3)


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    if there is none or the kernel source changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "%s_%s.md" % (kernel, workload))
    try:
        txt = open(path).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)\s+source_sha:\s*([0-9a-f]+)", txt)
    if not m or m.group(2) != source_hash(*KERNEL_SOURCES[kernel]):
        return None
    return float(m.group(1))


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark(self) -> int:
        """Index of the next sample: summarise(a, b) covers samples between marks."""
        return len(self.lines)

    def stop(self):
        """Stop sampling; summary of every sample taken since start()."""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)
        return self.summarise(0, None)

    def summarise(self, a: int, b):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm, mx, pw, reasons = [], [], [], set()
        for line in self.lines[a:b]:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                pw.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# the oracle (CPU baseline and reference arm)
# ----------------------------------------------------------------------------
def oracle_sample(w, seconds: float, max_frames=None, threads=None):
    """Time the fp64 oracle fwd + bwd on the host cores (all of them, or
    `threads`) over a bounded sample of workload w: whole batches (or the first
    max_frames frames) repeated until `seconds` have passed.  Returns
    (evals/s, frames/s, cores, sample, seconds per repetition)."""
    import oracle  # test infrastructure: only the CPU-baseline leg runs it
    B = w.B if max_frames is None else min(w.B, max_frames)
    p, g = make_inputs(w)
    p, g = p[:B].copy(), g[:B].copy()
    ev = in_grid_evals(p, w.H, w.W, w.k)
    threads = oracle.max_threads() if threads is None else max(1, int(threads))
    cores = min(threads, B)  # OpenMP over frames: at most one thread per frame
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.render_fwd(p, w.H, w.W, w.k, threads)
        oracle.render_bwd(p, g, w.H, w.W, w.k, threads)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    sample = ("%d x fwd+bwd of %d/%d frames of %s (%s), fp64 oracle, OpenMP over frames "
              "on %d threads" % (reps, B, w.B, w.name, w.desc, cores))
    return ev * reps / dt, B * reps / dt, cores, sample, dt / reps


REFERENCE_BUDGET_S = 150.0  # host-core seconds the whole reference arm may take


def run_reference(args, w):
    """The oracle as the reference arm: fp64 fwd + bwd on the host cores, on
    whole batches of the workload (fewer frames per step only if K + W whole
    batches would take longer than REFERENCE_BUDGET_S)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import oracle  # test infrastructure: the reference arm is the oracle itself
    threads = oracle.max_threads()
    p_all, g_all = make_inputs(w)
    t0 = time.perf_counter()
    oracle.render_fwd(p_all, w.H, w.W, w.k, threads)
    oracle.render_bwd(p_all, g_all, w.H, w.W, w.k, threads)
    t_batch = time.perf_counter() - t0
    frames = w.B
    total = t_batch * (args.steps + args.warmup)
    if total > REFERENCE_BUDGET_S:
        frames = max(1, int(w.B * REFERENCE_BUDGET_S / total))
    p, g = p_all[:frames].copy(), g_all[:frames].copy()
    ev = in_grid_evals(p, w.H, w.W, w.k)
    cores = min(threads, frames)
    for _ in range(args.warmup):
        oracle.render_fwd(p, w.H, w.W, w.k, threads)
        oracle.render_bwd(p, g, w.H, w.W, w.k, threads)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.render_fwd(p, w.H, w.W, w.k, threads)
        oracle.render_bwd(p, g, w.H, w.W, w.k, threads)
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = ev * len(times) / tot
    sample = ("%d/%d frames of %s per step (%s), fp64 oracle, OpenMP over frames on %d threads"
              % (frames, w.B, w.name, w.desc, cores))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "frames_per_s": frames * len(times) / tot,
        "config": workload_config(w, evals_per_step=ev, frames=frames),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, **extra):
    cfg = {"workload": w.name, "desc": w.desc, "B": w.B, "C": w.C, "H": w.H, "W": w.W,
           "N": w.N, "k": w.k, "s": [w.s_mean, w.s_std], "amplitudes": list(w.amp),
           "seed": w.seed}
    cfg.update(extra)
    return cfg


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------
def graph_kernel_nodes(graph) -> int:
    """Kernel nodes in a captured CUDA graph (all of them library kernels)."""
    try:
        from cuda.bindings import runtime as rt
        g = rt.cudaGraph_t(init_value=graph.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(g, numNodes=0)
        err, nodes, n = rt.cudaGraphGetNodes(g, numNodes=n)
        kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes]
        return sum(1 for k in kinds if k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:  # pragma: no cover - reporting only
        return -1


class Step:
    """One training-style pass on one batch: forward (binning included; for
    frames of at most 16 tiles the binning runs inside the forward launch),
    then the backward reusing the forward's bins.  Captured as CUDA graphs:
      main  -- [event] forward, backward [event]           (the timed step)
      split -- [event] forward [event] backward [event]    (stage times)
      fwd   -- [event] bins [event] forward from bins [event] (k_fwd alone)"""

    def __init__(self, R, torch, w, seed, device, dtype=None):
        self.R, self.torch, self.w, self.device = R, torch, w, device
        self.dtype = torch.float32 if dtype is None else dtype  # image / dL/dI storage
        p, g = make_inputs(w, seed)
        self.evals = in_grid_evals(p, w.H, w.W, w.k)
        self.h_params = torch.from_numpy(p).pin_memory()
        self.h_grad = torch.from_numpy(g).pin_memory()
        self.params = self.h_params.to(device)
        self.grad = self.h_grad.to(device).to(self.dtype)
        self.image = torch.empty((w.B, w.C, w.H, w.W), dtype=self.dtype, device=device)
        self.dparams = torch.empty_like(self.params)
        self.ws = R.Workspace.for_sizes(w.B, w.N, w.C, w.H, w.W, w.k, device)
        self.graphs, self.events = {}, {}

    def fwd(self, reuse_bins=False):
        w = self.w
        self.R.render_fwd(self.params, w.H, w.W, w.k, self.ws, self.image, reuse_bins=reuse_bins,
                          dtype=self.dtype)

    def bwd(self):
        w = self.w
        self.R.render_bwd(self.params, self.grad, w.H, w.W, w.k, self.ws, self.dparams,
                          reuse_bins=True)

    def bins(self):
        w = self.w
        self.R.build_bins(self.params, w.H, w.W, w.k, self.ws)

    def eager(self):
        self.fwd()
        self.bwd()

    def _capture(self, name, parts):
        torch = self.torch
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(parts) + 1)]
        g = torch.cuda.CUDAGraph(keep_graph=True)  # kept so its kernel nodes can be counted
        with torch.cuda.graph(g):
            ev[0].record()
            for j, part in enumerate(parts):
                for fn in part:
                    fn()
                ev[j + 1].record()
        g.instantiate()
        self.graphs[name], self.events[name] = g, ev

    def capture(self):
        torch = self.torch
        s = torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            for _ in range(2):
                self.eager()
                self.bins()
                self.fwd(reuse_bins=True)
        torch.cuda.current_stream(self.device).wait_stream(s)
        torch.cuda.synchronize(self.device)
        self._capture("main", [[self.fwd, self.bwd]])
        self._capture("split", [[self.fwd], [self.bwd]])
        self._capture("fwd", [[self.bins], [lambda: self.fwd(reuse_bins=True)]])
        torch.cuda.synchronize(self.device)

    def replay(self, name="main"):
        self.graphs[name].replay()

    def times(self, name):
        e = self.events[name]
        return [e[j].elapsed_time(e[j + 1]) for j in range(len(e) - 1)]


def time_graph(step, name, flush, K, stream):
    """K replays of one graph, L2 flushed before each; per-step [total, stages...] ms."""
    out = []
    for _ in range(K):
        flush.fill_(1)
        step.replay(name)
        stream.synchronize()
        st = step.times(name)
        out.append([sum(st)] + st)
    return np.array(out)


def time_eager_steps(step, torch, flush, K, stream):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = []
    for _ in range(K):
        flush.fill_(1)
        e0.record()
        step.eager()
        e1.record()
        stream.synchronize()
        out.append(e0.elapsed_time(e1))
    return np.array(out)


def time_e2e_steps(step, torch, K, stream):
    """The host-buffer C-ABI call (pdr_step_host): H2D inputs, fwd, bwd, D2H
    image and gradients, all inside the timed events."""
    R, w = step.R, step.w
    bufs = None
    _, _, bufs = R.step_host(step.h_params, step.h_grad, w.H, w.W, w.k, None, step.device)
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = []
    for _ in range(K):
        e0.record()
        R.step_host(step.h_params, step.h_grad, w.H, w.W, w.k, bufs, step.device)
        e1.record()
        stream.synchronize()
        out.append(e0.elapsed_time(e1))
    h2d = step.h_params.numel() * 4 + step.h_grad.numel() * 4
    d2h = bufs["h_image"].numel() * 4 + bufs["h_grad_params"].numel() * 4
    return np.array(out), h2d, d2h


# FP32 instructions per pixel of the L1 + SSIM loss in its separable form:
# x^2, y^2, xy (3); five moments, two 11-tap passes (110); SSIM map and the
# three gradient coefficients (~25); three coefficient maps, two passes (66);
# the final combination and the L1 term (6).
LOSS_OPS_PER_PX = 210


class LossBench:
    """The L1 + SSIM loss on a workload's image shape: image ~ U[0, 1],
    target = clip(image + N(0, 0.1)); one call per step, CUDA-graph replay,
    CUDA events, L2 flushed before every call."""

    def __init__(self, R, torch, w, seed, device):
        self.workload = w.name
        rng = np.random.default_rng(seed + 7)
        x = rng.uniform(0, 1, (w.B, w.C, w.H, w.W)).astype(np.float32)
        y = np.clip(x + rng.normal(0, 0.1, x.shape), 0, 1).astype(np.float32)
        self.x, self.y = x, y
        self.xt, self.yt = torch.from_numpy(x).to(device), torch.from_numpy(y).to(device)
        self.ws = torch.empty(max(R.loss_workspace_bytes(w.B, w.C, w.H, w.W), 256),
                              dtype=torch.uint8, device=device)
        self.grad = torch.empty_like(self.xt)
        self.loss = torch.empty(1, dtype=torch.float32, device=device)
        self.R, self.torch, self.px = R, torch, x.size
        self.call()
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        self.ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        with torch.cuda.graph(g):
            self.ev[0].record()
            self.call()
            self.ev[1].record()
        self.graph = g

    def call(self):
        self.R.l1_ssim_loss(self.xt, self.yt, 0.2, 1.0, self.ws, self.grad, self.loss)

    def time(self, flush, K, stream):
        out = []
        for _ in range(K):
            flush.fill_(1)
            self.graph.replay()
            stream.synchronize()
            out.append(self.ev[0].elapsed_time(self.ev[1]))
        return float(np.mean(out))

    def traffic(self):
        a = profiled_traffic("k_loss_coef", self.workload)
        b = profiled_traffic("k_loss_grad", self.workload)
        return None if a is None or b is None else a + b

    def entry(self, ms, peak_tops):
        ops = self.px * LOSS_OPS_PER_PX
        achieved = ops / (ms * 1e-3) / 1e12
        return {"ms_per_call": ms, "px_per_s": self.px / (ms * 1e-3),
                "roofline": {"bound": "alu", "kernel": "k_loss_coef + k_loss_grad (one call)",
                             "achieved": achieved,
                             "peak": peak_tops, "unit": "Tinst/s", "frac": achieved / peak_tops,
                             "ops_per_px": LOSS_OPS_PER_PX,
                             "traffic": self.traffic(),
                             "algorithmic_bytes": 12 * self.px},
                "data": "image ~ U[0,1], target = clip(image + N(0, 0.1)), lam 0.2"}


def loss_oracle_rate(x, y, seconds):
    """fp64 oracle (numpy) pixels/s on whole frames of (x, y), about `seconds`."""
    from oracle import loss as oracle_loss  # test infrastructure: the CPU-baseline leg only
    reps, t0, px = 0, time.perf_counter(), 0
    B = x.shape[0]
    nf = 1
    while True:
        xs, ys = x[:nf], y[:nf]
        oracle_loss.l1_ssim_loss(xs, ys)
        reps += 1
        px += xs.size
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
        nf = min(B, nf * 2)
    return px / dt, "%d oracle calls on up to %d of %d frames (numpy fp64, 1 process)" % (reps, nf, B)


def roofline_entry(kernel, ms, evals, C, peak_tops, workload, w):
    ops_f, ops_b = fp32_ops_per_eval(C)
    fwd = kernel.startswith("k_fwd")
    ops = evals * (ops_f if fwd else ops_b)
    achieved = ops / (ms * 1e-3) / 1e12
    if fwd:
        alg_bytes = 4 * w.B * w.N * (5 + C) + 4 * w.B * C * w.H * w.W
    else:
        alg_bytes = 8 * w.B * w.N * (5 + C) + 4 * w.B * C * w.H * w.W
    return {"bound": "alu", "kernel": kernel, "achieved": achieved, "peak": peak_tops,
            "unit": "Tinst/s", "frac": achieved / peak_tops,
            "traffic": profiled_traffic(kernel, workload),
            "ops_per_launch": ops, "algorithmic_bytes": alg_bytes,
            "ms_per_launch": ms}


def run_gpu(args, w):
    import torch
    import torch.distributed as dist
    from differentiable_gaussian_splatting_pdr_b200 import api as R
    from differentiable_gaussian_splatting_pdr_b200 import build as pdr_build

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print("warning: WORLD_SIZE=%d but --gpus %d" % (world, args.gpus), file=sys.stderr)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    if rank == 0:
        pdr_build.build()
    if world > 1:
        dist.barrier()
    R._lib.load()
    stream = torch.cuda.current_stream(device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    step = Step(R, torch, w, rank_seed(w, rank), device)
    step.capture()
    for _ in range(args.warmup):
        flush.fill_(1)
        step.replay()
    R.check_device_error(step.ws, device)

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(device).uuid).replace("GPU-", "")
    clocks = ClockSampler(gpu_id)
    clocks.start()
    m0 = clocks.mark()  # the soak runs the timed step itself, so it counts as timed load
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < args.soak:   # clocks settle under the same step
        flush.fill_(1)
        step.replay()
    stream.synchronize()

    # ---------------- timed region ----------------
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    per = time_graph(step, "main", flush, args.steps, stream)
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    # ----------------------------------------------
    m1 = clocks.mark()
    R.check_device_error(step.ws, device)

    eager = time_eager_steps(step, torch, flush, args.steps, stream)
    e2e, h2d, d2h = time_e2e_steps(step, torch, args.steps, stream)
    evals_all, (max_ms, eager_ms, e2e_ms) = aggregate_over_ranks(
        torch, dist, world, device, step.evals, float(per[:, 0].sum()),
        (float(eager.sum()), float(e2e.sum())))
    value = throughput(evals_all, args.steps, max_ms)
    frames_per_s = throughput(w.B * world, args.steps, max_ms)
    eager_value = throughput(evals_all, args.steps, eager_ms)
    e2e_value = throughput(evals_all, args.steps, e2e_ms)

    # Stage breakdown (after the timed region, same L2 flushing).
    split = time_graph(step, "split", flush, args.steps, stream)
    fsplit = time_graph(step, "fwd", flush, args.steps, stream)
    ms_fwd_step = float(np.mean(split[:, 1]))     # forward incl. binning, as in the step
    ms_bwd = float(np.mean(split[:, 2]))          # k_bwd alone
    ms_bins = float(np.mean(fsplit[:, 1]))        # binning alone
    ms_fwd = float(np.mean(fsplit[:, 2]))         # k_fwd alone, from prebuilt bins

    pk = measured_peaks()
    sm_max = float(pk.get("sm_max_mhz") or 1965.0)
    peak_tops = SM_COUNT * FP32_LANES_PER_SM * sm_max * 1e6 / 1e12
    # The forward kernel of the step: k_fwd_cluster (binning inside, so its
    # time is the step's whole forward) or k_fwd (timed from prebuilt bins).
    fk = forward_kernel(w)
    ms_fk = ms_fwd_step if fk == "k_fwd_cluster" else ms_fwd
    kern = sorted([(ms_fk, fk), (ms_bwd, "k_bwd")], reverse=True)
    roof = roofline_entry(kern[0][1], kern[0][0], step.evals, w.C, peak_tops, w.name, w)
    roof["peak_source"] = ("148 SMs x 128 FP32 lanes x %.0f MHz (sm_max_mhz, MEASURED_PEAKS.json)"
                           % sm_max)
    other = roofline_entry(kern[1][1], kern[1][0], step.evals, w.C, peak_tops, w.name, w)

    lb = LossBench(R, torch, w, rank_seed(w, rank), device)
    loss_ms = lb.time(flush, args.steps, stream)
    loss_entry = lb.entry(loss_ms, peak_tops)
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        rate, sample = loss_oracle_rate(lb.x, lb.y, min(3.0, args.cpu_seconds))
        loss_entry["cpu_oracle_px_per_s"] = rate
        loss_entry["cpu_oracle_sample"] = sample
    del lb

    sweep = {}
    if args.sweep and rank == 0:
        for name in WORKLOAD_ORDER:
            if name == w.name:
                continue
            sw = WORKLOADS[name]
            st = Step(R, torch, sw, sw.seed, device)
            st.capture()
            for _ in range(5):
                flush.fill_(1)
                st.replay()
            pr = time_graph(st, "main", flush, args.sweep_steps, stream)
            sp = time_graph(st, "split", flush, args.sweep_steps, stream)
            fs = time_graph(st, "fwd", flush, args.sweep_steps, stream)
            R.check_device_error(st.ws, device)
            e2e_s, h2d_s, d2h_s = time_e2e_steps(st, torch, args.sweep_steps, stream)
            tot = float(pr[:, 0].mean())
            f_ms, b_ms = float(fs[:, 2].mean()), float(sp[:, 2].mean())
            of, ob = fp32_ops_per_eval(sw.C)
            sweep[name] = {
                "evals_per_s": st.evals / (tot * 1e-3), "frames_per_s": sw.B / (tot * 1e-3),
                "ms_per_step": tot, "ms_fwd_incl_bins": float(sp[:, 1].mean()),
                "ms_bins": float(fs[:, 1].mean()), "ms_fwd": f_ms,
                "ms_bwd": b_ms, "evals_per_step": st.evals,
                "kernels_per_step": graph_kernel_nodes(st.graphs["main"]),
                "fwd_frac": st.evals * of / (f_ms * 1e-3) / 1e12 / peak_tops,
                "bwd_frac": st.evals * ob / (b_ms * 1e-3) / 1e12 / peak_tops,
                "step_frac": st.evals * (of + ob) / (tot * 1e-3) / 1e12 / peak_tops,
                "e2e": {"value": st.evals / (float(e2e_s.mean()) * 1e-3), "unit": UNIT,
                        "h2d_bytes_per_step": h2d_s, "d2h_bytes_per_step": d2h_s,
                        "api": "pdr_step_host"},
            }
            del st
            lbs = LossBench(R, torch, sw, sw.seed, device)
            lms = lbs.time(flush, args.sweep_steps, stream)
            sweep[name]["ms_loss_l1_ssim"] = lms
            sweep[name]["loss_frac"] = lbs.entry(lms, peak_tops)["roofline"]["frac"]
            del lbs

    # A training iteration: render, L1 + SSIM against a target image, backward
    # from the loss's dL/dI (one graph).
    train = {}
    if rank == 0:
        st = Step(R, torch, w, rank_seed(w, rank), device)
        tgt = torch.clamp(st.image.new_empty(st.image.shape).normal_(0.5, 0.25), 0, 1)
        lws = torch.empty(max(R.loss_workspace_bytes(w.B, w.C, w.H, w.W), 256), dtype=torch.uint8,
                          device=device)
        lgrad = torch.empty_like(st.image)
        lval = torch.empty(1, dtype=torch.float32, device=device)

        def train_step():
            st.fwd()
            R.l1_ssim_loss(st.image, tgt, 0.2, 1.0, lws, lgrad, lval)
            R.render_bwd(st.params, lgrad, w.H, w.W, w.k, st.ws, st.dparams, reuse_bins=True)

        st.capture()
        st._capture("train", [[train_step]])
        for _ in range(5):
            flush.fill_(1)
            st.replay("train")
        pr = time_graph(st, "train", flush, args.steps, stream)
        R.check_device_error(st.ws, device)
        tot = float(pr[:, 0].mean())
        train = {"ms_per_step": tot, "evals_per_s": st.evals / (tot * 1e-3),
                 "frames_per_s": w.B / (tot * 1e-3),
                 "step": "render_fwd (binning inside) + l1_ssim_loss (target ~ clip(N(0.5, 0.25))) "
                         "+ render_bwd from the loss's dL/dI, one CUDA graph",
                 "kernels_per_step": graph_kernel_nodes(st.graphs["train"])}
        del st

    # Reduced-precision storage of image and dL/dI (fp32 sums): the same step.
    storage = {}
    if rank == 0:
        for dname in ("float16", "bfloat16"):
            st = Step(R, torch, w, rank_seed(w, rank), device, dtype=getattr(torch, dname))
            st.capture()
            for _ in range(5):
                flush.fill_(1)
                st.replay()
            pr = time_graph(st, "main", flush, args.sweep_steps, stream)
            R.check_device_error(st.ws, device)
            tot = float(pr[:, 0].mean())
            storage[dname] = {"ms_per_step": tot, "evals_per_s": st.evals / (tot * 1e-3)}
            del st

    knobs = {}
    if args.knobs and args.sweep and rank == 0:
        from differentiable_gaussian_splatting_pdr_b200.inputs import knob_workloads
        for name, kw in knob_workloads(w.name if w.name in ("mono64",) else "mono64").items():
            st = Step(R, torch, kw, kw.seed, device)
            st.capture()
            for _ in range(5):
                flush.fill_(1)
                st.replay()
            pr = time_graph(st, "main", flush, args.sweep_steps, stream)
            R.check_device_error(st.ws, device)
            tot = float(pr[:, 0].mean())
            of, ob = fp32_ops_per_eval(kw.C)
            knobs[name] = {"desc": kw.desc, "evals_per_step": st.evals, "ms_per_step": tot,
                           "evals_per_s": st.evals / (tot * 1e-3),
                           "step_frac": st.evals * (of + ob) / (tot * 1e-3) / 1e12 / peak_tops}
            del st

    clk = clocks.stop()   # every GPU timed region of this run lies between start and here
    clk_main = clocks.summarise(m0, m1)

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        v, fps, cores, sample, _ = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
               "frames_per_s": fps}
        v1, fps1, _, sample1, _ = oracle_sample(w, min(3.0, args.cpu_seconds), max_frames=1,
                                                threads=1)
        cpu["single_core"] = {"value": v1, "unit": UNIT, "cores": 1, "sample": sample1,
                              "frames_per_s": fps1}
        # The oracle beside every other workload of the sweep (a bounded sample each).
        for name in sweep:
            sw = WORKLOADS[name]
            ov, ofps, oc, osample, _ = oracle_sample(sw, min(2.0, args.cpu_seconds))
            sweep[name]["cpu_baseline"] = {"value": ov, "unit": UNIT, "cores": oc,
                                           "kind": "oracle", "sample": osample,
                                           "frames_per_s": ofps}

    if rank == 0:
        launches_per_step = graph_kernel_nodes(step.graphs["main"])
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "frames_per_s": frames_per_s,
            "config": workload_config(
                w, evals_per_step_per_gpu=step.evals, evals_per_step_all_gpus=evals_all,
                frames_per_gpu=w.B,
                l2="flushed before every timed step (256 MiB write, outside the timed events)",
                step="forward (with its binning) + backward, CUDA-graph replay, per-step CUDA events",
                parallelism="dp%d (frames sharded per rank, no data-path collective)" % world),
            "roofline": roof,
            "roofline_other_kernel": other,
            "stages_ms": {"step": float(per[:, 0].mean()), "fwd_incl_bins": ms_fwd_step,
                          "k_bwd": ms_bwd, "bins_alone": ms_bins, "k_fwd_alone": ms_fwd,
                          "note": "step = forward (binning inside) + backward, one graph; "
                                  "the other figures come from split graphs timed after it"},
            "eager": {"value": eager_value, "unit": UNIT,
                      "note": "same step without graph replay (per-call launches)"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "api": "pdr_step_host: pinned host -> device, fwd, bwd, device -> host"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "clocks_main_region": clk_main,
            "cpu_baseline": cpu,
            "loss_l1_ssim": loss_entry,
            "sweep": sweep,
            "knobs": knobs,
            "storage_half": storage,
            "train_step": train,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        del step
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=WORKLOAD_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--soak", type=float, default=2.0,
                    help="seconds of untimed steps while the clock sampler starts")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="host-core time budget of the oracle baseline (0 = skip)")
    ap.add_argument("--no-sweep", dest="sweep", action="store_false")
    ap.add_argument("--no-knobs", dest="knobs", action="store_false",
                    help="skip the knob variants (grid layout, Gaussian count, window size)")
    ap.add_argument("--sweep-steps", type=int, default=50)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
