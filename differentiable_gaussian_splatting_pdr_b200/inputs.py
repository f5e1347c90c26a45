"""Seeded synthetic inputs for the additive 2D Gaussian-splatting renderer.

This module only draws random numbers; it holds none of the renderer's
arithmetic.  Both the fp64 oracle (tests) and the CUDA path (tests, bench)
take their inputs from here, so the two sides always see the same bytes.

Parameter layout (one row per Gaussian, 5 + C fp32 values):
    (mu_x, mu_y, s_1, s_2, theta, a_0 ... a_{C-1})
"position, scale, rotation, and C channel amplitudes" -- "Learning Video
Dynamics with Predictive Differentiable Rendering", abstract.

The five workloads stand in for the paper's TaxiBJ / WeatherBench / KTH /
Human3.6M experiments (abstract; reading notes, "Dataset / Evaluation"),
which are not available here: only their shapes (frames, channels, grid,
Gaussians per frame, window size) are mimicked.

Draw order per workload (numpy PCG64 ``default_rng(seed)``, fp64 draws cast
to fp32 once): mu_x ~ U[0, W), mu_y ~ U[0, H) (or, for the grid layout, the
jitters of a regular grid), s_1, s_2 ~ N(m, sd),
theta ~ U[0, pi), a (row-major [B, N, C]), then dL/dI ~ N(0, 1) as [B, C, H, W].
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, Tuple

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int          # frames
    C: int          # channels
    H: int          # rows
    W: int          # columns
    N: int          # Gaussians per frame
    k: int          # odd window size (k x k pixels around round(mu))
    s_mean: float
    s_std: float
    amp: Tuple[str, float, float] = ("normal", 0.0, 1.0)  # (kind, p0, p1)
    seed: int = 0
    desc: str = ""
    layout: str = "uniform"  # "uniform" means, or "grid": a jittered regular grid

    @property
    def P(self) -> int:
        """Parameters per Gaussian (5 + C)."""
        return 5 + self.C

    @property
    def tiles(self) -> int:
        return ((self.H + 15) // 16) * ((self.W + 15) // 16)

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five synthetic workloads (frames, channels, grid, Gaussians, window,
# scale / amplitude distributions).  Seeds: 0 for the tiny case, otherwise the
# workload's index.
WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", B=1, C=1, H=32, W=32, N=64, k=7, s_mean=0.3, s_std=0.3,
                 amp=("normal", 0.0, 1.0), seed=0,
                 desc="1 frame, C=1, 32x32, N=64, k=7"),
        Workload("mono64", B=16, C=1, H=64, W=64, N=1024, k=9, s_mean=0.5, s_std=0.4,
                 amp=("exponential", 1.0, 0.0), seed=1,
                 desc="16 frames, C=1, 64x64, N=1024/frame, k=9, a~Exp(1)"),
        Workload("rgb128", B=16, C=3, H=128, W=128, N=4096, k=11, s_mean=0.7, s_std=0.5,
                 amp=("normal", 0.5, 0.3), seed=2,
                 desc="16 frames, C=3, 128x128, N=4096/frame, k=11"),
        Workload("field32x64", B=320, C=4, H=32, W=64, N=2048, k=9, s_mean=0.8, s_std=0.3,
                 amp=("normal", 0.0, 1.0), seed=3,
                 desc="320 frames, C=4, 32x64 lat-lon-shaped grid, N=2048/frame, k=9"),
        Workload("stress512", B=8, C=3, H=512, W=512, N=65536, k=15, s_mean=1.0, s_std=0.8,
                 amp=("normal", 0.0, 1.0), seed=4,
                 desc="8 frames, C=3, 512x512, N=65536/frame, k=15"),
    ]
}

WORKLOAD_ORDER = ["tiny", "mono64", "rgb128", "field32x64", "stress512"]


def _grid_means(rng, w: Workload):
    """Grid-initialised means (the initial layout of a Gaussian field): the N
    Gaussians of a frame on the first N cells of a ceil(sqrt(N W / H)) x
    ceil(N / that) grid over the frame, each jittered U(-1/4, 1/4) of a cell."""
    B, N = w.B, w.N
    gx = max(1, int(np.ceil(np.sqrt(N * w.W / w.H))))
    gy = max(1, int(np.ceil(N / gx)))
    cell = np.arange(N)
    cx = (cell % gx + 0.5) * (w.W / gx)
    cy = (cell // gx + 0.5) * (w.H / gy)
    jx = rng.uniform(-0.25, 0.25, size=(B, N)) * (w.W / gx)
    jy = rng.uniform(-0.25, 0.25, size=(B, N)) * (w.H / gy)
    return cx[None, :] + jx, cy[None, :] + jy


def _draw(w: Workload, seed, want_grad: bool):
    rng = np.random.default_rng(w.seed if seed is None else seed)
    B, N, C = w.B, w.N, w.C
    if w.layout == "grid":
        mu_x, mu_y = _grid_means(rng, w)
    elif w.layout == "uniform":
        mu_x = rng.uniform(0.0, float(w.W), size=(B, N))
        mu_y = rng.uniform(0.0, float(w.H), size=(B, N))
    else:
        raise ValueError(w.layout)
    s1 = rng.normal(w.s_mean, w.s_std, size=(B, N))
    s2 = rng.normal(w.s_mean, w.s_std, size=(B, N))
    theta = rng.uniform(0.0, np.pi, size=(B, N))
    kind, p0, p1 = w.amp
    if kind == "normal":
        a = rng.normal(p0, p1, size=(B, N, C))
    elif kind == "exponential":
        a = rng.exponential(p0, size=(B, N, C))
    else:
        raise ValueError(kind)
    params = np.empty((B, N, 5 + C), dtype=np.float32)
    params[..., 0] = mu_x
    params[..., 1] = mu_y
    params[..., 2] = s1
    params[..., 3] = s2
    params[..., 4] = theta
    params[..., 5:] = a
    grad = None
    if want_grad:
        grad = rng.standard_normal(size=(B, C, w.H, w.W)).astype(np.float32)
    return params, grad


def make_params(w: Workload, seed: int | None = None) -> np.ndarray:
    """Draw the [B, N, 5+C] fp32 parameter tensor of a workload."""
    return _draw(w, seed, False)[0]


def make_grad_image(w: Workload, seed: int | None = None) -> np.ndarray:
    """Draw dL/dI ~ N(0, 1) as [B, C, H, W] fp32 (drawn after the parameters)."""
    return _draw(w, seed, True)[1]


def make_inputs(w: Workload, seed: int | None = None):
    """(params [B,N,5+C], grad_image [B,C,H,W]) for a workload, fp32."""
    return _draw(w, seed, True)


def knob_workloads(base: str = "mono64"):
    """Variants of one workload along the knobs the pages name (reading notes,
    "Relation To Prior Work" and "Limitation": grid-initialised Gaussians, the
    Gaussian count and the kernel support): name -> Workload."""
    w = WORKLOADS[base]
    out = {"%s-grid" % base: replace(w, layout="grid", name="%s-grid" % base,
                                      desc=w.desc + ", grid-initialised means")}
    for n in (w.N // 4, w.N * 4):
        out["%s-N%d" % (base, n)] = replace(w, N=n, name="%s-N%d" % (base, n),
                                              desc=_desc(w, N=n))
    for k in (5, 13, 17):
        out["%s-k%d" % (base, k)] = replace(w, k=k, name="%s-k%d" % (base, k),
                                              desc=_desc(w, k=k))
    return out


def _desc(w: Workload, **kw) -> str:
    """Description of workload w with some of its sizes replaced."""
    v = replace(w, **kw)
    amp = {"normal": "a~N(%g,%g)", "exponential": "a~Exp(%g)"}[v.amp[0]]
    amp = amp % ((v.amp[1],) if v.amp[0] == "exponential" else (v.amp[1], v.amp[2]))
    return "%d frames, C=%d, %dx%d, N=%d/frame, k=%d, %s" % (v.B, v.C, v.H, v.W, v.N, v.k, amp)


def rank_seed(w: Workload, rank: int) -> int:
    """Seed for one rank's shard of frames when frames are split over ranks."""
    return w.seed + 1000 * rank
