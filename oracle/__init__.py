"""fp64 CPU oracle for the additive 2D Gaussian-splatting renderer.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are its only callers.  The CUDA product path never imports,
loads or calls anything here, and shares no code with it.

Thin ctypes wrapper around ``oracle.c`` (see that file for what is computed
and for every reading of the paper's pages).  All three entry points take the
fp32 parameter tensor ``params[B, N, 5 + C]`` = (mu_x, mu_y, s_1, s_2, theta,
a_0 .. a_{C-1}) and return fp64 results.

Parity status: every function here is pinned by the CPU tests
(tests/test_oracle_pins.py): closed forms, invariants, an independent
separable-sum evaluation, brute-force window indicators and central finite
differences.  No function is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_longlong)
        i32p = ctypes.POINTER(ctypes.c_int)
        c_int = ctypes.c_int
        lib.oracle_render_fwd.argtypes = [f32p] + [c_int] * 6 + [f64p, c_int]
        lib.oracle_render_fwd.restype = c_int
        lib.oracle_render_bwd.argtypes = [f32p, f32p] + [c_int] * 6 + [f64p, c_int]
        lib.oracle_render_bwd.restype = c_int
        lib.oracle_render_fwd_f64.argtypes = [f64p] + [c_int] * 6 + [f64p, c_int]
        lib.oracle_render_fwd_f64.restype = c_int
        lib.oracle_render_bwd_f64.argtypes = [f64p, f64p] + [c_int] * 6 + [f64p, c_int]
        lib.oracle_render_bwd_f64.restype = c_int
        lib.oracle_bin.argtypes = [f32p] + [c_int] * 6 + [i64p, i32p, ctypes.c_longlong]
        lib.oracle_bin.restype = ctypes.c_longlong
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = c_int
        _lib = lib
    return _lib


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _params(params):
    dt = np.float64 if np.asarray(params).dtype == np.float64 else np.float32
    params = np.ascontiguousarray(params, dtype=dt)
    if params.ndim != 3 or params.shape[2] < 6:
        raise ValueError("params must be [B, N, 5 + C] with C >= 1")
    B, N, P = params.shape
    return params, B, N, P - 5


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def render_fwd(params, H: int, W: int, k: int, threads: int = 1) -> np.ndarray:
    """I[b, c, y, x] (fp64) from params [B, N, 5+C] (fp32, or fp64 for FD checks)."""
    lib = _load()
    params, B, N, C = _params(params)
    img = np.empty((B, C, H, W), dtype=np.float64)
    if params.dtype == np.float64:
        rc = lib.oracle_render_fwd_f64(_p(params, ctypes.c_double), B, N, C, H, W, k,
                                       _p(img, ctypes.c_double), int(threads))
    else:
        rc = lib.oracle_render_fwd(_p(params, ctypes.c_float), B, N, C, H, W, k,
                                   _p(img, ctypes.c_double), int(threads))
    if rc != 0:
        raise ValueError("oracle_render_fwd: bad arguments")
    return img


def render_bwd(params, grad_image, H: int, W: int, k: int, threads: int = 1) -> np.ndarray:
    """dL/dparams [B, N, 5+C] (fp64) from dL/dI [B, C, H, W].

    fp32 params and dL/dI take the fp32 entry point; fp64 params (finite-
    difference checks) take the fp64 one, with dL/dI widened to fp64."""
    lib = _load()
    params, B, N, C = _params(params)
    out = np.empty((B, N, 5 + C), dtype=np.float64)
    if params.dtype == np.float64:
        g = np.ascontiguousarray(grad_image, dtype=np.float64)
        if g.shape != (B, C, H, W):
            raise ValueError("grad_image must be [B, C, H, W]")
        rc = lib.oracle_render_bwd_f64(_p(params, ctypes.c_double), _p(g, ctypes.c_double),
                                       B, N, C, H, W, k, _p(out, ctypes.c_double), int(threads))
    else:
        g = np.ascontiguousarray(grad_image, dtype=np.float32)
        if g.shape != (B, C, H, W):
            raise ValueError("grad_image must be [B, C, H, W]")
        rc = lib.oracle_render_bwd(_p(params, ctypes.c_float), _p(g, ctypes.c_float),
                                   B, N, C, H, W, k, _p(out, ctypes.c_double), int(threads))
    if rc != 0:
        raise ValueError("oracle_render_bwd: bad arguments")
    return out


def bin_tiles(params, H: int, W: int, k: int):
    """Brute-force 16x16 tile lists.

    Returns (tile_offsets [B*T + 1] int64, tile_ids [E] int32): the entries of
    tile t of frame b are tile_ids[tile_offsets[b*T + t] : tile_offsets[b*T + t + 1]],
    frame-local Gaussian indices in ascending order; tiles row-major.
    """
    lib = _load()
    params, B, N, C = _params(params)
    params = np.ascontiguousarray(params, dtype=np.float32)
    T = ((H + 15) // 16) * ((W + 15) // 16)
    offs = np.empty(B * T + 1, dtype=np.int64)
    e = lib.oracle_bin(_p(params, ctypes.c_float), B, N, C, H, W, k,
                       _p(offs, ctypes.c_longlong), None, 0)
    if e < 0:
        raise ValueError("oracle_bin: bad arguments")
    ids = np.empty(max(int(e), 1), dtype=np.int32)
    e2 = lib.oracle_bin(_p(params, ctypes.c_float), B, N, C, H, W, k,
                        _p(offs, ctypes.c_longlong), _p(ids, ctypes.c_int), int(e))
    assert e2 == e
    return offs, ids[: int(e)]
