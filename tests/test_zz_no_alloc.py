"""pdr_render_fwd_noalloc: the forward render for callers that cannot allocate
device memory (for example a plugin whose host application owns all device
memory, or a loop that must not allocate after start-up).  It uses a scratch
array built into the library instead of a caller workspace; its output must
match the workspace entry point pdr_render_fwd, call after call, and the
fp64 oracle; repeated calls must leave the device's free memory unchanged.

This file is collected last on purpose, so that a failure here comes after
every other test has run.
"""
import numpy as np
import pytest
import torch

import oracle
from differentiable_gaussian_splatting_pdr_b200 import _lib
from differentiable_gaussian_splatting_pdr_b200 import api as R
from differentiable_gaussian_splatting_pdr_b200 import build as pdr_build
from differentiable_gaussian_splatting_pdr_b200.inputs import WORKLOADS, make_params

pytestmark = pytest.mark.gpu

FWD_TOL = 1e-5   # the forward tolerance of the parity tests (normwise per frame, channel)
PDR_ERR_TOO_LARGE = 6


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pdr_build.build()
    return _lib.load()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _noalloc(lib, params, H, W, k):
    B, N, P = params.shape
    out = torch.full((B, P - 5, H, W), float("nan"), device=params.device)
    _lib.check("pdr_render_fwd_noalloc", lib.pdr_render_fwd_noalloc(
        params.data_ptr(), B, N, P - 5, H, W, k, out.data_ptr(), _stream()))
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _with_workspace(params, H, W, k):
    img, ws = R.render_fwd(params, H, W, k)
    R.check_device_error(ws)
    return img.cpu().numpy()


def _normwise(a, b):
    worst = 0.0
    for bb in range(b.shape[0]):
        for c in range(b.shape[1]):
            scale = np.abs(b[bb, c]).max()
            err = np.abs(a[bb, c].astype(np.float64) - b[bb, c]).max()
            worst = max(worst, err / scale if scale > 0 else err)
    return worst


def test_noalloc_matches_workspace_entry_point_call_after_call(lib):
    cases = [(WORKLOADS["mono64"], None),
             (WORKLOADS["rgb128"].scaled(B=2), 77),
             (WORKLOADS["mono64"], 5)]
    for w, seed in cases:
        p = torch.from_numpy(make_params(w, seed)).cuda()
        got = _noalloc(lib, p, w.H, w.W, w.k)
        want = _with_workspace(p, w.H, w.W, w.k)
        assert np.isfinite(got).all()
        assert _normwise(got, want) <= FWD_TOL


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    w = WORKLOADS["field32x64"]
    assert R.workspace_bytes(w.B, w.N, w.C, w.H, w.W, w.k) > (16 << 20)
    p = torch.zeros((1, 1, 5 + w.C), device="cuda")
    img = torch.zeros((1, 1, 1, 1), device="cuda")
    st = lib.pdr_render_fwd_noalloc(p.data_ptr(), w.B, w.N, w.C, w.H, w.W, w.k,
                                    img.data_ptr(), _stream())
    assert st == PDR_ERR_TOO_LARGE


def test_noalloc_frame_without_gaussians(lib):
    """N = 0: the image is zeroed (the empty sum), params may be NULL."""
    p = torch.zeros((2, 0, 7), device="cuda")
    got = _noalloc(lib, p, 40, 24, 9)
    assert got.shape == (2, 2, 40, 24) and not got.any()


def test_noalloc_matches_the_oracle(lib):
    w = WORKLOADS["rgb128"].scaled(B=3)
    p_np = make_params(w, 11)
    got = _noalloc(lib, torch.from_numpy(p_np).cuda(), w.H, w.W, w.k)
    ref = oracle.render_fwd(p_np, w.H, w.W, w.k, max(1, oracle.max_threads()))
    assert _normwise(got, ref) <= FWD_TOL


def test_noalloc_allocates_nothing_and_reports_device_errors(lib):
    """After the first call, further calls leave the device's free memory as it
    was; the scratch's device error word reads back clear."""
    w = WORKLOADS["mono64"]
    p = torch.from_numpy(make_params(w, 3)).cuda()
    out = torch.empty((w.B, w.C, w.H, w.W), device="cuda")
    args = (p.data_ptr(), w.B, w.N, w.C, w.H, w.W, w.k, out.data_ptr(), _stream())
    _lib.check("pdr_render_fwd_noalloc", lib.pdr_render_fwd_noalloc(*args))
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        _lib.check("pdr_render_fwd_noalloc", lib.pdr_render_fwd_noalloc(*args))
    _lib.check("pdr_check_device_error_noalloc", lib.pdr_check_device_error_noalloc(_stream()))
    assert torch.cuda.mem_get_info()[0] == free0
