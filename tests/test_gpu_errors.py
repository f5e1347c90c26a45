"""The device error word: kernels only set its bits (a bounds check that
fires), binning clears it stream-ordered before its first kernel, and
pdr_check_device_error reads and clears it.  A bad tile offset planted from
the host into built bins must be reported, and must not disturb the tiles
whose list ranges are intact (they still match the oracle).

The planted offset lies far outside the frame's list region; every kernel
validates a tile's list range before it reads a list entry or a record, so
nothing out of bounds is touched.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from differentiable_gaussian_splatting_pdr_b200 import _lib
from differentiable_gaussian_splatting_pdr_b200 import api as R
from differentiable_gaussian_splatting_pdr_b200 import build as pdr_build
from differentiable_gaussian_splatting_pdr_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

PDR_ERR_INTERNAL = 5


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pdr_build.build()


@pytest.mark.parametrize("name", ["mono64", "rgb128", "stress512"])
def test_bad_tile_offset_is_reported_and_other_tiles_stay_right(name):
    w = WORKLOADS[name]
    w = w.scaled(B=min(w.B, 4))
    p, g = make_inputs(w)
    B, N, C, H, W, k = w.B, w.N, w.C, w.H, w.W, w.k
    T = w.tiles
    TX = (W + 15) // 16
    pt, gt = torch.from_numpy(p).cuda(), torch.from_numpy(g).cuda()
    ws = R.build_bins(pt, H, W, k)
    R.check_device_error(ws)  # clean bins
    # Plant an offset far beyond every frame's region: tile t of frame b
    # (and tile t - 1, whose end it is) must then render as empty lists.
    b, t = B - 1, T // 2 + TX // 2
    off, nbytes = R.workspace_part(B, N, C, H, W, k, "tile_offsets")
    assert nbytes == 4 * B * (T + 1)
    bad = torch.tensor([2 ** 30], dtype=torch.int32)
    dst = ws.buf[off + 4 * (b * (T + 1) + t): off + 4 * (b * (T + 1) + t) + 4]
    dst.copy_(bad.view(torch.uint8))
    img, _ = R.render_fwd(pt, H, W, k, ws, reuse_bins=True)
    dp = R.render_bwd(pt, gt, H, W, k, ws, reuse_bins=True)
    lib = _lib.load()
    st = lib.pdr_check_device_error(ws.buf.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == PDR_ERR_INTERNAL
    # read and cleared: a second check is clean
    R.check_device_error(ws)

    ref = oracle.render_fwd(p, H, W, k, max(1, oracle.max_threads()))
    got = img.cpu().numpy()
    bad_tiles = {t - 1, t}
    mask = np.ones((H, W), bool)
    for tt in bad_tiles:
        ty, tx = divmod(tt, TX)
        mask[16 * ty:16 * ty + 16, 16 * tx:16 * tx + 16] = False
    for bb in range(B):
        for c in range(C):
            scale = np.abs(ref[bb, c]).max()
            m = mask if bb == b else np.ones((H, W), bool)
            err = np.abs(got[bb, c][m] - ref[bb, c][m]).max() / scale
            assert err <= 1e-5, (bb, c, err)
        if bb == b:
            for tt in bad_tiles:  # those tiles rendered as empty lists
                ty, tx = divmod(tt, TX)
                assert not got[bb, :, 16 * ty:16 * ty + 16, 16 * tx:16 * tx + 16].any()
    # Gradients of Gaussians whose home tile kept a valid list match the oracle.
    ref_dp = oracle.render_bwd(p, g, H, W, k, max(1, oracle.max_threads()))
    dpn = dp.cpu().numpy()
    cx = np.clip(np.floor(p[..., 0].astype(np.float64) + 0.5), 0, W - 1).astype(int) // 16
    cy = np.clip(np.floor(p[..., 1].astype(np.float64) + 0.5), 0, H - 1).astype(int) // 16
    home = cy * TX + cx
    for bb in range(B):
        keep = np.ones(N, bool) if bb != b else ~np.isin(home[bb], list(bad_tiles))
        for j in range(5 + C):
            scale = np.abs(ref_dp[bb, :, j]).max()
            err = np.abs(dpn[bb, keep, j] - ref_dp[bb, keep, j]).max() / scale
            assert err <= 1e-4, (bb, j, err)


def test_binning_clears_the_word_before_its_kernels():
    """A set word is cleared by the next binning call (stream-ordered)."""
    w = WORKLOADS["tiny"]
    p, _ = make_inputs(w)
    pt = torch.from_numpy(p).cuda()
    ws = R.build_bins(pt, w.H, w.W, w.k)
    off, _ = R.workspace_part(w.B, w.N, w.C, w.H, w.W, w.k, "error_word")
    ws.buf[off:off + 4].copy_(torch.tensor([1], dtype=torch.int32).view(torch.uint8))
    R.build_bins(pt, w.H, w.W, w.k, ws)
    R.check_device_error(ws)
