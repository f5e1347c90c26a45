"""CUDA path vs the fp64 oracle, through the C ABI (via the ctypes binding).

Bars (normwise, per the stated tolerances): forward images within 1e-5 of
max|I_ref| per (frame, channel); gradients within 1e-4 of max|ref| per
parameter field (mu_x, mu_y, s_1, s_2, theta, each a_c) per frame; tile
binning bit-exact.  Inputs are the seeded workloads of inputs.py plus edge
cases (ties at .5, off-grid and non-finite means, k = 1, windows spanning
three tiles, ragged grids, odd widths, long lists, C up to 8, frames without
Gaussians, the largest window with the largest C, a frame of the most tiles
allowed), and the host-buffer step (back to back on one stream, and from two
threads at once).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from differentiable_gaussian_splatting_pdr_b200 import build as pdr_build
from differentiable_gaussian_splatting_pdr_b200 import api as R
from differentiable_gaussian_splatting_pdr_b200.inputs import (WORKLOADS, WORKLOAD_ORDER,
                                                                Workload, make_inputs)

pytestmark = pytest.mark.gpu

FWD_TOL = 1e-5
BWD_TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pdr_build.build()


def threads():
    return max(1, oracle.max_threads())


def fwd_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    B, C = ref.shape[:2]
    worst = 0.0
    for b in range(B):
        for c in range(C):
            scale = np.abs(ref[b, c]).max()
            err = np.abs(gpu[b, c].astype(np.float64) - ref[b, c]).max()
            worst = max(worst, err / scale if scale > 0 else err)
    return worst


def bwd_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    B, N, P = ref.shape
    worst = 0.0
    for b in range(B):
        for j in range(P):
            scale = np.abs(ref[b, :, j]).max()
            err = np.abs(gpu[b, :, j].astype(np.float64) - ref[b, :, j]).max()
            worst = max(worst, err / scale if scale > 0 else err)
    return worst


def run_gpu(params: np.ndarray, grad: np.ndarray, H, W, k):
    p = torch.from_numpy(params).cuda()
    g = torch.from_numpy(grad).cuda()
    img, ws = R.render_fwd(p, H, W, k)
    dp = R.render_bwd(p, g, H, W, k, ws)
    R.check_device_error(ws)
    return img.cpu().numpy(), dp.cpu().numpy()


def check_bins(params: np.ndarray, H, W, k):
    p = torch.from_numpy(params).cuda()
    offs, ids, cap = R.bin_tiles(p, H, W, k)
    offs, ids = offs.cpu().numpy(), ids.cpu().numpy()
    roffs, rids = oracle.bin_tiles(params, H, W, k)
    B = params.shape[0]
    T = offs.shape[1] - 1
    for b in range(B):
        frame_start = roffs[b * T]
        assert offs[b, 0] == b * cap
        for t in range(T):
            got = ids[offs[b, t]:offs[b, t + 1]]
            want = rids[roffs[b * T + t]:roffs[b * T + t + 1]]
            assert np.array_equal(got, want), (b, t)
        assert offs[b, T] - offs[b, 0] == roffs[(b + 1) * T] - frame_start


def check_all(params, grad, H, W, k, bins=True):
    if bins:
        check_bins(params, H, W, k)
    img, dp = run_gpu(params, grad, H, W, k)
    ref_img = oracle.render_fwd(params, H, W, k, threads())
    ref_dp = oracle.render_bwd(params, grad, H, W, k, threads())
    ef, eb = fwd_err(img, ref_img), bwd_err(dp, ref_dp)
    assert ef <= FWD_TOL, ef
    assert eb <= BWD_TOL, eb
    return ef, eb


@pytest.mark.parametrize("name", WORKLOAD_ORDER)
def test_workload_parity_full_size(name):
    """Every workload at its full size: exact bins, all outputs vs the oracle."""
    w = WORKLOADS[name]
    p, g = make_inputs(w)
    check_all(p, g, w.H, w.W, w.k)


@pytest.mark.parametrize("name", ["tiny", "mono64", "rgb128"])
def test_bitwise_reproducible(name):
    w = WORKLOADS[name]
    p, g = make_inputs(w)
    a = run_gpu(p, g, w.H, w.W, w.k)
    b = run_gpu(p, g, w.H, w.W, w.k)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("k", [13, 15])
@pytest.mark.parametrize("H,W", [(48, 64), (45, 50)])
def test_pixel_pair_centres_one_pixel_off_grid(k, H, W):
    """Window centres one pixel past every edge and corner (round(mu) = -1 or W / H), on
    grids of whole tiles (a centre at W then lies 16 pixels into the last tile column,
    inside the pixel-pair backward's staged rows and columns) and ragged ones, next to
    centres two and more pixels off the grid (read from global memory)."""
    rng = np.random.default_rng(30 + k + W)
    B, N, C = 1, 120, 3
    p = _edge_params(rng, B, N, C, H, W, k)
    near = [-0.75, -0.5001, W - 0.25, W - 0.5]           # round(mu) = -1 / W
    nearh = [-0.75, -0.5001, H - 0.25, H - 0.5]
    inside_x, inside_y = rng.uniform(0, W, 40), rng.uniform(0, H, 40)
    xs = np.concatenate([rng.choice(near, 40), inside_x[:20], rng.choice(near, 20)])
    ys = np.concatenate([inside_y[:20], rng.choice(nearh, 40), rng.choice(nearh, 20)])
    p[0, :80, 0], p[0, :80, 1] = xs[:80], ys[:80]
    p[0, 80:100, 0] = rng.choice([-2.6, -4.0, W + 1.6, W + 3.0], 20)  # further off
    p[0, 80:100, 1] = rng.uniform(0, H, 20)
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    check_all(p, g, H, W, k)


@pytest.mark.parametrize("name,B", [("mono64", 4), ("rgb128", 2), ("stress512", 1)])
def test_render_loss_backward_chain_matches_staged(name, B):
    """Forward, L1 + SSIM loss and backward enqueued back to back on one stream (each
    kernel a programmatic dependent launch of the one before, the backward reading the
    loss's dL/dI) give bitwise the results of the same calls with the stream
    synchronised between the stages."""
    w = WORKLOADS[name].scaled(B=B)
    p, _ = make_inputs(w)
    pt = torch.from_numpy(p).cuda()
    rng = np.random.default_rng(40 + B)
    tgt = torch.from_numpy(np.clip(rng.normal(0.5, 0.25, (B, w.C, w.H, w.W)), 0, 1)
                           .astype(np.float32)).cuda()

    def chain(staged):
        img, ws = R.render_fwd(pt, w.H, w.W, w.k)
        if staged:
            torch.cuda.synchronize()
        loss, g = R.l1_ssim_loss(img, tgt)
        if staged:
            torch.cuda.synchronize()
        dp = R.render_bwd(pt, g, w.H, w.W, w.k, ws)
        torch.cuda.synchronize()
        R.check_device_error(ws)
        return img, loss, g, dp

    a, b = chain(False), chain(True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("name", ["tiny", "mono64", "rgb128", "field32x64", "stress512"])
def test_graph_replay_matches_eager(name):
    """Binning, forward and backward captured in one CUDA graph (the kernels are chained
    as programmatic dependent launches, each waiting for its predecessor) and replayed
    several times give bitwise the results of the same calls launched eagerly."""
    w = WORKLOADS[name]
    if name in ("field32x64", "stress512"):
        w = w.scaled(B=4 if name == "field32x64" else 2)
    p, g = make_inputs(w)
    pt, gt = torch.from_numpy(p).cuda(), torch.from_numpy(g).cuda()
    img0, ws = R.render_fwd(pt, w.H, w.W, w.k)
    dp0 = R.render_bwd(pt, gt, w.H, w.W, w.k, ws)
    R.check_device_error(ws)
    img, dp = torch.empty_like(img0), torch.empty_like(dp0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up off the capture
        R.render_fwd(pt, w.H, w.W, w.k, ws, img)
        R.render_bwd(pt, gt, w.H, w.W, w.k, ws, dp)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        R.render_fwd(pt, w.H, w.W, w.k, ws, img)
        R.render_bwd(pt, gt, w.H, w.W, w.k, ws, dp)
    img.zero_()
    dp.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    R.check_device_error(ws)
    assert torch.equal(img, img0) and torch.equal(dp, dp0)


def _edge_params(rng, B, N, C, H, W, k, smean=0.4, ssd=0.4):
    p = np.empty((B, N, 5 + C), dtype=np.float32)
    p[..., 0] = rng.uniform(-k, W + k, (B, N))
    p[..., 1] = rng.uniform(-k, H + k, (B, N))
    p[..., 2] = rng.normal(smean, ssd, (B, N))
    p[..., 3] = rng.normal(smean, ssd, (B, N))
    p[..., 4] = rng.uniform(-7, 7, (B, N))
    p[..., 5:] = rng.normal(0, 1, (B, N, C))
    return p


@pytest.mark.parametrize("B,N,C,H,W,k", [
    (2, 300, 2, 40, 56, 17),    # windows spanning 2x2 tiles, ragged tiles
    (1, 200, 1, 23, 37, 21),    # 3 tiles per axis, ragged both ways, odd width
    (3, 150, 5, 48, 48, 31),    # largest window
    (2, 100, 8, 33, 47, 9),     # C = 8, odd width
    (1, 64, 3, 16, 16, 1),      # single-pixel windows
    (4, 1, 4, 20, 30, 5),       # N = 1
    (1, 500, 6, 7, 9, 3),       # grid smaller than a tile
    # pixel-pair backward (C <= 4, k 13 and 15) and the scalar one beside it, centres on and off the grid
    (2, 400, 3, 40, 56, 15),    # ragged, both window parities, rows wider than a tile
    (1, 300, 4, 23, 37, 9),     # ragged both ways, slots kept per lane
    (2, 200, 1, 33, 47, 11),
    (1, 100, 2, 50, 20, 13),
    (1, 250, 1, 37, 29, 15),
    (3, 80, 3, 16, 16, 3),
    (2, 120, 4, 30, 45, 7),
    (1, 64, 8, 40, 40, 31),     # largest C with the largest window: the biggest backward halo
])
def test_edge_shapes(B, N, C, H, W, k):
    rng = np.random.default_rng(B * 1000 + N + C)
    p = _edge_params(rng, B, N, C, H, W, k)
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    check_all(p, g, H, W, k)


def test_ties_offgrid_and_nonfinite_means():
    rng = np.random.default_rng(7)
    B, N, C, H, W, k = 1, 40, 2, 32, 48, 7
    p = _edge_params(rng, B, N, C, H, W, k)
    p[0, :8, 0] = [0.5, 15.5, np.nextafter(np.float32(16.5), np.float32(0)), -0.5, W - 0.5,
                   np.float32(0.49999997), -3.4999, W + 2.5]
    p[0, :8, 1] = [16.5, 0.5, 31.5, 2.5, -3.5, H - 0.5, 10.0, 5.0]
    p[0, 8:12, 0] = [np.nan, np.inf, 1e30, -1e30]
    p[0, 12:14, 1] = [np.nan, -np.inf]
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    check_all(p, g, H, W, k)
    _, dp = run_gpu(p, g, H, W, k)
    assert np.all(dp[0, 8:14] == 0.0)


def test_long_lists_in_one_tile():
    """Thousands of Gaussians in one tile: several staging batches per block."""
    rng = np.random.default_rng(8)
    B, N, C, H, W, k = 2, 3000, 3, 32, 32, 9
    p = _edge_params(rng, B, N, C, H, W, k)
    p[..., 0] = rng.uniform(3, 12, (B, N))
    p[..., 1] = rng.uniform(3, 12, (B, N))
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    check_all(p, g, H, W, k)


@pytest.mark.parametrize("W", [32, 30])
def test_long_lists_pixel_pair_backward(W):
    """Thousands of home Gaussians in one tile with k = 15: more than the pixel-pair
    backward's record area holds, so the block runs several record rounds; W = 32
    stages dL/dI with vector loads, W = 30 element by element."""
    rng = np.random.default_rng(9 + W)
    B, N, C, H, k = 2, 3000, 3, 32, 15
    p = _edge_params(rng, B, N, C, H, W, k)
    p[..., 0] = rng.uniform(3, 12, (B, N))
    p[..., 1] = rng.uniform(3, 12, (B, N))
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    check_all(p, g, H, W, k)


@pytest.mark.parametrize("k", [7, 9, 11, 13, 15])
@pytest.mark.parametrize("s1,s2", [(-1.0, 2.0), (2.0, -1.0), (-1.5, -1.5)])
def test_backward_row_moments_narrow_and_elongated(k, s1, s2):
    """Narrow and strongly elongated Gaussians on the backward kernels that form the five
    sums of a window column from its row moments (the pixel-pair kernel for k = 13, 15,
    the scalar kernel's column walk for k = 7, 9, 11): the terms of that expansion cancel
    most when the Gaussian is narrow across the column and long along it."""
    rng = np.random.default_rng(20 + k)
    B, N, C, H, W = 2, 300, 3, 48, 64
    p = _edge_params(rng, B, N, C, H, W, k)
    p[..., 2] = rng.normal(s1, 0.2, (B, N))
    p[..., 3] = rng.normal(s2, 0.2, (B, N))
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    check_all(p, g, H, W, k)


def test_autograd_matches_direct_calls():
    w = WORKLOADS["mono64"].scaled(B=3)
    p, g = make_inputs(w)
    pt = torch.from_numpy(p).cuda().requires_grad_(True)
    img = R.render(pt, w.H, w.W, w.k)
    gt = torch.from_numpy(g).cuda()
    (img * gt).sum().backward()
    img2, dp2 = run_gpu(p, g, w.H, w.W, w.k)
    assert np.array_equal(img.detach().cpu().numpy(), img2)
    assert np.array_equal(pt.grad.cpu().numpy(), dp2)


@pytest.mark.parametrize("name,B", [("rgb128", 2), ("stress512", 1), ("stress512", 2),
                                    ("stress512", 5)])
def test_host_step_matches_device_path(name, B):
    """The host step gives bitwise the results of one device-buffer forward +
    backward over the whole batch: in one chunk (small copies), and pipelined
    over chunks of frames (stress512-sized frames: 2 chunks, and 4 uneven ones
    for 5 frames)."""
    w = WORKLOADS[name].scaled(B=B)
    p, g = make_inputs(w)
    hp = torch.from_numpy(p).pin_memory()
    hg = torch.from_numpy(g).pin_memory()
    h_img, h_dp, _ = R.step_host(hp, hg, w.H, w.W, w.k)
    torch.cuda.synchronize()
    img, dp = run_gpu(p, g, w.H, w.W, w.k)
    assert np.array_equal(h_img.numpy(), img)
    assert np.array_equal(h_dp.numpy(), dp)


def test_host_steps_back_to_back_on_one_stream():
    """Consecutive host steps share the device buffers; only the caller's
    stream is synchronised, so the library's side-stream copies must be
    ordered after the previous step and joined back into that stream."""
    w = WORKLOADS["mono64"].scaled(B=4)
    pa, ga = make_inputs(w)
    pb, gb = make_inputs(w.scaled(seed=w.seed + 1))
    ref_a = run_gpu(pa, ga, w.H, w.W, w.k)
    ref_b = run_gpu(pb, gb, w.H, w.W, w.k)
    hosts = [(torch.from_numpy(p).pin_memory(), torch.from_numpy(g).pin_memory())
             for p, g in ((pa, ga), (pb, gb))]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        _, _, bufs = R.step_host(*hosts[0], w.H, w.W, w.k)
        outs = []
        for j in (1, 0, 1):
            mine = dict(bufs)
            mine["h_image"] = torch.empty_like(bufs["h_image"]).pin_memory()
            mine["h_grad_params"] = torch.empty_like(bufs["h_grad_params"]).pin_memory()
            outs.append((j,) + R.step_host(*hosts[j], w.H, w.W, w.k, mine)[:2])
        stream.synchronize()
    for j, h_img, h_dp in outs:
        img, dp = (ref_a, ref_b)[j]
        assert np.array_equal(h_img.numpy(), img)
        assert np.array_equal(h_dp.numpy(), dp)


def test_host_steps_from_two_threads():
    """Two host threads, each with its own stream and buffers, run host steps
    at the same time; each thread's side stream and events are its own."""
    import threading
    w = WORKLOADS["mono64"].scaled(B=3)
    inputs = [make_inputs(w.scaled(seed=w.seed + j)) for j in range(2)]
    refs = [run_gpu(p, g, w.H, w.W, w.k) for p, g in inputs]
    results, errors = [None, None], []

    def worker(j):
        try:
            hp = torch.from_numpy(inputs[j][0]).pin_memory()
            hg = torch.from_numpy(inputs[j][1]).pin_memory()
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                bufs = None
                for _ in range(5):
                    h_img, h_dp, bufs = R.step_host(hp, hg, w.H, w.W, w.k, bufs)
                stream.synchronize()
            results[j] = (h_img.numpy().copy(), h_dp.numpy().copy())
        except Exception as e:  # reported below, in the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(j,)) for j in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for j in range(2):
        assert np.array_equal(results[j][0], refs[j][0])
        assert np.array_equal(results[j][1], refs[j][1])


@pytest.mark.parametrize("B,C,H,W,k", [(2, 3, 40, 24, 9), (3, 1, 64, 64, 9), (1, 4, 128, 96, 15)])
def test_frames_without_gaussians(B, C, H, W, k):
    """N = 0, the empty sum: zero images (every storage type, overwriting what
    was there), no gradients, all-zero tile offsets, also through the host
    step and autograd."""
    rng = np.random.default_rng(B + H)
    p = np.zeros((B, 0, 5 + C), dtype=np.float32)
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    check_bins(p, H, W, k)
    pt, gt = torch.from_numpy(p).cuda(), torch.from_numpy(g).cuda()
    for dtype in (torch.float32, torch.float16, torch.bfloat16):
        out = torch.full((B, C, H, W), 7.0, dtype=dtype, device="cuda")
        img, ws = R.render_fwd(pt, H, W, k, out=out, dtype=dtype)
        dp = R.render_bwd(pt, gt, H, W, k, ws)
        R.check_device_error(ws)
        assert not img.any() and dp.shape == (B, 0, 5 + C)
    offs, ids, cap = R.bin_tiles(pt, H, W, k)
    assert cap == 0 and ids.numel() == 0 and not offs.any()
    h_img, h_dp, _ = R.step_host(torch.from_numpy(p).pin_memory(),
                                 torch.from_numpy(g).pin_memory(), H, W, k)
    torch.cuda.synchronize()
    assert not h_img.any() and h_dp.shape == (B, 0, 5 + C)
    pa = pt.clone().requires_grad_(True)
    (R.render(pa, H, W, k) * gt).sum().backward()
    assert pa.grad is not None and pa.grad.shape == pa.shape


def test_invalid_arguments_rejected_on_device_buffers():
    p = torch.zeros((1, 4, 6), device="cuda")
    with pytest.raises(ValueError):
        R.render_fwd(p, 16, 16, 4)
    with pytest.raises(R._lib.PdrError):
        lib = R._lib.load()
        img = torch.empty((1, 1, 16, 16), device="cuda")
        ws = torch.empty(16, dtype=torch.uint8, device="cuda")
        R._lib.check("pdr_render_fwd", lib.pdr_render_fwd(
            p.data_ptr(), 1, 4, 1, 16, 16, 5, img.data_ptr(), ws.data_ptr(), 16, 0, None))


def test_separate_bins_then_render_matches_one_call():
    w = WORKLOADS["rgb128"].scaled(B=3)
    p, g = make_inputs(w)
    pt, gt = torch.from_numpy(p).cuda(), torch.from_numpy(g).cuda()
    ws = R.build_bins(pt, w.H, w.W, w.k)
    img, _ = R.render_fwd(pt, w.H, w.W, w.k, ws, reuse_bins=True)
    dp = R.render_bwd(pt, gt, w.H, w.W, w.k, ws, reuse_bins=True)
    R.check_device_error(ws)
    img2, dp2 = run_gpu(p, g, w.H, w.W, w.k)
    assert np.array_equal(img.cpu().numpy(), img2)
    assert np.array_equal(dp.cpu().numpy(), dp2)


@pytest.mark.parametrize("B,N,C,H,W,k", [
    (1, 100000, 1, 160, 160, 5),  # 100 tiles, 64-Gaussian slabs, 1563 per frame: the scan's runs exceed its registers
    (2, 20000, 2, 200, 240, 3),   # 195 tiles: 128-Gaussian slabs, a ragged last one
    (1, 20000, 2, 300, 240, 3),   # 285 tiles: 256-Gaussian slabs, a ragged last one
    (1, 3000, 1, 2048, 2048, 5),  # the most tiles a frame may have (16384): one 8192-Gaussian slab, 1-warp blocks
    (3, 1000, 2, 96, 176, 11),    # 66 tiles, few Gaussians
    (2, 30000, 2, 200, 328, 21),  # windows over up to 3 tiles per axis
    (1, 5000, 3, 512, 768, 31),   # the largest window: 1536 tiles, 768-Gaussian slabs counted in three rounds
])
def test_slab_binning_paths(B, N, C, H, W, k):
    """Frames of more than 64 tiles, binned by the slab kernels (records and
    per-slab counts, the prefix over slabs per tile, the per-warp stable
    scatter): slabs of 64 to 8192 Gaussians, windows over 2 and 3 tiles per
    axis, ragged last slabs."""
    rng = np.random.default_rng(N + H)
    p = _edge_params(rng, B, N, C, H, W, k, smean=0.2, ssd=0.3)
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    check_all(p, g, H, W, k)


@pytest.mark.parametrize("B,N,C,H,W,k", [
    (3, 1000, 2, 96, 176, 11),   # 66 tiles, a frame block
    (2, 4000, 1, 144, 128, 9),   # 72 tiles, 4000 ids
    (5, 333, 4, 32, 64, 9),      # 8 tiles: the clustered binner
    (2, 5000, 3, 48, 80, 7),     # 15 tiles: the clustered binner, 5000 ids
    (1, 980, 1, 192, 256, 5),    # 192 tiles, 16-warp frame blocks
])
def test_frame_block_binning(B, N, C, H, W, k):
    """Many frames (B becomes 150 here, at least one frame per SM): frames of 65
    to 256 tiles are binned by one block each, frames of at most 64 tiles by one
    thread-block cluster each; windows partly and wholly off the grid, ragged
    last warp of ids."""
    B = 150
    rng = np.random.default_rng(B * 7 + N + W)
    p = _edge_params(rng, B, N, C, H, W, k)
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    check_all(p, g, H, W, k)


@pytest.mark.parametrize("B,N,C,H,W,k", [
    (1, 300, 2, 16, 16, 9),      # one tile: a cluster of one block
    (4, 5000, 1, 64, 64, 9),     # 16 tiles: 16 blocks, the largest (non-portable) cluster
    (3, 7, 3, 40, 56, 15),       # fewer Gaussians than blocks: empty chunks
    (2, 2501, 4, 33, 47, 7),     # ragged tiles, a chunk size not dividing N
    (2, 3000, 1, 48, 48, 31),    # windows over 3 tiles per axis
    (2, 3000, 3, 64, 128, 11),   # 32 tiles in 16 blocks
    (1, 70000, 1, 64, 64, 5),    # 4375 Gaussians per block: many scatter rounds
    (1, 500, 2, 100, 100, 9),    # 49 tiles, ragged both ways
    (3, 20, 1, 128, 128, 5),     # 64 tiles, the most the clustered binner takes; few Gaussians
])
def test_cluster_binning(B, N, C, H, W, k):
    """Frames of at most 64 tiles, binned by one thread-block cluster of up to 16
    blocks each (chunk counts exchanged through distributed shared memory)."""
    rng = np.random.default_rng(B * 13 + N + W)
    p = _edge_params(rng, B, N, C, H, W, k)
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    check_all(p, g, H, W, k)


@pytest.mark.parametrize("B", [149, 300, 450])
def test_many_small_frames(B):
    """More frames than SMs: smaller frame-binning blocks, one wave."""
    w = WORKLOADS["field32x64"].scaled(B=B, N=300)
    p, g = make_inputs(w)
    check_all(p, g, w.H, w.W, w.k)


@pytest.mark.parametrize("name", ["mono64-grid", "mono64-N256", "mono64-N4096", "mono64-k5",
                                  "mono64-k13", "mono64-k17"])
def test_knob_workloads(name):
    """The knobs the pages name: grid-initialised means, Gaussian count, window size."""
    from differentiable_gaussian_splatting_pdr_b200.inputs import knob_workloads
    w = knob_workloads()[name]
    p, g = make_inputs(w)
    check_all(p, g, w.H, w.W, w.k)


@pytest.mark.parametrize("dtype,bar", [("float16", 1e-3), ("bfloat16", 8e-3)])
@pytest.mark.parametrize("name", ["mono64", "rgb128", "field32x64", "stress512-small"])
def test_reduced_precision_storage(name, dtype, bar):
    """Image and dL/dI stored as fp16 / bf16, sums in fp32: the stored image is
    the fp32 image rounded once; gradients from a half-precision dL/dI match the
    oracle given the same (widened) values at the fp32 bar.  stress512-small
    (one 96 x 128 frame of stress512's distributions, k = 15) takes the
    pixel-pair backward with its element-wise dL/dI staging."""
    import torch
    from differentiable_gaussian_splatting_pdr_b200 import api as R
    tdt = getattr(torch, dtype)
    w = (WORKLOADS["stress512"].scaled(B=1, H=96, W=128, N=3072) if name == "stress512-small"
         else WORKLOADS[name])
    p, g = make_inputs(w)
    dev = torch.device("cuda:0")
    pt = torch.from_numpy(p).to(dev)
    img32, ws = R.render_fwd(pt, w.H, w.W, w.k)
    imgh, _ = R.render_fwd(pt, w.H, w.W, w.k, ws, reuse_bins=True, dtype=tdt)
    torch.cuda.synchronize()
    assert imgh.dtype == tdt
    assert torch.equal(imgh, img32.to(tdt))  # rounded once, to nearest
    ref = oracle.render_fwd(p, w.H, w.W, w.k)
    assert fwd_err(imgh.float().cpu().numpy(), ref) <= bar
    gh = torch.from_numpy(g).to(dev).to(tdt)
    dp = R.render_bwd(pt, gh, w.H, w.W, w.k, ws, reuse_bins=True)
    torch.cuda.synchronize()
    gw = gh.float().cpu().numpy()
    rdp = oracle.render_bwd(p, gw, w.H, w.W, w.k)
    assert bwd_err(dp.cpu().numpy(), rdp) <= 1e-4
