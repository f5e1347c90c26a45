"""CUDA L1 + SSIM loss (pdr_loss_l1_ssim) vs the fp64 oracle (oracle/loss.py).

Bars as for the renderer: the loss within 1e-5 relative, dL/dI within 1e-4
normwise per (frame, channel) image (fp32 vs fp64); bitwise reproducible."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from oracle import loss as oracle_loss  # noqa: E402


def _api():
    from differentiable_gaussian_splatting_pdr_b200 import api as R
    from differentiable_gaussian_splatting_pdr_b200 import build
    build.build()
    return R


def _pair(rng, B, C, H, W, noise=0.1):
    x = rng.uniform(0, 1, (B, C, H, W)).astype(np.float32)
    y = np.clip(x + rng.normal(0, noise, x.shape), 0, 1).astype(np.float32)
    return x, y


def _gpu(x, y, lam):
    R = _api()
    dev = torch.device("cuda:0")
    xt, yt = torch.from_numpy(x).to(dev), torch.from_numpy(y).to(dev)
    loss, grad = R.l1_ssim_loss(xt, yt, lam)
    torch.cuda.synchronize()
    return float(loss.item()), grad.cpu().numpy()


def _check(x, y, lam):
    loss, grad = _gpu(x, y, lam)
    rl, rg, _ = oracle_loss.l1_ssim_loss(x, y, lam)
    assert abs(loss - rl) <= 1e-5 * max(abs(rl), 1e-3), (loss, rl)
    B, C = x.shape[:2]
    for b in range(B):
        for c in range(C):
            ref = rg[b, c]
            err = np.abs(grad[b, c] - ref).max() / max(np.abs(ref).max(), 1e-30)
            assert err <= 1e-4, (b, c, err)


@pytest.mark.parametrize("B,C,H,W", [
    (1, 1, 32, 32),     # one tile
    (2, 3, 37, 45),     # ragged tiles
    (1, 2, 8, 5),       # smaller than the window
    (3, 4, 32, 64),     # lat-lon-shaped field frames
    (16, 1, 64, 64),    # the mono64 frames
    (2, 3, 128, 96),
])
@pytest.mark.parametrize("lam", [0.0, 0.2, 1.0])
def test_loss_matches_oracle(B, C, H, W, lam):
    rng = np.random.default_rng(B * 100 + C * 10 + H + W)
    x, y = _pair(rng, B, C, H, W)
    _check(x, y, lam)


def test_full_size_field_frames():
    """320 frames x 4 channels of 32 x 64, as the lat-lon field workload."""
    rng = np.random.default_rng(11)
    x, y = _pair(rng, 320, 4, 32, 64, noise=0.05)
    _check(x, y, 0.2)


def test_smooth_bright_images():
    """Large means, small variances: the regime where fp32 moments cancel."""
    rng = np.random.default_rng(12)
    yy, xx = np.mgrid[0:48, 0:80]
    base = 0.9 + 0.05 * np.sin(xx / 7.0) * np.cos(yy / 5.0)
    x = (base + rng.normal(0, 0.002, (2, 2, 48, 80))).astype(np.float32)
    y = (base + rng.normal(0, 0.002, (2, 2, 48, 80))).astype(np.float32)
    _check(x, y, 0.2)


def test_identical_images_give_zero():
    rng = np.random.default_rng(13)
    x, _ = _pair(rng, 2, 2, 40, 40)
    loss, grad = _gpu(x, x.copy(), 0.2)
    assert abs(loss) < 1e-6
    assert np.abs(grad).max() < 1e-9


def test_reproducible_and_autograd():
    R = _api()
    rng = np.random.default_rng(14)
    x, y = _pair(rng, 2, 3, 50, 70)
    dev = torch.device("cuda:0")
    xt, yt = torch.from_numpy(x).to(dev), torch.from_numpy(y).to(dev)
    l1, g1 = R.l1_ssim_loss(xt, yt)
    l2, g2 = R.l1_ssim_loss(xt, yt)
    assert torch.equal(l1, l2) and torch.equal(g1, g2)
    xa = xt.clone().requires_grad_(True)
    out = R.l1_ssim(xa, yt) * 3.0
    out.backward()
    assert torch.allclose(out, 3.0 * l1[0])
    assert torch.equal(xa.grad, 3.0 * g1)


def test_rejects_bad_arguments():
    R = _api()
    from differentiable_gaussian_splatting_pdr_b200 import _lib
    lib = _lib.load()
    dev = torch.device("cuda:0")
    x = torch.rand(1, 1, 16, 16, device=dev)
    ws = torch.empty(4096, dtype=torch.uint8, device=dev)
    out = torch.empty(1, device=dev)
    g = torch.empty_like(x)
    s = torch.cuda.current_stream().cuda_stream
    args = lambda lam, dr, nb: (x.data_ptr(), x.data_ptr(), 1, 1, 16, 16, lam, dr, out.data_ptr(),
                                g.data_ptr(), ws.data_ptr(), nb, s)
    assert lib.pdr_loss_l1_ssim(*args(1.5, 1.0, 4096)) == _lib.STATUS_CODES["PDR_ERR_INVALID_ARG"]
    assert lib.pdr_loss_l1_ssim(*args(0.2, 0.0, 4096)) == _lib.STATUS_CODES["PDR_ERR_INVALID_ARG"]
    assert lib.pdr_loss_l1_ssim(*args(0.2, 1.0, 0)) == _lib.STATUS_CODES["PDR_ERR_WORKSPACE_TOO_SMALL"]
    with pytest.raises(ValueError):
        R.l1_ssim_loss(x, torch.rand(1, 1, 16, 8, device=dev))
