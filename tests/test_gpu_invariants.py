"""Invariants of the CUDA renderer's own outputs, independent of the oracle.

The rendered field I_c(p) = sum_i a_ic exp(-1/2 (p-mu_i)^T Sigma_i^{-1} (p-mu_i))
over each Gaussian's k x k window ("Learning Video Dynamics with Predictive
Differentiable Rendering": abstract -- 5 + C parameters per Gaussian; reading
notes, "Method" -- additive accumulation) is linear in the amplitudes, so the
backward must satisfy the adjoint identity <dL/dI, I> = sum a * dL/da; it is
invariant under theta for isotropic Gaussians; and moving every mean by an
integer pixel offset moves the image by that offset (the window follows
round(mu)).  Bars: fp32 rounding, normwise as in the parity tests.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _api():
    from differentiable_gaussian_splatting_pdr_b200 import api as R
    from differentiable_gaussian_splatting_pdr_b200 import build
    build.build()
    return R


def _render(params, grad, H, W, k):
    R = _api()
    p = torch.from_numpy(np.ascontiguousarray(params)).cuda()
    img, ws = R.render_fwd(p, H, W, k)
    dp = None
    if grad is not None:
        dp = R.render_bwd(p, torch.from_numpy(np.ascontiguousarray(grad)).cuda(), H, W, k, ws)
    R.check_device_error(ws)
    return img.cpu().numpy().astype(np.float64), None if dp is None else dp.cpu().numpy().astype(np.float64)


def _params(rng, B, N, C, H, W, lo=0.0, margin=0.0, iso=False, dyadic=False):
    p = np.empty((B, N, 5 + C), dtype=np.float32)
    p[..., 0] = rng.uniform(lo + margin, W - margin, (B, N))
    p[..., 1] = rng.uniform(lo + margin, H - margin, (B, N))
    if dyadic:  # means on a 1/1024 grid: integer shifts stay exact in fp32
        p[..., :2] = np.round(p[..., :2] * 1024.0) / 1024.0
    p[..., 2] = rng.normal(0.5, 0.4, (B, N))
    p[..., 3] = p[..., 2] if iso else rng.normal(0.5, 0.4, (B, N))
    p[..., 4] = rng.uniform(0, np.pi, (B, N))
    p[..., 5:] = rng.normal(0, 1, (B, N, C))
    return p


def _normwise(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)


@pytest.mark.parametrize("B,N,C,H,W,k", [(2, 500, 3, 48, 80, 9), (1, 3000, 2, 128, 96, 15),
                                         (4, 300, 1, 64, 64, 7)])
def test_adjoint_identity(B, N, C, H, W, k):
    """<g, I> = sum_{i,c} a_ic dL/da_ic, per frame (I is linear in a)."""
    rng = np.random.default_rng(N + k)
    p = _params(rng, B, N, C, H, W)
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    img, dp = _render(p, g, H, W, k)
    for b in range(B):
        lhs = float((g[b].astype(np.float64) * img[b]).sum())
        rhs = float((p[b, :, 5:].astype(np.float64) * dp[b, :, 5:]).sum())
        scale = float((np.abs(g[b]) * np.abs(img[b])).sum())
        assert abs(lhs - rhs) <= 1e-5 * scale, (b, lhs, rhs)


def test_linearity_in_amplitudes():
    """Doubling every amplitude doubles the image (a power of two, the same
    summation order: exact but for subnormal partial sums); a sum of
    amplitude sets renders to the sum."""
    rng = np.random.default_rng(3)
    B, N, C, H, W, k = 2, 800, 3, 64, 48, 11
    p = _params(rng, B, N, C, H, W)
    img, _ = _render(p, None, H, W, k)
    p2 = p.copy()
    p2[..., 5:] *= 2.0
    img2, _ = _render(p2, None, H, W, k)
    assert np.abs(img2 - 2.0 * img).max() <= 1e-30 + 1e-7 * np.abs(img).max()
    pa, pb = p.copy(), p.copy()
    pb[..., 5:] = rng.normal(0, 1, (B, N, C)).astype(np.float32)
    psum = p.copy()
    psum[..., 5:] = pa[..., 5:] + pb[..., 5:]
    ia, _ = _render(pa, None, H, W, k)
    ib, _ = _render(pb, None, H, W, k)
    isum, _ = _render(psum, None, H, W, k)
    assert _normwise(isum, ia + ib) <= 1e-5


def test_isotropic_gaussians_ignore_theta():
    """s_1 = s_2: the image does not depend on theta and dL/dtheta vanishes."""
    rng = np.random.default_rng(4)
    B, N, C, H, W, k = 2, 600, 2, 64, 64, 13
    p = _params(rng, B, N, C, H, W, iso=True)
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    img, dp = _render(p, g, H, W, k)
    q = p.copy()
    q[..., 4] = rng.uniform(-7, 7, (B, N)).astype(np.float32)
    img2, _ = _render(q, None, H, W, k)
    assert _normwise(img2, img) <= 1e-5
    for b in range(B):
        scale = np.abs(dp[b, :, 0:4]).max()
        assert np.abs(dp[b, :, 4]).max() <= 1e-4 * scale


@pytest.mark.parametrize("dx,dy", [(5, 3), (16, 16), (-7, 11)])
def test_integer_shift_moves_the_image(dx, dy):
    """Every mean moved by (dx, dy) whole pixels, windows kept inside the grid:
    the image moves by (dx, dy) and the gradients (with dL/dI moved along)
    stay the same."""
    rng = np.random.default_rng(abs(dx) * 31 + abs(dy))
    B, N, C, H, W, k = 2, 400, 3, 96, 96, 9
    m = (k - 1) // 2 + 1 + 16  # windows stay inside before and after the shift
    p = _params(rng, B, N, C, H, W, margin=m, dyadic=True)
    g = rng.standard_normal((B, C, H, W)).astype(np.float32)
    img, dp = _render(p, g, H, W, k)
    q = p.copy()
    q[..., 0] += dx
    q[..., 1] += dy
    gs = np.roll(np.roll(g, dy, axis=2), dx, axis=3)
    img2, dp2 = _render(q, gs, H, W, k)
    moved = np.roll(np.roll(img, dy, axis=2), dx, axis=3)
    assert _normwise(img2, moved) <= 1e-5
    for b in range(B):
        for j in range(5 + C):
            assert _normwise(dp2[b, :, j], dp[b, :, j]) <= 1e-4, (b, j)
