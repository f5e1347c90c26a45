"""Pins of the L1 + SSIM loss oracle (oracle/loss.py) to facts that do not
come from the oracle itself: SSIM(x, x) = 1 with a vanishing gradient, the
closed form of SSIM on constant images, symmetry, a brute-force per-pixel
SSIM written independently, the adjoint identity of the window sum that the
gradient relies on, and central finite differences of the whole loss."""
import math

import numpy as np
import pytest

from oracle import loss as L


def test_window_taps_normalised_and_symmetric():
    g = L.gaussian_taps()
    assert g.shape == (11,)
    assert abs(g.sum() - 1.0) < 1e-15
    assert np.allclose(g, g[::-1], rtol=0, atol=0)
    # ratio of neighbouring taps is the Gaussian's: exp(-(2j+1) / (2 sigma^2))
    for j in range(5):
        assert math.isclose(g[6 + j] / g[5 + j], math.exp(-(2 * j + 1) / (2 * 1.5 ** 2)), rel_tol=1e-13)


def test_ssim_of_an_image_with_itself_is_one_with_zero_gradient():
    rng = np.random.default_rng(0)
    x = rng.uniform(0, 1, (2, 3, 13, 17))
    assert np.allclose(L.ssim_map(x[0, 0], x[0, 0]), 1.0, rtol=0, atol=1e-13)
    loss, grad, (l1, s) = L.l1_ssim_loss(x, x, lam=1.0)
    assert abs(loss) < 1e-13 and abs(s - 1.0) < 1e-13 and l1 == 0.0
    assert np.abs(grad).max() < 1e-12


def test_constant_images_match_the_closed_form_away_from_borders():
    a, b = 0.3, 0.75
    x = np.full((40, 40), a)
    y = np.full((40, 40), b)
    S = L.ssim_map(x, y)
    C1 = 0.01 ** 2
    want = (2 * a * b + C1) / (a * a + b * b + C1)  # variances and covariance vanish
    assert np.allclose(S[5:-5, 5:-5], want, rtol=0, atol=1e-12)
    assert not np.allclose(S[0, 0], want)  # zero padding changes the border


def test_ssim_is_symmetric():
    rng = np.random.default_rng(1)
    x, y = rng.uniform(0, 1, (2, 12, 15))
    assert np.allclose(L.ssim_map(x, y), L.ssim_map(y, x), rtol=0, atol=1e-14)


def _ssim_brute(x, y):
    """Per-pixel SSIM by explicit loops over the window (pure Python)."""
    H, W = x.shape
    g = [math.exp(-(d * d) / (2 * 1.5 ** 2)) for d in range(-5, 6)]
    s = sum(g)
    g = [v / s for v in g]
    C1, C2 = 0.01 ** 2, 0.03 ** 2
    out = np.zeros((H, W))
    for i in range(H):
        for j in range(W):
            m1 = m2 = e11 = e22 = e12 = 0.0
            for dy in range(-5, 6):
                for dx in range(-5, 6):
                    yy, xx = i + dy, j + dx
                    if 0 <= yy < H and 0 <= xx < W:
                        wgt = g[dy + 5] * g[dx + 5]
                        a, b = x[yy, xx], y[yy, xx]
                        m1 += wgt * a
                        m2 += wgt * b
                        e11 += wgt * a * a
                        e22 += wgt * b * b
                        e12 += wgt * a * b
            v1, v2, c12 = e11 - m1 * m1, e22 - m2 * m2, e12 - m1 * m2
            out[i, j] = ((2 * m1 * m2 + C1) * (2 * c12 + C2)) / ((m1 * m1 + m2 * m2 + C1) * (v1 + v2 + C2))
    return out


def test_ssim_map_matches_brute_force():
    rng = np.random.default_rng(2)
    x, y = rng.uniform(0, 1, (2, 7, 9))
    assert np.allclose(L.ssim_map(x, y), _ssim_brute(x, y), rtol=0, atol=1e-13)


def test_window_sum_is_self_adjoint():
    rng = np.random.default_rng(3)
    a, b = rng.standard_normal((2, 14, 19))
    w2 = L.window_2d()
    lhs = (L.window_sum(a, w2) * b).sum()
    rhs = (a * L.window_sum(b, w2)).sum()
    assert math.isclose(lhs, rhs, rel_tol=1e-13)


def test_l1_only():
    rng = np.random.default_rng(4)
    x, y = rng.uniform(0, 1, (2, 2, 3, 6, 5))
    y[0, 0, 0, 0] = x[0, 0, 0, 0]  # a tie: sign(0) = 0
    loss, grad, (l1, _) = L.l1_ssim_loss(x, y, lam=0.0)
    n = x.size
    assert math.isclose(loss, np.abs(x - y).mean(), rel_tol=1e-14)
    assert np.array_equal(grad, np.sign(x - y) / n)
    assert grad[0, 0, 0, 0] == 0.0


@pytest.mark.parametrize("lam", [0.2, 1.0])
def test_gradient_matches_central_differences(lam):
    rng = np.random.default_rng(5)
    x = rng.uniform(0, 1, (2, 2, 9, 11))
    y = np.clip(x + rng.normal(0, 0.2, x.shape), 0, 1)
    _, grad, _ = L.l1_ssim_loss(x, y, lam=lam)
    h = 1e-6
    for idx in [(0, 0, 0, 0), (0, 1, 4, 5), (1, 0, 8, 10), (1, 1, 2, 9), (0, 0, 5, 0), (1, 1, 7, 3)]:
        if abs(x[idx] - y[idx]) < 10 * h:
            continue  # the L1 kink
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        fd = (L.l1_ssim_loss(xp, y, lam=lam)[0] - L.l1_ssim_loss(xm, y, lam=lam)[0]) / (2 * h)
        assert math.isclose(grad[idx], fd, rel_tol=1e-6, abs_tol=1e-11), (idx, grad[idx], fd)


def test_a_plausible_mistake_is_caught():
    """Dropping the covariance term of the gradient breaks the difference check."""
    rng = np.random.default_rng(6)
    x = rng.uniform(0, 1, (1, 1, 9, 9))
    y = rng.uniform(0, 1, (1, 1, 9, 9))
    P = L.ssim_parts(x[0, 0], y[0, 0])
    w2 = L.window_2d()
    n = x.size
    wrong = (L.window_sum(2 * P["my"] * P["N2"] / (P["D1"] * P["D2"]) - 2 * P["mx"] * P["S"] / P["D1"], w2)) / n
    _, grad, _ = L.l1_ssim_loss(x, y, lam=1.0)
    assert not np.allclose(-wrong, grad[0, 0], rtol=1e-3)
