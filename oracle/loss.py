"""fp64 oracle of the L1 + SSIM training loss and its gradient dL/dI.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the CUDA product path
never imports or calls it and shares no code with it.

What it computes.  The pages (reading notes, section "Method", third point;
section "Key Insight / Why It Works") state that PDR trains the rendered
field with an L1 + SSIM objective and that this pairing is essential, but
give neither the weights nor the SSIM constants.  Readings taken here (the
plainest ones, those of the usual Gaussian-splatting training loss):

    L = (1 - lam) * mean |I - T|  +  lam * (1 - mean SSIM(I, T)),  lam = 0.2 by default,

with SSIM the structural-similarity index of Wang et al. (2004) computed per
(frame, channel) image: local means, variances and covariance from an 11 x 11
Gaussian window (sigma 1.5, taps normalised to sum 1), zero padding at the
borders ("same" size maps), C1 = (0.01 * L)^2, C2 = (0.03 * L)^2 with data
range L = 1, and the mean taken over every pixel of every channel and frame.

The gradient is the exact derivative of that definition: with the window
moments mu_x = G * x, E_xx = G * x^2, E_xy = G * (x y) (and the same for y),
the SSIM map S(p) = N1 N2 / (D1 D2), N1 = 2 mu_x mu_y + C1, N2 = 2 s_xy + C2,
D1 = mu_x^2 + mu_y^2 + C1, D2 = s_xx + s_yy + C2, and since every moment is
a window sum of x,

    dS_mean / dx(q) = (1/n) [ (G * A)(q) + 2 x(q) (G * B)(q) + y(q) (G * Cxy)(q) ],
    A = dS/dmu_x - 2 mu_x dS/ds_xx - mu_y dS/ds_xy,   B = dS/ds_xx,   Cxy = dS/ds_xy,
    dS/dmu_x = 2 mu_y N2 / (D1 D2) - 2 mu_x S / D1,  dS/ds_xx = -S / D2,  dS/ds_xy = 2 N1 / (D1 D2),

where G * is the zero-padded window sum (the window is symmetric, so the
adjoint of the forward window sum is the same operation).  The L1 term
contributes (1 - lam) sign(I - T) / n (sign(0) = 0).

Parity status: pinned by tests/test_loss_oracle_pins.py (SSIM(x, x) = 1 with a
zero gradient, the closed form on constant images, symmetry, a brute-force
per-pixel SSIM, the window's adjoint identity, and central finite
differences of the whole loss).  No function here is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

WINDOW = 11
SIGMA = 1.5
K1, K2 = 0.01, 0.03
DEFAULT_LAMBDA = 0.2


def gaussian_taps(size: int = WINDOW, sigma: float = SIGMA) -> np.ndarray:
    """1D Gaussian window taps, centred, normalised to sum 1 (fp64)."""
    r = (size - 1) // 2
    x = np.arange(-r, r + 1, dtype=np.float64)
    t = np.exp(-(x * x) / (2.0 * sigma * sigma))
    return t / t.sum()


def window_2d(size: int = WINDOW, sigma: float = SIGMA) -> np.ndarray:
    """The 2D window: outer product of the 1D taps."""
    g = gaussian_taps(size, sigma)
    return np.outer(g, g)


def window_sum(img: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """Zero-padded, same-size window sum out(p) = sum_o w2[o] img[p + o - r]
    over the last two axes of img (each 2D image on its own), written out
    over the window offsets (fp64)."""
    kh, kw = w2.shape
    ry, rx = (kh - 1) // 2, (kw - 1) // 2
    H, W = img.shape[-2:]
    pad = np.zeros(img.shape[:-2] + (H + 2 * ry, W + 2 * rx), dtype=np.float64)
    pad[..., ry:ry + H, rx:rx + W] = img
    out = np.zeros(img.shape, dtype=np.float64)
    for dy in range(kh):
        for dx in range(kw):
            out += w2[dy, dx] * pad[..., dy:dy + H, dx:dx + W]
    return out


def ssim_parts(x: np.ndarray, y: np.ndarray, data_range: float = 1.0):
    """Window moments and the SSIM map of image pairs (last two axes, fp64)."""
    w2 = window_2d()
    C1 = (K1 * data_range) ** 2
    C2 = (K2 * data_range) ** 2
    mx, my = window_sum(x, w2), window_sum(y, w2)
    sxx = window_sum(x * x, w2) - mx * mx
    syy = window_sum(y * y, w2) - my * my
    sxy = window_sum(x * y, w2) - mx * my
    N1 = 2.0 * mx * my + C1
    N2 = 2.0 * sxy + C2
    D1 = mx * mx + my * my + C1
    D2 = sxx + syy + C2
    S = (N1 * N2) / (D1 * D2)
    return dict(mx=mx, my=my, sxx=sxx, syy=syy, sxy=sxy, N1=N1, N2=N2, D1=D1, D2=D2, S=S)


def ssim_map(x: np.ndarray, y: np.ndarray, data_range: float = 1.0) -> np.ndarray:
    return ssim_parts(np.asarray(x, np.float64), np.asarray(y, np.float64), data_range)["S"]


def l1_ssim_loss(image: np.ndarray, target: np.ndarray, lam: float = DEFAULT_LAMBDA,
                 data_range: float = 1.0):
    """Loss and dL/dI for image, target of shape [B, C, H, W] (read as fp64).

    Returns (loss, grad, parts) with parts = (mean |I - T|, mean SSIM)."""
    x = np.asarray(image, dtype=np.float64)
    y = np.asarray(target, dtype=np.float64)
    B, C, H, W = x.shape
    n = float(B * C * H * W)
    w2 = window_2d()
    l1 = np.abs(x - y).sum() / n
    grad = (1.0 - lam) * np.sign(x - y) / n
    P = ssim_parts(x, y, data_range)  # every (frame, channel) image on its own
    S, N1, N2, D1, D2 = P["S"], P["N1"], P["N2"], P["D1"], P["D2"]
    dS_dmx = 2.0 * P["my"] * N2 / (D1 * D2) - 2.0 * P["mx"] * S / D1
    dS_dsxx = -S / D2
    dS_dsxy = 2.0 * N1 / (D1 * D2)
    A = dS_dmx - 2.0 * P["mx"] * dS_dsxx - P["my"] * dS_dsxy
    dssim = (window_sum(A, w2) + 2.0 * x * window_sum(dS_dsxx, w2)
             + y * window_sum(dS_dsxy, w2)) / n
    grad -= lam * dssim
    ssim_mean = S.sum() / n
    loss = (1.0 - lam) * l1 + lam * (1.0 - ssim_mean)
    return loss, grad, (l1, ssim_mean)
