"""Pins for the fp64 oracle, each against something other than the oracle.

The rendered field is I_c(p) = sum_i a_ic exp(-1/2 (p-mu_i)^T Sigma_i^{-1} (p-mu_i)),
Sigma_i = R(theta_i) diag(e^{2 s_i}) R(theta_i)^T, truncated to the k x k window
around round(mu_i), accumulated additively ("Learning Video Dynamics with
Predictive Differentiable Rendering": abstract -- 5 + C parameters per
Gaussian; reading notes, "Method" -- additive accumulation; "Key Insight" /
"Limitation" -- kernel size / support).  The pages print no worked example, so
the pins are mathematical: closed forms, an independent covariance-matrix
evaluation, exact rational rounding, invariants, the adjoint identity, central
finite differences and brute-force window indicators.  Each is chosen so that a
plausible slip (a dropped term, a swapped axis or scale, a wrong sign of the
rotation, an off-by-one window, ties rounded the wrong way) fails one of them.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from differentiable_gaussian_splatting_pdr_b200.inputs import WORKLOADS, make_inputs


def gauss(mx, my, s1, s2, th, amps, dtype=np.float32):
    row = [mx, my, s1, s2, th] + list(amps)
    return np.asarray(row, dtype=dtype)[None, None, :]


def stack(rows, dtype=np.float32):
    return np.concatenate([np.asarray(r, dtype=dtype).reshape(1, 1, -1) for r in rows], axis=1)


def exact_round_half_up(v: float) -> int:
    """round(v) with ties up, in exact rational arithmetic."""
    return math.floor(Fraction(float(v)) + Fraction(1, 2))


# --------------------------------------------------------------------------
# 1. Closed form: an untruncated Gaussian on a large grid sums to 2 pi e^{s1+s2} a
#    (isotropic case 2 pi e^{2s} a).  Poisson summation bounds the lattice-sum
#    error by ~4 exp(-2 pi^2 min eig(Sigma)) <= 1.1e-8 relative for s >= 0.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("s1,s2,th,mx,my", [
    (0.0, 0.0, 0.3, 47.3, 48.7),
    (0.5, 0.5, 1.1, 48.49, 47.51),
    (0.2, 0.7, 0.6, 48.2, 47.9),
    (0.7, 0.1, 2.5, 47.8, 48.3),
    (0.05, 0.4, 3.0, 48.0, 48.0),
])
def test_total_mass_closed_form(s1, s2, th, mx, my):
    amps = [1.7, -0.4, 2.5]
    smax = max(s1, s2)
    k = 2 * math.ceil(10.0 * math.exp(smax)) + 1
    p = gauss(mx, my, s1, s2, th, amps)
    img = oracle.render_fwd(p, 96, 96, k)
    s1f, s2f = float(p[0, 0, 2]), float(p[0, 0, 3])
    for c, a in enumerate(p[0, 0, 5:]):
        mass = 2.0 * math.pi * float(a) * math.exp(s1f + s2f)
        assert abs(img[0, c].sum() - mass) <= 1e-7 * abs(mass)


# --------------------------------------------------------------------------
# 2. Closed form: at theta = 0 the weight factorises, so the truncated, clipped
#    image is a * outer(f_y, f_x) of two independently computed 1-D profiles
#    (s_1 acts along x, s_2 along y).  At theta = pi/2 the roles swap.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("mx,my,k,H,W", [
    (5.3, 7.8, 7, 16, 20),
    (0.2, 15.6, 9, 16, 16),
    (19.5, 2.5, 5, 12, 20),
    (-2.3, 3.4, 9, 10, 12),
    (11.49, 9.51, 11, 13, 17),
    (3.0, 3.0, 1, 8, 8),
])
@pytest.mark.parametrize("quarter_turn", [False, True])
def test_separable_truncated_window(mx, my, k, H, W, quarter_turn):
    s1, s2, a = 0.4, -0.3, 1.3
    th = math.pi / 2 if quarter_turn else 0.0
    p = gauss(mx, my, s1, s2, th, [a], dtype=np.float64)
    img = oracle.render_fwd(p, H, W, k)[0, 0]
    r = (k - 1) // 2
    cx, cy = exact_round_half_up(mx), exact_round_half_up(my)
    xs = np.array([x for x in range(W) if abs(x - cx) <= r], dtype=np.float64)
    ys = np.array([y for y in range(H) if abs(y - cy) <= r], dtype=np.float64)
    sx, sy = (s2, s1) if quarter_turn else (s1, s2)
    fx = np.exp(-0.5 * (xs - mx) ** 2 * math.exp(-2 * sx))
    fy = np.exp(-0.5 * (ys - my) ** 2 * math.exp(-2 * sy))
    want = np.zeros((H, W))
    if len(xs) and len(ys):
        want[np.ix_(ys.astype(int), xs.astype(int))] = a * np.outer(fy, fx)
    np.testing.assert_allclose(img, want, rtol=1e-13, atol=1e-300)


# --------------------------------------------------------------------------
# 3. Independent evaluation of the stated formula with an explicit covariance
#    matrix and a numerical inverse (dense over the grid, masked by the window
#    computed with exact rational rounding).  Pins the rotation direction, the
#    scale-to-axis assignment and the amplitude channels for arbitrary theta.
# --------------------------------------------------------------------------
def dense_reference(params, H, W, k):
    params = np.asarray(params, dtype=np.float64)
    B, N, P = params.shape
    C = P - 5
    r = (k - 1) // 2
    ys, xs = np.mgrid[0:H, 0:W].astype(np.float64)
    out = np.zeros((B, C, H, W))
    for b in range(B):
        for i in range(N):
            mx, my, s1, s2, th = params[b, i, :5]
            if not (np.isfinite(mx) and np.isfinite(my)):
                continue
            R = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
            Sigma = R @ np.diag([math.exp(2 * s1), math.exp(2 * s2)]) @ R.T
            Si = np.linalg.inv(Sigma)
            dx, dy = xs - mx, ys - my
            q = Si[0, 0] * dx * dx + (Si[0, 1] + Si[1, 0]) * dx * dy + Si[1, 1] * dy * dy
            w = np.exp(-0.5 * q)
            cx, cy = exact_round_half_up(mx), exact_round_half_up(my)
            mask = (np.abs(xs - cx) <= r) & (np.abs(ys - cy) <= r)
            for c in range(C):
                out[b, c] += np.where(mask, params[b, i, 5 + c] * w, 0.0)
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_covariance_matrix_form(seed):
    rng = np.random.default_rng(100 + seed)
    B, N, C, H, W, k = 2, 9, 2, 21, 27, 9
    p = np.empty((B, N, 5 + C), dtype=np.float32)
    p[..., 0] = rng.uniform(-3, W + 3, (B, N))
    p[..., 1] = rng.uniform(-3, H + 3, (B, N))
    p[..., 2] = rng.normal(0.5, 0.5, (B, N))
    p[..., 3] = rng.normal(0.5, 0.5, (B, N))
    p[..., 4] = rng.uniform(-4, 4, (B, N))
    p[..., 5:] = rng.normal(0, 1, (B, N, C))
    got = oracle.render_fwd(p, H, W, k)
    want = dense_reference(p, H, W, k)
    scale = np.abs(want).max()
    assert np.abs(got - want).max() <= 1e-12 * scale


def test_covariance_pin_catches_the_slips_it_targets():
    """A rotation of the wrong sense, swapped scales, or a window one pixel too
    small, planted in the independent reference, moves it far outside the
    covariance pin's 1e-12 bar: the pin can tell the oracle from each slip."""
    rng = np.random.default_rng(7)
    B, N, C, H, W, k = 1, 9, 2, 21, 27, 9
    p = np.empty((B, N, 5 + C), dtype=np.float32)
    p[..., 0] = rng.uniform(4, W - 4, (B, N))
    p[..., 1] = rng.uniform(4, H - 4, (B, N))
    p[..., 2] = rng.normal(0.8, 0.3, (B, N))
    p[..., 3] = p[..., 2] - 0.7                      # clearly anisotropic
    p[..., 4] = rng.uniform(0.3, 1.2, (B, N))        # away from multiples of pi/2
    p[..., 5:] = rng.normal(0, 1, (B, N, C))
    got = oracle.render_fwd(p, H, W, k)
    scale = np.abs(got).max()
    flipped = p.copy()
    flipped[..., 4] *= -1.0
    swapped = p.copy()
    swapped[..., [2, 3]] = p[..., [3, 2]]
    for slip in (dense_reference(flipped, H, W, k), dense_reference(swapped, H, W, k),
                 dense_reference(p, H, W, k - 2)):
        assert np.abs(got - slip).max() > 1e-3 * scale


def test_rotation_direction_on_diagonals():
    """theta = pi/4: the first axis (scale e^{s_1}) points along (1, 1) in (x, y)."""
    s1, s2 = 0.9, -0.2
    p = gauss(20.0, 20.0, s1, s2, math.pi / 4, [1.0], dtype=np.float64)
    img = oracle.render_fwd(p, 40, 40, 15)[0, 0]
    for t in (1, 2, 3):
        along = math.exp(-0.5 * (2 * t * t) * math.exp(-2 * s1))
        across = math.exp(-0.5 * (2 * t * t) * math.exp(-2 * s2))
        assert img[20 + t, 20 + t] == pytest.approx(along, rel=1e-13)
        assert img[20 - t, 20 + t] == pytest.approx(across, rel=1e-13)


# --------------------------------------------------------------------------
# 4. Window centre: round half up, evaluated exactly on the fp32 value.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("mu32,centre", [
    (np.float32(10.5), 11),
    (np.nextafter(np.float32(10.5), np.float32(0)), 10),
    (np.float32(0.49999997), 0),     # fl32(mu + 0.5) would round this to 1
    (np.float32(-0.5), 0),
    (np.float32(-1.5), -1),
    (np.float32(7.0), 7),
    (np.nextafter(np.float32(7.5), np.float32(100)), 8),
])
def test_window_centre_rounding(mu32, centre):
    k, W = 5, 24
    p = gauss(float(mu32), 3.0, 4.0, 4.0, 0.0, [1.0])
    assert p[0, 0, 0] == mu32
    img = oracle.render_fwd(p, 8, W, k)[0, 0]
    cols = set(np.nonzero(img.sum(axis=0))[0].tolist())
    assert cols == {x for x in range(W) if abs(x - centre) <= 2}
    assert centre == exact_round_half_up(mu32)


def test_nonfinite_and_far_means_contribute_nothing():
    rows = [[np.nan, 3.0, 0.0, 0.0, 0.0, 1.0],
            [3.0, np.inf, 0.0, 0.0, 0.0, 1.0],
            [-np.inf, 3.0, 0.0, 0.0, 0.0, 1.0],
            [1e30, 3.0, 0.0, 0.0, 0.0, 1.0],
            [-20.0, 3.0, 0.0, 0.0, 0.0, 1.0],   # window [-22, -18] misses the grid
            [3.0, 12.6, 0.0, 0.0, 0.0, 1.0]]    # window [11, 15] misses rows 0..9
    p = stack(rows)
    g = np.ones((1, 1, 10, 10), dtype=np.float32)
    assert np.all(oracle.render_fwd(p, 10, 10, 5) == 0.0)
    assert np.all(oracle.render_bwd(p, g, 10, 10, 5) == 0.0)
    offs, ids = oracle.bin_tiles(p, 10, 10, 5)
    assert len(ids) == 0 and np.all(offs == 0)


# --------------------------------------------------------------------------
# 5. Invariants.
# --------------------------------------------------------------------------
def _random_params(seed, B=2, N=12, C=3, H=24, W=28):
    rng = np.random.default_rng(seed)
    p = np.empty((B, N, 5 + C), dtype=np.float64)
    p[..., 0] = rng.uniform(0, W, (B, N))
    p[..., 1] = rng.uniform(0, H, (B, N))
    p[..., 2] = rng.normal(0.5, 0.5, (B, N))
    p[..., 3] = rng.normal(0.5, 0.5, (B, N))
    p[..., 4] = rng.uniform(0, np.pi, (B, N))
    p[..., 5:] = rng.normal(0, 1, (B, N, C))
    return p, H, W


def test_linearity_in_amplitudes():
    p, H, W = _random_params(1)
    q = p.copy()
    q[..., 5:] = np.random.default_rng(2).normal(0, 1, q[..., 5:].shape)
    mix = p.copy()
    mix[..., 5:] = 2.5 * p[..., 5:] - 0.75 * q[..., 5:]
    lhs = oracle.render_fwd(mix, H, W, 9)
    rhs = 2.5 * oracle.render_fwd(p, H, W, 9) - 0.75 * oracle.render_fwd(q, H, W, 9)
    assert np.abs(lhs - rhs).max() <= 1e-13 * np.abs(rhs).max()


def test_channel_independence():
    p, H, W = _random_params(3)
    full = oracle.render_fwd(p, H, W, 7)
    for c in range(p.shape[2] - 5):
        one = np.concatenate([p[..., :5], p[..., 5 + c:6 + c]], axis=2)
        np.testing.assert_array_equal(oracle.render_fwd(one, H, W, 7)[:, 0], full[:, c])


def test_additivity_over_gaussian_sets():
    p, H, W = _random_params(4)
    a, b = p[:, :5], p[:, 5:]
    both = oracle.render_fwd(p, H, W, 9)
    parts = oracle.render_fwd(a, H, W, 9) + oracle.render_fwd(b, H, W, 9)
    assert np.abs(both - parts).max() <= 1e-13 * np.abs(both).max()


def test_a_frame_without_gaussians():
    """N = 0, the empty sum: an all-zero image, no gradients, empty tile lists;
    and splitting a set into itself and the empty set changes nothing."""
    p, H, W = _random_params(4)
    empty = p[:, :0]
    img = oracle.render_fwd(empty, H, W, 9)
    assert img.shape == (p.shape[0], p.shape[2] - 5, H, W) and not img.any()
    g = np.random.default_rng(9).standard_normal(img.shape).astype(np.float32)
    assert oracle.render_bwd(empty, g, H, W, 9).shape == (p.shape[0], 0, p.shape[2])
    offs, ids = oracle.bin_tiles(empty, H, W, 9)
    assert not offs.any() and ids.size == 0
    assert np.array_equal(oracle.render_fwd(p, H, W, 9), oracle.render_fwd(p, H, W, 9) + img)


def test_isotropic_theta_invariance_and_zero_theta_grad():
    p, H, W = _random_params(5)
    p[..., 3] = p[..., 2]
    q = p.copy()
    q[..., 4] += 0.7
    I1, I2 = oracle.render_fwd(p, H, W, 9), oracle.render_fwd(q, H, W, 9)
    assert np.abs(I1 - I2).max() <= 1e-13 * np.abs(I1).max()
    g = np.random.default_rng(6).normal(0, 1, I1.shape)
    d = oracle.render_bwd(p, g, H, W, 9)
    assert np.abs(d[..., 4]).max() <= 1e-12 * np.abs(d).max()


def test_theta_period_pi_and_quarter_turn_swaps_scales():
    p, H, W = _random_params(7)
    I0 = oracle.render_fwd(p, H, W, 9)
    q = p.copy()
    q[..., 4] += np.pi
    assert np.abs(oracle.render_fwd(q, H, W, 9) - I0).max() <= 1e-12 * np.abs(I0).max()
    s = p.copy()
    s[..., 4] += np.pi / 2
    s[..., 2], s[..., 3] = p[..., 3].copy(), p[..., 2].copy()
    assert np.abs(oracle.render_fwd(s, H, W, 9) - I0).max() <= 1e-12 * np.abs(I0).max()


def test_integer_shift_equivariance():
    rng = np.random.default_rng(8)
    N, H, W, k = 10, 40, 40, 7
    p = np.empty((1, N, 6), dtype=np.float32)
    p[..., 0] = rng.uniform(12, 22, (1, N))
    p[..., 1] = rng.uniform(12, 22, (1, N))
    p[..., 2:4] = rng.normal(0.3, 0.3, (1, N, 2))
    p[..., 4] = rng.uniform(0, 3, (1, N))
    p[..., 5] = rng.normal(0, 1, (1, N))
    p = p.astype(np.float64)        # so that mu + 5 is exact
    q = p.copy()
    q[..., 0] += 5
    q[..., 1] += 3
    I0 = oracle.render_fwd(p, H, W, k)[0, 0]
    I1 = oracle.render_fwd(q, H, W, k)[0, 0]
    np.testing.assert_array_equal(I1[3:, 5:], I0[:-3, :-5])


# --------------------------------------------------------------------------
# 6. Gradient closed forms for g == 1 on an untruncated Gaussian:
#    M = 2 pi a e^{s1+s2};  dM/da = 2 pi e^{s1+s2};  dM/ds_j = M;  dM/dmu = dM/dtheta = 0.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("s1,s2,th", [(0.0, 0.3, 0.4), (0.6, 0.1, 2.0), (0.3, 0.3, 1.0)])
def test_gradient_closed_forms(s1, s2, th):
    a = 1.9
    k = 2 * math.ceil(10.0 * math.exp(max(s1, s2))) + 1
    p = gauss(48.3, 47.6, s1, s2, th, [a])
    g = np.ones((1, 1, 96, 96), dtype=np.float32)
    d = oracle.render_bwd(p, g, 96, 96, k)[0, 0]
    s1f, s2f = float(p[0, 0, 2]), float(p[0, 0, 3])
    M = 2 * math.pi * float(p[0, 0, 5]) * math.exp(s1f + s2f)
    assert d[5] == pytest.approx(2 * math.pi * math.exp(s1f + s2f), rel=1e-7)
    assert d[2] == pytest.approx(M, rel=1e-7)
    assert d[3] == pytest.approx(M, rel=1e-7)
    assert abs(d[0]) <= 1e-7 * abs(M) and abs(d[1]) <= 1e-7 * abs(M)
    assert abs(d[4]) <= 1e-7 * abs(M)


# --------------------------------------------------------------------------
# 7. Adjoint identity: the image is linear in a, so <g, I> = sum_{i,c} a_ic dL/da_ic.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["tiny", "mono64"])
def test_adjoint_identity(name):
    w = WORKLOADS[name].scaled(B=min(WORKLOADS[name].B, 2))
    p, g = make_inputs(w)
    I = oracle.render_fwd(p, w.H, w.W, w.k)
    d = oracle.render_bwd(p, g, w.H, w.W, w.k)
    lhs = float(np.sum(g.astype(np.float64) * I))
    rhs = float(np.sum(p[..., 5:].astype(np.float64) * d[..., 5:]))
    assert lhs == pytest.approx(rhs, rel=1e-12)


# --------------------------------------------------------------------------
# 8. Central finite differences of L = <g, I(params)> for every parameter.
# --------------------------------------------------------------------------
def test_finite_differences_every_parameter():
    rng = np.random.default_rng(9)
    B, N, C, H, W, k = 2, 6, 2, 16, 18, 7
    p = np.empty((B, N, 5 + C))
    # integer + fractional part kept away from .5 so the window cannot move
    frac = rng.choice([0.15, 0.3, 0.7, 0.85], size=(B, N, 2))
    p[..., 0] = rng.integers(-2, W + 2, (B, N)) + frac[..., 0]
    p[..., 1] = rng.integers(-2, H + 2, (B, N)) + frac[..., 1]
    p[..., 2] = rng.normal(0.3, 0.4, (B, N))
    p[..., 3] = rng.normal(0.3, 0.4, (B, N))
    p[..., 4] = rng.uniform(0, np.pi, (B, N))
    p[..., 5:] = rng.normal(0, 1, (B, N, C))
    g = rng.normal(0, 1, (B, C, H, W))

    def L(pp):
        return float(np.sum(g * oracle.render_fwd(pp, H, W, k)))

    an = oracle.render_bwd(p, g, H, W, k)
    fd = np.zeros_like(an)
    for idx in np.ndindex(p.shape):
        h = 1e-5 * max(1.0, abs(p[idx]))
        pp, pm = p.copy(), p.copy()
        pp[idx] += h
        pm[idx] -= h
        fd[idx] = (L(pp) - L(pm)) / (2 * h)
    for j in range(5 + C):
        scale = np.abs(an[..., j]).max()
        assert scale > 0
        assert np.abs(fd[..., j] - an[..., j]).max() <= 1e-6 * scale, j


# --------------------------------------------------------------------------
# 9. Binning against brute-force window indicators: render each Gaussian alone
#    with a = 1 and a huge scale (w ~ 1 on its window), read off the 16x16
#    tiles with a nonzero pixel, compare with the rectangle-test lists.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("H,W,k,seed", [(32, 32, 7, 0), (40, 56, 17, 1), (23, 37, 21, 2), (16, 16, 1, 3)])
def test_binning_matches_window_indicators(H, W, k, seed):
    rng = np.random.default_rng(seed)
    N = 40
    p = np.zeros((1, N, 6), dtype=np.float32)
    p[0, :, 0] = rng.uniform(-k, W + k, N)
    p[0, :, 1] = rng.uniform(-k, H + k, N)
    p[0, :5, 0] = [0.5, 15.5, 16.49999, -0.5, W - 0.5]
    p[0, :, 2:4] = 8.0
    p[0, :, 5] = 1.0
    offs, ids = oracle.bin_tiles(p, H, W, k)
    TX, TY = (W + 15) // 16, (H + 15) // 16
    single = p.reshape(N, 1, 6)               # one Gaussian per frame
    ind = oracle.render_fwd(single, H, W, k)[:, 0] > 0
    want = [[] for _ in range(TX * TY)]
    for i in range(N):
        for ty in range(TY):
            for tx in range(TX):
                if ind[i, 16 * ty:16 * ty + 16, 16 * tx:16 * tx + 16].any():
                    want[ty * TX + tx].append(i)
    got = [ids[offs[t]:offs[t + 1]].tolist() for t in range(TX * TY)]
    assert got == want
    assert offs[-1] == len(ids) == sum(len(x) for x in want)


def test_grid_layout_puts_one_gaussian_per_cell():
    """Knob workloads: the grid-initialised layout is seeded, inside the frame,
    and holds exactly one mean per grid cell (jitter under half a cell)."""
    from differentiable_gaussian_splatting_pdr_b200.inputs import knob_workloads, make_inputs
    w = knob_workloads()["mono64-grid"]
    p1, _ = make_inputs(w)
    p2, _ = make_inputs(w)
    assert np.array_equal(p1, p2)
    mx, my = p1[..., 0].astype(np.float64), p1[..., 1].astype(np.float64)
    assert mx.min() >= 0 and mx.max() < w.W and my.min() >= 0 and my.max() < w.H
    gx = int(np.ceil(np.sqrt(w.N * w.W / w.H)))
    gy = int(np.ceil(w.N / gx))
    cell = np.floor(my / (w.H / gy)) * gx + np.floor(mx / (w.W / gx))
    for b in range(w.B):
        assert np.array_equal(np.sort(cell[b]), np.arange(w.N))


@pytest.mark.parametrize("H,W,k,seed", [(40, 56, 17, 1), (23, 37, 21, 2), (64, 64, 9, 3), (7, 9, 3, 4)])
def test_binning_matches_a_python_rect_test(H, W, k, seed):
    """The oracle's tile lists against a rect test written here from the
    definition alone (window = k x k pixels centred on round(mu) with ties up,
    clipped to the grid; a Gaussian enters every 16 x 16 tile the clipped
    window touches, ids ascending), sharing no code with the oracle."""
    import math
    rng = np.random.default_rng(seed)
    N = 60
    p = np.zeros((1, N, 6), dtype=np.float32)
    p[0, :, 0] = rng.uniform(-k, W + k, N)
    p[0, :, 1] = rng.uniform(-k, H + k, N)
    p[0, :6, 0] = [0.5, 15.5, np.nextafter(np.float32(16.5), np.float32(0)), -0.5, W - 0.5, np.nan]
    p[0, :, 2:4] = 0.5
    p[0, :, 5] = 1.0
    offs, ids = oracle.bin_tiles(p, H, W, k)
    r = (k - 1) // 2
    TX, TY = (W + 15) // 16, (H + 15) // 16
    want = [[] for _ in range(TX * TY)]
    for i in range(N):
        mx, my = float(p[0, i, 0]), float(p[0, i, 1])
        if not (math.isfinite(mx) and math.isfinite(my)):
            continue
        cx, cy = math.floor(mx + 0.5), math.floor(my + 0.5)  # exact: fp32 + 0.5 in fp64
        x0, x1 = max(cx - r, 0), min(cx + r, W - 1)
        y0, y1 = max(cy - r, 0), min(cy + r, H - 1)
        if x0 > x1 or y0 > y1:
            continue
        for ty in range(y0 // 16, y1 // 16 + 1):
            for tx in range(x0 // 16, x1 // 16 + 1):
                want[ty * TX + tx].append(i)
    got = [ids[offs[t]:offs[t + 1]].tolist() for t in range(TX * TY)]
    assert got == want
