"""The oracle still reproduces its committed regression fixture bit for bit."""
import os

import numpy as np

import oracle
from differentiable_gaussian_splatting_pdr_b200.inputs import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.txt")


def _load():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


def test_oracle_matches_golden_fixture():
    gold = _load()
    w = WORKLOADS["tiny"]
    p, g = make_inputs(w)
    img = oracle.render_fwd(p, w.H, w.W, w.k)
    grad = oracle.render_bwd(p, g, w.H, w.W, w.k)
    offs, ids = oracle.bin_tiles(p, w.H, w.W, w.k)
    np.testing.assert_array_equal(offs, np.array(gold["tile_offsets"], dtype=np.int64))
    np.testing.assert_array_equal(ids, np.array(gold["tile_ids"], dtype=np.int32))
    np.testing.assert_array_equal(img.ravel(), np.array(gold["image"], dtype=np.float64))
    np.testing.assert_array_equal(grad.ravel(), np.array(gold["grad_params"], dtype=np.float64))


LOSS_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "loss_oracle.txt")


def test_loss_oracle_matches_golden_fixture():
    """The L1 + SSIM oracle on the fixture's seeded pair reproduces the stored
    loss, its two terms and dL/dI (a regression lock on oracle/loss.py)."""
    import sys
    sys.path.insert(0, os.path.dirname(LOSS_GOLDEN))
    from make_golden import loss_pair
    from oracle import loss as oracle_loss
    gold = {}
    with open(LOSS_GOLDEN) as f:
        for line in f:
            if not line.startswith("#"):
                key, *vals = line.split()
                gold[key] = np.array(vals, dtype=np.float64)
    x, y = loss_pair()
    loss, grad, (l1, ssim) = oracle_loss.l1_ssim_loss(x, y, 0.2)
    np.testing.assert_allclose([loss, l1, ssim], [gold["loss"][0], gold["l1"][0], gold["ssim"][0]],
                               rtol=1e-14, atol=0)
    np.testing.assert_allclose(grad.ravel(), gold["grad"], rtol=1e-12, atol=1e-18)
