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
