"""Write tests/golden/tiny_oracle.txt and tests/golden/loss_oracle.txt from
the fp64 oracle alone.

The pages print no worked numeric example for the renderer, so this fixture is
a regression lock on the oracle itself: the "tiny" workload (1 frame, C=1,
32x32, N=64, k=7, seed 0) rendered and differentiated by oracle/ and nothing
else.  Re-run only when the oracle's arithmetic changes for a reason that a
passage of the pages (or a reading of one) justifies.

    python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from oracle import loss as oracle_loss  # noqa: E402
from differentiable_gaussian_splatting_pdr_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


def loss_pair():
    """The loss fixture's image / target pair: seeded draws, no arithmetic of
    the method (image ~ U[0, 1), target = clip(image + N(0, 0.1)), fp32)."""
    rng = np.random.default_rng(11)
    x = rng.uniform(0, 1, (1, 2, 12, 17)).astype(np.float32)
    y = np.clip(x + rng.normal(0, 0.1, x.shape), 0, 1).astype(np.float32)
    return x, y


def write_loss():
    x, y = loss_pair()
    loss, grad, (l1, ssim) = oracle_loss.l1_ssim_loss(x, y, 0.2)
    path = os.path.join(HERE, "loss_oracle.txt")
    with open(path, "w") as f:
        f.write("# L1 + SSIM loss oracle (lam 0.2, range 1) on a seeded 1x2x12x17 pair\n")
        f.write("# written by tests/golden/make_golden.py, which calls only oracle/\n")
        f.write("loss %.17g\n" % loss)
        f.write("l1 %.17g\n" % l1)
        f.write("ssim %.17g\n" % ssim)
        f.write("grad " + " ".join("%.17g" % v for v in grad.ravel()) + "\n")
    print(path)


def main():
    w = WORKLOADS["tiny"]
    p, g = make_inputs(w)
    img = oracle.render_fwd(p, w.H, w.W, w.k)
    grad = oracle.render_bwd(p, g, w.H, w.W, w.k)
    offs, ids = oracle.bin_tiles(p, w.H, w.W, w.k)
    path = os.path.join(HERE, "tiny_oracle.txt")
    with open(path, "w") as f:
        f.write("# oracle outputs for workload 'tiny' (1x1x32x32, N=64, k=7, seed 0)\n")
        f.write("# written by tests/golden/make_golden.py, which calls only oracle/\n")
        f.write("tile_offsets " + " ".join(str(int(v)) for v in offs) + "\n")
        f.write("tile_ids " + " ".join(str(int(v)) for v in ids) + "\n")
        f.write("image " + " ".join("%.17g" % v for v in img.ravel()) + "\n")
        f.write("grad_params " + " ".join("%.17g" % v for v in grad.ravel()) + "\n")
    print(path)


if __name__ == "__main__":
    main()
    write_loss()
