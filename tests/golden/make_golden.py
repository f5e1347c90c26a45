"""Write tests/golden/tiny_oracle.txt from the fp64 oracle alone.

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
from differentiable_gaussian_splatting_pdr_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


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
