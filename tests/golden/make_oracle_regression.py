"""Write oracle_regression_tiny.txt from the FP64 oracle (calls only oracle/ and
the seeded input generator). Run from the repository root:
    python tests/golden/make_oracle_regression.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402
import oracle  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_regression_tiny.txt")


def tiny_case():
    lw = mi.make_layer(seed=7, layer=0, d=64, f=32, E=8)
    x = mi.make_tokens(7, 3, d=64)
    return lw, x


def main():
    lw, x = tiny_case()
    out, ids, w, fl = oracle.moe_layer(x, lw.router_w, lw.router_scale, lw.gate_up, lw.down,
                                       lw.expert_scale, k=3)
    with open(OUT, "w") as fh:
        fh.write("# FP64 oracle on moe_inputs.make_layer(seed=7, d=64, f=32, E=8), "
                 "make_tokens(7, 3, d=64), k=3\n")
        fh.write("ids " + " ".join(str(int(v)) for v in ids.ravel()) + "\n")
        fh.write("w " + " ".join(repr(float(v)) for v in w.ravel()) + "\n")
        fh.write("out " + " ".join(repr(float(v)) for v in out.ravel()) + "\n")


if __name__ == "__main__":
    main()
