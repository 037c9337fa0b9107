"""Writes tiny_forward.txt: the oracle's outputs on the tiny block (d=256,
I=128, E=8, top-2, B=1, k=24, c=48, r=8, seed 0).  It calls only the oracle
and the seeded input generator; the file pins the oracle against unintended
changes of its arithmetic."""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from calibration_free_channel_b200 import synth  # noqa: E402
from oracle import oracle as O  # noqa: E402


def compute():
    W = synth.layer_weights(synth.TINY, seed=0)
    sk = O.build_sketch(W["w_gate"], W["w_up"], synth.rot_seed(0))
    lr = O.build_lowrank(W["w_down"], 8)
    x = synth.tokens(256, 1, seed=0)
    y, _, dbg = O.forward(x, W, sk, lr, k=24, c=48, r=8, top_e=2, debug=True)
    return y, dbg


def main():
    y, dbg = compute()
    with open(os.path.join(HERE, "tiny_forward.txt"), "w") as f:
        f.write("# oracle outputs, tiny block (d=256 I=128 E=8 top-2 B=1 k=24 c=48 r=8 seed 0)\n")
        f.write("# written by tests/golden/make_golden.py (calls only oracle/ and synth)\n")
        f.write("ids " + " ".join(map(str, dbg["ids"].ravel())) + "\n")
        for s in range(2):
            f.write(f"cand{s} " + " ".join(map(str, dbg["cand"][0, s])) + "\n")
            f.write(f"kept{s} " + " ".join(map(str, dbg["kept"][0, s])) + "\n")
        f.write("y " + " ".join(f"{v:04x}" for v in y.ravel()) + "\n")


if __name__ == "__main__":
    main()
