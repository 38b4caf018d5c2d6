"""Writes tests/golden/tiny_f32_digest.json from the float64 oracle.

Run from the repository root:  python tests/golden/make_golden.py
It calls only the oracle (and the seeded input generator for its inputs);
nothing here comes from the CUDA library.  The digest is a regression pin:
it changes only when the oracle's arithmetic or the input recipe changes.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import oracle  # noqa: E402
from lm_causal_depthwise_b200 import workloads as W  # noqa: E402

IDX = [(0, 0, 0), (0, 0, 255), (0, 1, 7), (0, 127, 100), (0, 128, 100), (0, 129, 3),
       (0, 200, 31), (0, 255, 0), (0, 255, 255)]


def digest():
    inp = W.generate(W.TINY_F32)
    out = oracle.prefill(**inp)
    y, h = out["y"], out["h_state"]
    return {
        "_what": "float64 oracle outputs on the tiny fp32 workload (B=1, T=256, D=256, seed 0, resets at t=0 and t=128)",
        "_made_by": "tests/golden/make_golden.py",
        "y_samples": [[list(i), float(y[i])] for i in IDX],
        "y_sum": float(y.sum()),
        "y_sumsq": float((y * y).sum()),
        "h_state_sum": float(h.sum()),
        "h_state_sumsq": float((h * h).sum()),
        "conv_state_sum": float(out["conv_state"].sum()),
    }


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_f32_digest.json")
    with open(path, "w") as f:
        json.dump(digest(), f, indent=1)
        f.write("\n")
    print("wrote", path)
