"""Writes tests/golden/tiny_layer_samples.json from the oracle alone.

Run from the repository root: ``python tests/golden/make_golden.py``. The
fixture records the fp64 oracle's output of the tiny workload (batch 1, 32x32
map, window 16, C=48, 3 heads, R=16, L=10, hidden 64, seed 0) at fixed
positions, so a later edit of the oracle that changes its arithmetic shows up
as a failing regression test.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from windowed_attention_b200.workloads import make_inputs  # noqa: E402

POSITIONS = [(0, 0, 0, 0), (0, 0, 31, 47), (0, 15, 16, 5), (0, 16, 15, 20), (0, 31, 0, 33),
             (0, 31, 31, 16), (0, 7, 23, 40), (0, 24, 9, 1)]


def main():
    inp = make_inputs("tiny")
    s = inp["shape"]
    Y, aux = oracle.rib_layer_forward(inp["X"], inp, s.heads, s.R, s.L, s.window)
    out = {
        "_source": "written by tests/golden/make_golden.py from oracle.rib_layer_forward on the tiny workload",
        "workload": "tiny",
        "positions": POSITIONS,
        "Y": [float(Y[p]) for p in POSITIONS],
        "Y_sum": float(Y.sum()),
        "Y_abs_sum": float(np.abs(Y).sum()),
        "Qp_head0_token0": [float(v) for v in aux["Qp"][0, 0]],
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_layer_samples.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
