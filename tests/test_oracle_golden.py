"""Regression of the oracle against the fixture that tests/golden/make_golden.py
wrote from the oracle itself (tiny workload, seed 0)."""
import json
import os

import numpy as np

import oracle
from windowed_attention_b200.workloads import make_inputs


def test_tiny_layer_regression():
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_layer_samples.json")) as f:
        g = json.load(f)
    inp = make_inputs("tiny")
    s = inp["shape"]
    Y, aux = oracle.rib_layer_forward(inp["X"], inp, s.heads, s.R, s.L, s.window)
    for p, v in zip(g["positions"], g["Y"]):
        assert abs(Y[tuple(p)] - v) < 1e-12
    assert abs(Y.sum() - g["Y_sum"]) < 1e-9
    assert abs(np.abs(Y).sum() - g["Y_abs_sum"]) < 1e-9
    assert np.allclose(aux["Qp"][0, 0], g["Qp_head0_token0"], atol=1e-13)
