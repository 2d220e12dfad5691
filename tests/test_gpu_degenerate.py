"""GPU parity on the method's degenerate cases, through the C-ABI against the
fp64 oracle (tolerances as in the other parity tests: max abs error <= 2e-2,
mean abs error <= 2e-3):

* a map smaller than one window: one window, most of it zero padding;
* zero position-MLP output weights (Qp = Kp = 0): the score is the content
  term alone, i.e. scaled dot-product attention of Qc, Kc, V (RIB write-up,
  section 2.2: the rank term is added to the content term);
* an all-zero map: Qc = Kc = V = 0, so O = softmax(S) V = 0 whatever the
  positional scores, and Y = O * sigmoid(G) is exactly zero.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from windowed_attention_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN = 2e-2, 2e-3


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _check(got, ref, what):
    d = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert d.max() <= TOL_MAX and d.mean() <= TOL_MEAN, f"{what}: max {d.max():.3e} mean {d.mean():.3e}"


def _run(cuda_lib, inp):
    from windowed_attention_b200.layer import RibLayer
    s = inp["shape"]
    lay = RibLayer(s, inp, "cuda")
    lay.Y.fill_(float("nan"))                  # every output element must be written
    dt = torch.float32 if s.dtype == "f32" else torch.bfloat16
    Y = lay.forward(inp["X"].to("cuda", dt).contiguous())
    torch.cuda.synchronize()
    cuda_lib.rib_device_error()
    return lay, Y


def test_map_smaller_than_one_window(cuda_lib):
    # 20 x 24 map, window 32: one window padded to 32 x 32 (496 of 1024 tokens real)
    layer = replace(WORKLOADS["tiny"].layer, H=20, W=24, window=32, dtype="bf16")
    inp = make_inputs("tiny", layer=layer)
    s = inp["shape"]
    _, Y = _run(cuda_lib, inp)
    ref, _ = oracle.rib_layer_forward(inp["X"], inp, s.heads, s.R, s.L, s.window)
    _check(_np(Y), ref, "20x24 map, window 32")


def test_zero_position_weights(cuda_lib):
    inp = make_inputs("tiny")
    inp["Wpq"] = torch.zeros_like(inp["Wpq"])
    inp["Wpk"] = torch.zeros_like(inp["Wpk"])
    s = inp["shape"]
    lay, Y = _run(cuda_lib, inp)
    qp, kp = lay.pos_cache(s.window)
    assert torch.count_nonzero(qp).item() == 0 and torch.count_nonzero(kp).item() == 0
    ref, _ = oracle.rib_layer_forward(inp["X"], inp, s.heads, s.R, s.L, s.window)
    _check(_np(Y), ref, "Qp = Kp = 0")


def test_zero_map_gives_zero_output(cuda_lib):
    layer = replace(WORKLOADS["tiny"].layer, H=40, W=36, dtype="bf16")   # padded bottom and right
    inp = make_inputs("tiny", layer=layer)
    inp["X"] = torch.zeros_like(inp["X"])
    _, Y = _run(cuda_lib, inp)
    assert torch.count_nonzero(Y).item() == 0
