"""Pins of the oracle's ConvFFN and full SST block (RIB/SST write-up, section
3.1 "模型架构设计": a block is LayerNorm -> RIB attention -> CLA -> ConvFFN
with FFN expansion 1.25).

GELU is pinned by closed forms and an identity; ConvFFN against an
independent torch fp64 route (linear, gelu, conv2d with one group per
channel); with its depthwise filters zero it is the plain two-layer FFN; the
SST block against the stack block plus a separately computed ConvFFN
residual.
"""
import math

import numpy as np
import torch

import oracle


def test_gelu_closed_forms():
    x = np.array([0.0, 1.0, -1.0, 2.0, -3.0, 0.5])
    g = oracle.gelu(x)
    assert g[0] == 0.0
    # GELU(1) = Phi(1) = 0.841344746068542948...
    assert abs(g[1] - 0.8413447460685429) < 1e-15
    # x Phi(x) - (-x) Phi(-x) = x (Phi(x) + Phi(-x) = 1)
    assert np.allclose(oracle.gelu(x) - oracle.gelu(-x), x, atol=1e-15)
    # large arguments: the identity and zero
    assert abs(oracle.gelu(np.array([10.0]))[0] - 10.0) < 1e-12
    assert abs(oracle.gelu(np.array([-10.0]))[0]) < 1e-12


def _ffn_params(rng, C, hid):
    return {"W1": rng.normal(size=(C, hid)) / math.sqrt(C), "b1": rng.normal(size=hid) / math.sqrt(C),
            "Wf": rng.normal(size=(hid, 3, 3)) / 3.0, "bf": rng.normal(size=hid) / 3.0,
            "W2": rng.normal(size=(hid, C)) / math.sqrt(hid), "b2": rng.normal(size=C) / math.sqrt(hid)}


def test_conv_ffn_matches_a_torch_route():
    rng = np.random.default_rng(5)
    B, H, W, C = 2, 7, 9, 12
    hid = 15                      # 1.25 C
    f = _ffn_params(rng, C, hid)
    x = rng.normal(size=(B, H, W, C))
    got = oracle.conv_ffn(x, **f)
    t = {k: torch.tensor(v) for k, v in f.items()}
    h = torch.nn.functional.gelu(torch.tensor(x) @ t["W1"] + t["b1"], approximate="none")
    hc = h.permute(0, 3, 1, 2)                      # [B, hid, H, W]
    d = torch.nn.functional.conv2d(hc, t["Wf"][:, None], t["bf"], padding=1, groups=hid)
    ref = (h + d.permute(0, 2, 3, 1)) @ t["W2"] + t["b2"]
    assert np.allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_conv_ffn_without_the_conv_is_the_plain_ffn():
    rng = np.random.default_rng(6)
    B, H, W, C, hid = 1, 5, 6, 8, 10
    f = _ffn_params(rng, C, hid)
    f["Wf"] = np.zeros_like(f["Wf"])
    f["bf"] = np.zeros_like(f["bf"])
    x = rng.normal(size=(B, H, W, C))
    t = {k: torch.tensor(v) for k, v in f.items()}
    ref = torch.nn.functional.linear(
        torch.nn.functional.gelu(torch.nn.functional.linear(torch.tensor(x), t["W1"].T, t["b1"]), approximate="none"),
        t["W2"].T, t["b2"])
    assert np.allclose(oracle.conv_ffn(x, **f), ref.numpy(), rtol=1e-12, atol=1e-12)
    # an identity-like depthwise filter (centre tap -1, bias 0) cancels h: out = b2
    f["Wf"][:, 1, 1] = -1.0
    assert np.allclose(oracle.conv_ffn(x, **f), np.broadcast_to(f["b2"], (B, H, W, C)), atol=1e-12)


def test_sst_block_is_the_stack_block_plus_the_ffn_residual():
    from windowed_attention_b200.workloads import make_inputs
    from dataclasses import replace
    from windowed_attention_b200.workloads import WORKLOADS
    layer = replace(WORKLOADS["tiny"].layer, H=16, W=20, dtype="bf16")
    inp = make_inputs("tiny", layer=layer)
    s = inp["shape"]
    rng = np.random.default_rng(7)
    f = _ffn_params(rng, s.C, 60)
    x = inp["X"].numpy().astype(np.float64)
    got = oracle.sst_block(x, inp, f, s.heads, s.R, s.L, s.window)
    x1 = oracle.stack_forward(x, [inp], [s.window], s.heads, s.R, s.L)
    ref = x1 + oracle.conv_ffn(oracle.layernorm(x1), **f)
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-13)
    two = oracle.sst_stack_forward(x, [inp, inp], [f, f], [s.window, s.window], s.heads, s.R, s.L)
    assert np.allclose(two, oracle.sst_block(got, inp, f, s.heads, s.R, s.L, s.window), rtol=1e-13, atol=1e-13)
