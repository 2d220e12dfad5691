"""GPU parity of the rest of the backward: the content projections
(rib_qkv_project_bwd) and the CLA gate (cla_gate_bwd), alone and inside the
layer's backward chain, against the fp64 oracle (whose layer backward the CPU
tests pin by finite differences).

Tolerance as in the other backward tests: max abs error <= 2e-2 and mean abs
error <= 2e-3 on gradients normalised by the largest magnitude of the
reference (weight gradients are sums over every token and grow with the
token count).
"""
import math
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


def _rel_check(got, ref, what):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    scale = float(np.abs(ref).max())
    assert scale > 0, f"{what}: reference is all zero"
    d = np.abs(got - ref) / scale
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    print(f"{what}: scale {scale:.3g} rel max {d.max():.2e} rel mean {d.mean():.2e}")
    assert d.max() <= TOL_MAX and d.mean() <= TOL_MEAN, f"{what}: max {d.max():.3e} mean {d.mean():.3e}"


# a C = 180 layer with bottom and right padding (40x36 map, window 16 -> 48x48)
PADDED_180 = replace(WORKLOADS["tiny"].layer, H=40, W=36, C=180, heads=6, dtype="bf16")


@pytest.mark.parametrize("wl,layer", [("tiny", None), ("tiny", PADDED_180)], ids=["tiny", "padded_c180"])
def test_layer_backward_dx_and_weight_grads(cuda_lib, wl, layer):
    from windowed_attention_b200.layer import RibLayer
    inp = make_inputs(wl, layer=layer, with_grad=True)
    s = inp["shape"]
    lay = RibLayer(s, inp, "cuda")
    dt = torch.float32 if s.dtype == "f32" else torch.bfloat16
    X = inp["X"].to("cuda", dt).contiguous()
    dY = inp["dY"].to("cuda", torch.bfloat16).contiguous()
    g = lay.backward(X, dY)
    torch.cuda.synchronize()
    cuda_lib.rib_device_error()
    ref, _ = oracle.rib_layer_backward(inp["X"], inp, inp["dY"], s.heads, s.R, s.L, s.window)
    _rel_check(_np(g["dX"]), ref["X"], "dX")
    for name in ("Wq", "Wk", "Wv", "Wpw", "Wdw", "bdw", "bpw"):
        _rel_check(_np(g["d" + name]), ref[name], "d" + name)


# (B, H, W, C, heads, window): the training shape; ragged tensor-core tiles
# (H % 4, W % 32 != 0, padded windows); an odd head count; maps the tensor-core
# path does not take (W*C % 8 != 0; W < 32) and that run on the CUDA cores
PROJ_GATE_SHAPES = {
    "train": (16, 96, 96, 180, 6, 96),
    "ragged_tc": (1, 42, 100, 180, 6, 16),
    "odd_heads_tc": (2, 32, 40, 48, 3, 16),
    "cuda_cores_wc": (2, 20, 33, 180, 6, 16),
    "cuda_cores_narrow": (1, 9, 24, 48, 3, 8),
}


@pytest.mark.parametrize("name", list(PROJ_GATE_SHAPES))
def test_projection_and_gate_bwd(cuda_lib, name):
    """Both entry points alone on seeded gradients, against the oracle; a
    second call must give bit-identical results (fixed-order reductions)."""
    rib = cuda_lib
    B, H, W, C, heads, M = PROJ_GATE_SHAPES[name]
    dh = C // heads
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    T = B * H * W
    gen = torch.Generator().manual_seed(21)
    X = torch.randn(B, H, W, C, generator=gen).to(torch.bfloat16)
    Ws = [torch.randn(C, C, generator=gen).mul(1 / math.sqrt(C)).to(torch.bfloat16) for _ in range(3)]
    # gradients of the stored projections in the padded head layout; columns
    # >= dh and the padding pixels must be ignored
    gp = [torch.randn(B, Hp, Wp, heads, 32, generator=gen) for _ in range(3)]
    q_scale = 1 / math.sqrt(dh)
    dev = "cuda"
    Xd = X.to(dev)
    Wd = [w.to(dev) for w in Ws]
    gd = [x.to(dev) for x in gp]

    def proj():
        dX = torch.empty(B, H, W, C, dtype=torch.float32, device=dev)
        dW = [torch.empty(C, C, dtype=torch.float32, device=dev) for _ in range(3)]
        rib.rib_qkv_project_bwd(Xd, B, H, W, C, heads, M, *Wd, q_scale, *gd, dX, *dW)
        return [dX] + dW

    first, second = proj(), proj()
    torch.cuda.synchronize()
    rib.rib_device_error()
    for a, b in zip(first, second):
        assert torch.equal(a, b), "projection backward differs between two calls"
    dX, dWq, dWk, dWv = first
    gimg = [x[:, :H, :W, :, :dh].reshape(T, C).numpy().astype(np.float64) for x in gp]
    gimg[0] = gimg[0] * q_scale
    Xn = X.float().numpy().astype(np.float64)
    rdX, rWq, rWk, rWv = oracle.qkv_project_backward(Xn.reshape(T, C), *[w.float().numpy() for w in Ws], *gimg)
    _rel_check(_np(dX).reshape(T, C), rdX, "projection dX")
    for nm, got, ref in (("dWq", dWq, rWq), ("dWk", dWk, rWk), ("dWv", dWv, rWv)):
        _rel_check(_np(got), ref, nm)

    # CLA gate: D is the depthwise output the forward leaves in cla_gate's
    # workspace (here the oracle's, rounded to bf16)
    Wdw = torch.randn(C, 3, 3, generator=gen).mul(1 / 3)
    bdw = torch.randn(C, generator=gen).mul(1 / 3)
    Wpw = torch.randn(C, C, generator=gen).mul(1 / math.sqrt(C)).to(torch.bfloat16)
    dG = torch.randn(B, H, W, C, generator=gen).to(torch.bfloat16)
    D = torch.tensor(oracle.dwconv3x3(Xn, Wdw.numpy(), bdw.numpy()), dtype=torch.float32).to(torch.bfloat16)
    dX0 = torch.randn(B, H, W, C, generator=gen)          # the gate part is added to this
    ws = torch.empty(rib.cla_gate_bwd_workspace_size(B, H, W, C) // 4, dtype=torch.float32, device=dev)
    args = (Wdw.to(dev), Wpw.to(dev), D.to(dev), dG.to(dev))

    def gate():
        dXg = dX0.to(dev)
        outs = [torch.empty(C, 3, 3, device=dev), torch.empty(C, device=dev), torch.empty(C, C, device=dev),
                torch.empty(C, device=dev)]
        rib.cla_gate_bwd(Xd, B, H, W, C, *args, dXg, *outs, ws)
        return [dXg] + outs

    first, second = gate(), gate()
    torch.cuda.synchronize()
    rib.rib_device_error()
    for a, b in zip(first, second):
        assert torch.equal(a, b), "gate backward differs between two calls"
    dXg, *outs = first
    rX, rWdw, rbdw, rWpw, rbpw = oracle.cla_gate_backward(Xn, Wdw.numpy(), bdw.numpy(), Wpw.float().numpy(),
                                                          dG.float().numpy())
    _rel_check(_np(dXg) - dX0.numpy(), rX, "gate dX")
    for nm, got, ref in (("dWdw", outs[0], rWdw), ("dbdw", outs[1], rbdw), ("dWpw", outs[2], rWpw),
                         ("dbpw", outs[3], rbpw)):
        _rel_check(_np(got), ref, nm)
