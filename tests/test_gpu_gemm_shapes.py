"""GPU parity of the token GEMM on shapes the workloads do not reach.

The projection (rib_qkv_project) maps padded-image tokens to rows of X and
bulk-copies runs of rows that are contiguous in X. These cases make the runs
break at every image row (W < Wp), start on rows whose byte offset is only
8-byte aligned (odd W with C = 180), take an X that is 8- but not 16-byte
aligned (no bulk copies at all), and end the gate on a ragged last tile whose
byte count is not a multiple of 16. Reference: the fp64 oracle; tolerance as
in the other parity tests (max abs 2e-2, mean abs 2e-3).
"""
import math

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN = 2e-2, 2e-3


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _check(got, ref, what):
    d = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert d.max() <= TOL_MAX and d.mean() <= TOL_MEAN, f"{what}: max {d.max():.3e} mean {d.mean():.3e}"


def _bf16_np(t):
    return t.float().numpy().astype(np.float64)


@pytest.mark.parametrize("B,H,W,C,heads,M,offset", [
    (2, 37, 71, 180, 6, 16, 0),    # odd W: runs start on 8-byte aligned rows, Wp > W
    (1, 40, 72, 48, 3, 32, 0),     # 96-byte rows (always 16-byte aligned), Wp > W
    (1, 33, 50, 180, 6, 32, 4),    # X offset by 8 bytes: every row read without bulk copies
])
def test_qkv_projection_ragged_shapes(cuda_lib, B, H, W, C, heads, M, offset):
    rib = cuda_lib
    g = torch.Generator().manual_seed(11)
    X = torch.randn(B, H, W, C, generator=g).to(torch.bfloat16)
    Wq, Wk, Wv = (torch.randn(C, C, generator=g).mul(1 / math.sqrt(C)).to(torch.bfloat16) for _ in range(3))
    dh = C // heads
    DP = rib.rib_head_pad(C, heads)
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    Tp = B * Hp * Wp
    dev = "cuda"
    buf = torch.zeros(X.numel() + 8, dtype=torch.bfloat16, device=dev)
    Xd = buf[offset:offset + X.numel()]
    Xd.copy_(X.reshape(-1).to(dev))
    Qc = torch.full((Tp * heads * DP,), float("nan"), dtype=torch.bfloat16, device=dev)
    Kc = torch.full((Tp * heads * DP,), float("nan"), dtype=torch.bfloat16, device=dev)
    V = torch.full((Tp * heads * 32,), float("nan"), dtype=rib.v_dtype(), device=dev)
    scale = 1 / math.sqrt(dh)
    rib.rib_qkv_project(Xd, B, H, W, C, heads, M, Wq.to(dev), Wk.to(dev), Wv.to(dev), scale, Qc, Kc, V)
    torch.cuda.synchronize()
    rib.rib_device_error()
    Xp = oracle.pad_to_windows(_bf16_np(X), M).reshape(Tp, C)
    qc, kc, v = oracle.qkv_project(Xp, _bf16_np(Wq), _bf16_np(Wk), _bf16_np(Wv))
    for name, got, ref, s, width in (("Qc", Qc, qc, scale, DP), ("Kc", Kc, kc, 1.0, DP), ("V", V, v, 1.0, 32)):
        gg = _np(got).reshape(Tp, heads, width)
        _check(gg[:, :, :dh], (ref * s).reshape(Tp, heads, dh), name)
        if name == "Qc":
            assert np.all(gg[:, :, dh:] == 0)
        elif dh < width:
            # V's ones columns (the softmax denominator), and Kc's when the head
            # is padded (the attention's reference columns)
            assert np.all(gg[:, :, dh:] == 1.0)
    pad = np.ones((B, Hp, Wp), bool)
    pad[:, :H, :W] = False
    assert np.all(_np(Qc).reshape(B, Hp, Wp, heads, DP)[pad] == 0)


@pytest.mark.parametrize("B,H,W,C", [
    (1, 37, 71, 180),   # W*C % 8 != 0: the two-pass path; last GEMM tile of 67 rows, 24120 bytes
    (2, 20, 30, 48),    # fused: ragged 4x16 tiles at the bottom and right
    (1, 37, 72, 180),   # fused: two M=128 products (channels 0-127 and 52-179), two TMA boxes per row
    (1, 13, 34, 132),   # fused: second product over channels 4-131
    (1, 8, 20, 256),    # fused: widest supported map (three TMA boxes per row, K = 256)
])
def test_cla_gate_ragged_shapes(cuda_lib, B, H, W, C):
    rib = cuda_lib
    g = torch.Generator().manual_seed(12)
    X = torch.randn(B, H, W, C, generator=g).to(torch.bfloat16)
    Wdw = torch.randn(C, 3, 3, generator=g).mul(0.3)
    bdw = torch.randn(C, generator=g).mul(0.1)
    Wpw = torch.randn(C, C, generator=g).mul(1 / math.sqrt(C)).to(torch.bfloat16)
    bpw = torch.randn(C, generator=g).mul(0.1)
    dev = "cuda"
    out = torch.full((B, H, W, C), float("nan"), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(rib.cla_gate_workspace_size(B, H, W, C) // 2 + 8, dtype=torch.bfloat16, device=dev)
    rib.cla_gate(X.to(dev), B, H, W, C, Wdw.to(dev), bdw.to(dev), Wpw.to(dev), bpw.to(dev), out, ws)
    torch.cuda.synchronize()
    rib.rib_device_error()
    ref = oracle.cla_gate(_bf16_np(X), Wdw.numpy().astype(np.float64), bdw.numpy().astype(np.float64),
                          _bf16_np(Wpw), bpw.numpy().astype(np.float64))
    _check(_np(out), ref, "sigmoid gate")
    dw = oracle.dwconv3x3(_bf16_np(X), Wdw.numpy().astype(np.float64), bdw.numpy().astype(np.float64))
    _check(_np(ws[:B * H * W * C]).reshape(dw.shape), dw, "depthwise output left in the workspace")
    if (W * C) % 8 == 0:
        # the fused kernel needs no workspace; the gate is the same to the bit
        out2 = torch.full_like(out, float("nan"))
        rib.cla_gate(X.to(dev), B, H, W, C, Wdw.to(dev), bdw.to(dev), Wpw.to(dev), bpw.to(dev), out2, None)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    else:
        with pytest.raises(rib.RibError):
            rib.cla_gate(X.to(dev), B, H, W, C, Wdw.to(dev), bdw.to(dev), Wpw.to(dev), bpw.to(dev), out, None)
