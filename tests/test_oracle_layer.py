"""Pins of the oracle's whole-layer forward, stack and backward.

Cited passages: RIB/SST write-up section 2.2 (RIB score), section 2.3 (CLA
gate O = softmax(S)V * sigma(G)), section 3.1 (block = LayerNorm -> RIB
attention -> CLA), section 3.2 (window cycle).

The map-level forward is pinned against an independent route built from
library routines only: torch views for the window rearrangement, fp64
``scaled_dot_product_attention`` with the positional term as an additive
mask (the write-up's RPB form), and ``conv2d`` for the gate. The backward is
pinned by central finite differences in fp64.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from windowed_attention_b200.workloads import LayerShape, WORKLOADS, make_inputs


def _params(rng, C, heads, R, L, hidden):
    e = 2 + 4 * L
    return {
        "Wq": rng.normal(size=(C, C)) / math.sqrt(C), "Wk": rng.normal(size=(C, C)) / math.sqrt(C),
        "Wv": rng.normal(size=(C, C)) / math.sqrt(C),
        "Wh": rng.normal(size=(e, hidden)) / math.sqrt(e), "bh": rng.normal(size=hidden) / math.sqrt(e),
        "Wpq": rng.normal(size=(hidden, heads * R)) / math.sqrt(hidden),
        "Wpk": rng.normal(size=(hidden, heads * R)) / math.sqrt(hidden),
        "Wdw": rng.normal(size=(C, 3, 3)) / 3.0, "bdw": rng.normal(size=C) / 3.0,
        "Wpw": rng.normal(size=(C, C)) / math.sqrt(C), "bpw": rng.normal(size=C) / math.sqrt(C),
    }


def _torch_layer(X, p, heads, R, L, M):
    """Independent route: torch views + SDPA with additive mask + conv2d."""
    X = torch.tensor(X)
    B, H, W, C = X.shape
    dh = C // heads
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    Xp = torch.zeros(B, Hp, Wp, C, dtype=torch.float64)
    Xp[:, :H, :W] = X
    # coordinate features, written with torch ops
    g = torch.linspace(-1, 1, M, dtype=torch.float64)
    coords = torch.stack(torch.meshgrid(g, g, indexing="ij"), -1).reshape(-1, 2)
    feats = [coords] + [f(coords * 2.0 ** i) for i in range(L) for f in (torch.sin, torch.cos)]
    r = torch.cat(feats, -1)
    h = torch.relu(r @ torch.tensor(p["Wh"]) + torch.tensor(p["bh"]))
    qp = (h @ torch.tensor(p["Wpq"])).view(-1, heads, R).transpose(0, 1)
    kp = (h @ torch.tensor(p["Wpk"])).view(-1, heads, R).transpose(0, 1)
    bias = qp @ kp.transpose(1, 2) / math.sqrt(R)                      # [heads, N, N]
    win = Xp.view(B, Hp // M, M, Wp // M, M, C).permute(0, 1, 3, 2, 4, 5).reshape(-1, M * M, C)
    def heads_of(t):
        return t.view(t.shape[0], M * M, heads, dh).transpose(1, 2)   # [nW, heads, N, dh]
    q = heads_of(win @ torch.tensor(p["Wq"]))
    k = heads_of(win @ torch.tensor(p["Wk"]))
    v = heads_of(win @ torch.tensor(p["Wv"]))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=bias[None])
    o = o.transpose(1, 2).reshape(-1, M * M, C)
    o = o.view(B, Hp // M, Wp // M, M, M, C).permute(0, 1, 3, 2, 4, 5).reshape(B, Hp, Wp, C)[:, :H, :W]
    x2 = X.permute(0, 3, 1, 2)
    dw = torch.nn.functional.conv2d(x2, torch.tensor(p["Wdw"])[:, None], torch.tensor(p["bdw"]), padding=1, groups=C)
    G = torch.nn.functional.conv2d(dw, torch.tensor(p["Wpw"]).T[:, :, None, None], torch.tensor(p["bpw"]))
    return (o * torch.sigmoid(G).permute(0, 2, 3, 1)).numpy()


@pytest.mark.parametrize("B,H,W,C,heads,R,L,hidden,M", [
    (1, 16, 16, 12, 3, 4, 3, 8, 8),
    (2, 13, 21, 8, 2, 4, 2, 6, 8),     # padded bottom and right
    (1, 12, 12, 6, 1, 2, 2, 5, 12),
])
def test_layer_matches_independent_torch_route(B, H, W, C, heads, R, L, hidden, M):
    rng = np.random.default_rng(B * 100 + H)
    X = rng.normal(size=(B, H, W, C))
    p = _params(rng, C, heads, R, L, hidden)
    Y, aux = oracle.rib_layer_forward(X, p, heads, R, L, M)
    ref = _torch_layer(X, p, heads, R, L, M)
    assert Y.shape == (B, H, W, C)
    assert np.max(np.abs(Y - ref)) < 1e-12


def test_layer_windows_subset_matches_full():
    rng = np.random.default_rng(11)
    B, H, W, C, heads, R, L, hidden, M = 2, 13, 21, 8, 2, 4, 2, 6, 8
    X = rng.normal(size=(B, H, W, C))
    p = _params(rng, C, heads, R, L, hidden)
    Y, _ = oracle.rib_layer_forward(X, p, heads, R, L, M)
    ids = [0, 2, 4, 5]   # includes right and bottom padded windows of both images
    for b, y0, x0, blk in oracle.rib_layer_forward_windows(X, p, heads, R, L, M, ids):
        assert np.max(np.abs(Y[b, y0:y0 + blk.shape[0], x0:x0 + blk.shape[1]] - blk)) < 1e-13


def test_open_gate_leaves_attention_output():
    rng = np.random.default_rng(12)
    X = rng.normal(size=(1, 8, 8, 4))
    p = _params(rng, 4, 2, 2, 2, 4)
    p["Wpw"] = np.zeros((4, 4))
    p["bpw"] = np.full(4, 60.0)
    Y, aux = oracle.rib_layer_forward(X, p, 2, 2, 2, 4)
    assert np.allclose(Y, aux["O"], atol=1e-15)


def test_stack_with_zero_value_weights_is_identity():
    rng = np.random.default_rng(13)
    x = rng.normal(size=(1, 8, 8, 4))
    blocks = []
    for _ in range(3):
        p = _params(rng, 4, 2, 2, 2, 4)
        p["Wv"] = np.zeros((4, 4))
        blocks.append(p)
    assert np.array_equal(oracle.stack_forward(x, blocks, [2, 4, 8], 2, 2, 2), x)


def test_stack_single_block_is_residual_of_layer():
    rng = np.random.default_rng(14)
    x = rng.normal(size=(1, 8, 8, 4)) * 2 + 0.5
    p = _params(rng, 4, 2, 2, 2, 4)
    ln = torch.nn.functional.layer_norm(torch.tensor(x), (4,), eps=1e-5).numpy()
    ref = x + _torch_layer(ln, p, 2, 2, 2, 4)
    assert np.max(np.abs(oracle.stack_forward(x, [p], [4], 2, 2, 2) - ref)) < 1e-12


# ---------------------------------------------------------------- backward
def _fd_check(f, x, g, idx_list, h=1e-6, tol=2e-6):
    for idx in idx_list:
        old = x[idx]
        x[idx] = old + h
        fp = f()
        x[idx] = old - h
        fm = f()
        x[idx] = old
        num = (fp - fm) / (2 * h)
        assert abs(num - g[idx]) <= tol * max(1.0, abs(num)), (idx, num, g[idx])


@pytest.mark.parametrize("H,W,M", [(4, 4, 4), (3, 6, 4)])
def test_layer_backward_finite_differences(H, W, M):
    # one 4x4 window, 2 heads (and a padded 2-window case)
    rng = np.random.default_rng(20 + W)
    B, C, heads, R, L, hidden = 1, 4, 2, 2, 2, 3
    X = rng.normal(size=(B, H, W, C))
    p = _params(rng, C, heads, R, L, hidden)
    dY = rng.normal(size=(B, H, W, C))
    g, _ = oracle.rib_layer_backward(X, p, dY, heads, R, L, M)

    def loss():
        return float((oracle.rib_layer_forward(X, p, heads, R, L, M)[0] * dY).sum())

    _fd_check(loss, X, g["X"], [tuple(i) for i in np.ndindex(X.shape)])
    for name in ("Wq", "Wk", "Wv", "Wh", "bh", "Wpq", "Wpk", "Wdw", "bdw", "Wpw", "bpw"):
        arr = p[name]
        idxs = [tuple(i) for i in np.ndindex(arr.shape)]
        _fd_check(loss, arr, g[name], idxs)


def test_window_backward_split_matches_concat_gradient():
    # dQ of the concatenated form splits into [dQc/sqrt(D), dQp/sqrt(R)]:
    # check against torch autograd on the concatenated product.
    rng = np.random.default_rng(30)
    n, dh, R = 10, 3, 2
    qc, kc, v, qp, kp, do = (rng.normal(size=(n, dh)), rng.normal(size=(n, dh)), rng.normal(size=(n, 3)),
                             rng.normal(size=(n, R)), rng.normal(size=(n, R)), rng.normal(size=(n, 3)))
    ts = [torch.tensor(a, requires_grad=True) for a in (qc, kc, v, qp, kp)]
    Q = torch.cat([ts[0] / math.sqrt(dh), ts[3] / math.sqrt(R)], 1)
    K = torch.cat([ts[1], ts[4]], 1)
    O = torch.softmax(Q @ K.T, dim=1) @ ts[2]
    (O * torch.tensor(do)).sum().backward()
    got = oracle.attention_window_backward(qc, kc, v, qp, kp, do, dh, R)
    for a, t in zip(got, [ts[0], ts[1], ts[2], ts[3], ts[4]]):
        assert np.max(np.abs(a - t.grad.numpy())) < 1e-13


def test_workload_shapes_are_the_stated_ones():
    full = WORKLOADS["full"].layer
    assert (full.H, full.W, full.C, full.heads, full.dh, full.R, full.window) == (360, 640, 180, 6, 30, 16, 64)
    assert full.tokens == 230400 and full.n_windows == 60
    assert abs(full.attention_flops() / 1e9 - 918.0) < 1.0
    tr = WORKLOADS["train"].layer
    assert tr.n_windows == 16 and tr.window * tr.window == 9216
    assert abs(tr.attention_flops() / 1e9 - 1239.0) < 1.0
    assert abs(tr.attention_bwd_flops() / 1e9 - 3229.0) < 2.0
    assert WORKLOADS["stack"].windows == (16, 32, 64, 16, 32, 64)


def test_generator_is_seeded_and_bf16_exact():
    a = make_inputs("tiny")
    b = make_inputs("tiny")
    assert torch.equal(a["X"], b["X"]) and torch.equal(a["Wpw"], b["Wpw"])
    s = LayerShape(B=1, H=8, W=8, C=12, heads=2, R=4, L=2, hidden=4, window=4)
    c = make_inputs("full", layer=s)
    assert torch.equal(c["X"], c["X"].bfloat16().float())
    assert torch.equal(c["Wq"], c["Wq"].bfloat16().float())
