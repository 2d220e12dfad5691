"""GPU parity of the backward (rib_attention_bwd_prep -> rib_window_attention_bwd
-> rib_pos_encode_bwd) against the fp64 oracle's analytic backward, which the
CPU tests pin by finite differences.

The GPU returns gradients with respect to the tensors as stored: Qc' = Qc /
sqrt(dh) and the cached Qp' = Qp / sqrt(R). The oracle's gradients are with
respect to the unscaled Qc, Qp, so dQc = dQc' / sqrt(dh) and dQp = dQp' /
sqrt(R); dKc, dKp and dV compare directly. Tolerance: max abs error <= 2e-2
and mean abs error <= 2e-3 on gradients normalised by the largest magnitude
of the reference (the gradients of a sum over many windows grow with the
window count, and the per-window ones shrink with the window size).
"""
import math

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
    scale = float(np.abs(ref).max())
    assert scale > 0, f"{what}: reference is all zero"
    d = np.abs(got - ref) / scale
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    print(f"{what}: scale {scale:.3g} rel max {d.max():.2e} rel mean {d.mean():.2e}")
    assert d.max() <= TOL_MAX and d.mean() <= TOL_MEAN, f"{what}: max {d.max():.3e} mean {d.mean():.3e} (scale {scale:.3g})"


def _run(wl_name):
    from windowed_attention_b200.layer import RibLayer
    inp = make_inputs(wl_name, with_grad=True)
    s = inp["shape"]
    lay = RibLayer(s, inp, "cuda")
    X = inp["X"].to("cuda", torch.bfloat16).contiguous()
    dY = inp["dY"].to("cuda", torch.bfloat16).contiguous()
    g = lay.backward(X, dY)
    import windowed_attention_b200 as rib
    rib.rib_device_error()
    return inp, s, lay, g


def _oracle_window(inp, s, w, hd, dO_w):
    """Oracle backward of window w, head hd (unscaled features)."""
    M = s.window
    dh = s.C // s.heads
    Xp = oracle.pad_to_windows(inp["X"], M)
    xw = oracle.window_partition(Xp, M)[w]
    sl = slice(hd * dh, (hd + 1) * dh)
    qc, kc, v = xw @ _np(inp["Wq"])[:, sl], xw @ _np(inp["Wk"])[:, sl], xw @ _np(inp["Wv"])[:, sl]
    qp, kp = oracle.pos_features(M, s.L, inp["Wh"], inp["bh"], inp["Wpq"], inp["Wpk"], s.heads, s.R)
    return oracle.attention_window_backward(qc, kc, v, qp[hd], kp[hd], dO_w[:, sl], dh, s.R)


def _gpu_window(g, s, w, hd, M):
    """GPU gradients of window w, head hd in window-token order."""
    Hp, Wp = s.Hp, s.Wp
    ny, nx = Hp // M, Wp // M
    b, rem = divmod(w, ny * nx)
    wy, wx = divmod(rem, nx)
    dh = s.C // s.heads

    def block(t):
        a = _np(t).reshape(s.B, Hp, Wp, s.heads, 32)
        return a[b, wy * M:(wy + 1) * M, wx * M:(wx + 1) * M, hd, :dh].reshape(M * M, dh)

    return block(g["dQc"]), block(g["dKc"]), block(g["dV"])


def _dO_windows(inp, s):
    gate = oracle.cla_gate(inp["X"], inp["Wdw"], inp["bdw"], inp["Wpw"], inp["bpw"])
    dO = _np(inp["dY"]) * gate
    Hp, Wp = s.Hp, s.Wp
    dOp = np.zeros((s.B, Hp, Wp, s.C))
    dOp[:, :s.H, :s.W] = dO
    return oracle.window_partition(dOp, s.window)


def test_backward_tiny_all_windows(cuda_lib):
    inp, s, lay, g = _run("tiny")
    M, dh, R = s.window, s.C // s.heads, s.R
    dOw = _dO_windows(inp, s)
    nwin = s.n_windows
    dqp_tot = np.zeros((s.heads, M * M, R))
    dkp_tot = np.zeros((s.heads, M * M, R))
    ws = _np(g["ws"])
    half = ws.size // 2
    for w in range(nwin):
        for hd in range(s.heads):
            gqc, gkc, gv, gqp, gkp = _oracle_window(inp, s, w, hd, dOw[w])
            dqc, dkc, dv = _gpu_window(g, s, w, hd, M)
            _rel_check(dqc / math.sqrt(dh), gqc, f"dQc w{w} h{hd}")
            _rel_check(dkc, gkc, f"dKc w{w} h{hd}")
            _rel_check(dv, gv, f"dV w{w} h{hd}")
            pq = ws[:half].reshape(nwin, s.heads, M * M, R)[w, hd]
            pk = ws[half:].reshape(nwin, s.heads, M * M, R)[w, hd]
            _rel_check(pq / math.sqrt(R), gqp, f"dQp partial w{w} h{hd}")
            _rel_check(pk, gkp, f"dKp partial w{w} h{hd}")
            dqp_tot[hd] += gqp
            dkp_tot[hd] += gkp
    _rel_check(_np(g["dQp"]).reshape(s.heads, M * M, R) / math.sqrt(R), dqp_tot, "dQp total")
    _rel_check(_np(g["dKp"]).reshape(s.heads, M * M, R), dkp_tot, "dKp total")
    ref = oracle.pos_features_backward(M, s.L, inp["Wh"], inp["bh"], inp["Wpq"], inp["Wpk"], s.heads, R, dqp_tot, dkp_tot)
    for name, key in (("Wh", "dWh"), ("bh", "dbh"), ("Wpq", "dWpq"), ("Wpk", "dWpk")):
        _rel_check(_np(g[key]), ref[name], f"MLP d{name}")


def test_backward_gate_gradient_tiny(cuda_lib):
    # dG = dY * O * sigma * (1 - sigma): the gradient into the CLA gate
    inp, s, lay, g = _run("tiny")
    Y, aux = oracle.rib_layer_forward(inp["X"], inp, s.heads, s.R, s.L, s.window)
    gate = aux["gate"]
    ref = _np(inp["dY"]) * aux["O"] * gate * (1 - gate)
    _rel_check(_np(g["dG"]), ref, "dG")


def test_backward_train_sampled_windows(cuda_lib):
    # 16 patches of 96x96, window 96 (N = 9216): eight (window, head) pairs,
    # eight different windows, every head at least once
    inp, s, lay, g = _run("train")
    M, dh, R = s.window, s.C // s.heads, s.R
    dOw = _dO_windows(inp, s)
    ws = _np(g["ws"])
    half = ws.size // 2
    nwin = s.n_windows
    for w, hd in ((0, 0), (2, 1), (5, 2), (7, 3), (9, 4), (11, 5), (13, 0), (15, 3)):
        gqc, gkc, gv, gqp, gkp = _oracle_window(inp, s, w, hd, dOw[w])
        dqc, dkc, dv = _gpu_window(g, s, w, hd, M)
        _rel_check(dqc / math.sqrt(dh), gqc, f"dQc w{w} h{hd}")
        _rel_check(dkc, gkc, f"dKc w{w} h{hd}")
        _rel_check(dv, gv, f"dV w{w} h{hd}")
        _rel_check(ws[:half].reshape(nwin, s.heads, M * M, R)[w, hd] / math.sqrt(R), gqp, f"dQp partial w{w}")
        _rel_check(ws[half:].reshape(nwin, s.heads, M * M, R)[w, hd], gkp, f"dKp partial w{w}")
    # the totals are the fixed-order sums of the partials
    tot_q = ws[:half].reshape(nwin, -1).sum(axis=0)
    assert np.allclose(_np(g["dQp"]).reshape(-1), tot_q, rtol=1e-5, atol=1e-4)
