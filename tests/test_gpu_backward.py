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


def _rel_check(got, ref, what, tol_max=TOL_MAX, tol_mean=TOL_MEAN):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    scale = float(np.abs(ref).max())
    assert scale > 0, f"{what}: reference is all zero"
    d = np.abs(got - ref) / scale
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    print(f"{what}: scale {scale:.3g} rel max {d.max():.2e} rel mean {d.mean():.2e}")
    assert d.max() <= tol_max and d.mean() <= tol_mean, f"{what}: max {d.max():.3e} mean {d.mean():.3e} (scale {scale:.3g})"


def _run(wl_name, layer=None):
    from windowed_attention_b200.layer import RibLayer
    inp = make_inputs(wl_name, layer=layer, with_grad=True)
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


def _oracle_threads(gb_per_task):
    """Threads for the oracle's per-(window, head) tasks: the host's cores,
    at most 8, and no more than the free memory holds (a task at N = 9216
    holds several N x N fp64 matrices)."""
    import psutil
    avail = psutil.virtual_memory().available / 2**30
    return max(1, min(8, oracle.oracle_cores(), int(avail // gb_per_task)))


def _windows_of(a, s, width):
    """[B][Hp][Wp][heads][width] (the padded head layout) -> [nW, N, C] in the
    oracle's window order and channel order head*dh + d."""
    dh = s.C // s.heads
    img = a.reshape(s.B, s.Hp, s.Wp, s.heads, width)[..., :dh].reshape(s.B, s.Hp, s.Wp, s.C)
    return oracle.window_partition(img, s.window)


def _check_layer_backward(inp, s, g, mlp_tol_mean):
    """Every gradient of RibLayer.backward against the oracle's layer backward:
    dQc, dKc, dV per (window, head) and in all, the dQp/dKp totals, dX, the
    projection and gate weights, and the coordinate-MLP weights end to end."""
    M, dh, R = s.window, s.C // s.heads, s.R
    ref, inner = oracle.rib_layer_backward(inp["X"], inp, inp["dY"], s.heads, s.R, s.L, M,
                                           threads=_oracle_threads(6.0))
    # the GPU's gradients are with respect to the stored Qc = Qc / sqrt(dh)
    # and the cached Qp = Qp / sqrt(R)
    got = {"Qc": _windows_of(_np(g["dQc"]), s, 32) / math.sqrt(dh), "Kc": _windows_of(_np(g["dKc"]), s, 32),
           "V": _windows_of(_np(g["dV"]), s, 32)}
    for k in ("Qc", "Kc", "V"):
        # each (window, head) block on its own scale, then the whole tensor
        for w in range(s.n_windows):
            for hd in range(s.heads):
                sl = slice(hd * dh, (hd + 1) * dh)
                _rel_check(got[k][w][:, sl], inner[k][w][:, sl], f"d{k} w{w} h{hd}")
        _rel_check(got[k], inner[k], f"d{k} (all windows)")
    _rel_check(_np(g["dQp"]).reshape(s.heads, M * M, R) / math.sqrt(R), inner["Qp"], "dQp total")
    _rel_check(_np(g["dKp"]).reshape(s.heads, M * M, R), inner["Kp"], "dKp total")
    for name in ("X", "Wq", "Wk", "Wv", "Wdw", "bdw", "Wpw", "bpw"):
        got = _np(g["d" + name]).reshape(np.shape(ref[name]))
        _rel_check(got, ref[name], f"d{name}")
    for name in ("Wh", "bh", "Wpq", "Wpk"):
        got = _np(g["d" + name]).reshape(np.shape(ref[name]))
        _rel_check(got, ref[name], f"d{name} (end to end)", tol_mean=mlp_tol_mean)
    return ref, inner


@pytest.mark.parametrize("window,H,W,C", [(16, 20, 40, 60), (32, 40, 72, 48), (64, 70, 64, 60)])
def test_backward_window_sizes_every_gradient(cuda_lib, window, H, W, C):
    """Windows 16, 32 and 64 (the lite model's cycle) on ragged maps padded to
    window multiples, with head widths below the padded width (dh = 20 of 32:
    the Q'' fold) and equal to it (dh = 16: P from the forward's lse). Each
    window size takes its own streamed-tile shape (64 tokens as 4 x 16, 2 x 32
    or 1 x 64 window cells) and its own 128-token tile; the whole chain
    (RibLayer.backward) against the oracle's layer backward. The end-to-end MLP
    gradients take mean <= 4e-3 as at the training shape (sums over every
    position of bf16-rounded dS)."""
    from windowed_attention_b200.workloads import LayerShape
    shape = LayerShape(B=1, H=H, W=W, C=C, heads=3, R=16, L=10, hidden=64, window=window, dtype="bf16")
    inp, s, lay, g = _run("tiny", layer=shape)
    assert s.window == window and s.n_windows == (-(-H // window)) * (-(-W // window))
    _check_layer_backward(inp, s, g, mlp_tol_mean=4e-3)


def test_backward_train_every_gradient(cuda_lib):
    """The training shape (16 patches of 96x96, C = 180, 6 heads, window 96:
    N = 9216, one window per patch) through the whole backward chain
    (RibLayer.backward), every gradient against the oracle's layer backward:
    dQc, dKc, dV of every window and head, the dQp/dKp totals over the 16
    windows, the coordinate-MLP weight gradients (the GPU's chunked reduction
    at N = 9216), dX and every weight gradient."""
    inp, s, lay, g = _run("train")
    M, R = s.window, s.R
    # end to end (through the GPU's own dQp/dKp) the MLP gradients are sums
    # over all N positions of dQp/dKp, whose rows of dS sum to zero exactly:
    # the bf16 roundings of the operands (Qc, Kc, V, the position caches, dO,
    # dS) then show in the normalised mean error at about 1.1-1.5e-3 at
    # N = 4096 (no single rounding dominates) and 2.4e-3 at N = 9216, so the
    # chained comparison takes mean <= 4e-3 (max stays 2e-2)
    ref, inner = _check_layer_backward(inp, s, g, mlp_tol_mean=4e-3)
    # The coordinate-MLP backward alone at N = 9216: rib_pos_encode_bwd fed
    # the oracle's dQp/dKp totals (as gradients of the caches: the cached Qp
    # carries 1/sqrt(R)) against the oracle's MLP gradients from the same totals.
    dev = "cuda"
    dqp = torch.tensor(inner["Qp"] * math.sqrt(R), dtype=torch.float32, device=dev).contiguous()
    dkp = torch.tensor(inner["Kp"], dtype=torch.float32, device=dev).contiguous()
    out = {"Wh": torch.empty(s.enc_dim, s.hidden, device=dev), "bh": torch.empty(s.hidden, device=dev),
           "Wpq": torch.empty(s.hidden, s.heads * R, device=dev), "Wpk": torch.empty(s.hidden, s.heads * R, device=dev)}
    import windowed_attention_b200 as rib
    ws = torch.empty(rib.rib_pos_encode_bwd_workspace_size(lay.mlp, M) // 4, dtype=torch.float32, device=dev)
    rib.rib_pos_encode_bwd(lay.mlp, M, dqp, dkp, out["Wh"], out["bh"], out["Wpq"], out["Wpk"], ws)
    torch.cuda.synchronize()
    rib.rib_device_error()
    for name in ("Wh", "bh", "Wpq", "Wpk"):
        _rel_check(_np(out[name]), ref[name], f"MLP d{name} from the oracle's dQp/dKp")
