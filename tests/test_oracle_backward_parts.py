"""Pins of the oracle's backward building blocks on their own (the GPU tests
call them directly, with gradients that do not come from a layer): each is
checked by central finite differences of the matching forward function in
fp64, and the content projection by brute-force loops.

The forward functions are the pages' definitions: Qc, Kc, V = X Wq, X Wk,
X Wv (the RIB write-up, section 2.2, content vectors), the CLA gate's
G = PWConv(DWConv3x3(X)) (section 2.3) and the coordinate MLP
h = ReLU(r Wh + bh), Qp = h Wp_q, Kp = h Wp_k (section 2.2).
"""
import numpy as np
import pytest

import oracle


def _fd(loss, arr, h=1e-6):
    """Central differences of a scalar loss over every element of arr."""
    g = np.zeros_like(arr)
    for idx in np.ndindex(arr.shape):
        old = arr[idx]
        arr[idx] = old + h
        fp = loss()
        arr[idx] = old - h
        fm = loss()
        arr[idx] = old
        g[idx] = (fp - fm) / (2 * h)
    return g


def _close(a, b, tol=2e-6):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    assert np.max(np.abs(a - b)) <= tol * max(1.0, float(np.max(np.abs(b))))


def test_qkv_project_brute_force():
    rng = np.random.default_rng(40)
    T, C = 5, 6
    X = rng.normal(size=(T, C))
    Ws = [rng.normal(size=(C, C)) for _ in range(3)]
    got = oracle.qkv_project(X, *Ws)
    for W, out in zip(Ws, got):
        ref = np.zeros((T, C))
        for t in range(T):
            for j in range(C):
                s = 0.0
                for k in range(C):
                    s += X[t, k] * W[k, j]
                ref[t, j] = s
        assert np.max(np.abs(out - ref)) < 1e-12
    # the three outputs use their own weights (not a shared or swapped one)
    assert not np.allclose(got[0], got[1]) and not np.allclose(got[1], got[2])


def test_qkv_project_backward_finite_differences():
    rng = np.random.default_rng(41)
    T, C = 4, 5
    X = rng.normal(size=(T, C))
    Wq, Wk, Wv = (rng.normal(size=(C, C)) for _ in range(3))
    gq, gk, gv = (rng.normal(size=(T, C)) for _ in range(3))

    def loss():
        q, k, v = oracle.qkv_project(X, Wq, Wk, Wv)
        return float((q * gq).sum() + (k * gk).sum() + (v * gv).sum())

    dX, dWq, dWk, dWv = oracle.qkv_project_backward(X, Wq, Wk, Wv, gq, gk, gv)
    _close(dX, _fd(loss, X))
    _close(dWq, _fd(loss, Wq))
    _close(dWk, _fd(loss, Wk))
    _close(dWv, _fd(loss, Wv))


@pytest.mark.parametrize("B,H,W,C", [(1, 3, 4, 4), (2, 2, 5, 8), (1, 1, 1, 4)])
def test_cla_gate_backward_finite_differences(B, H, W, C):
    # G = DWConv3x3(X) Wpw + bpw; loss = sum(G * dG); includes 1-pixel maps
    # (every tap but the centre falls on the zero border)
    rng = np.random.default_rng(42 + H * W)
    X = rng.normal(size=(B, H, W, C))
    Wdw = rng.normal(size=(C, 3, 3))
    bdw = rng.normal(size=C)
    Wpw = rng.normal(size=(C, C))
    bpw = rng.normal(size=C)
    dG = rng.normal(size=(B, H, W, C))

    def loss():
        G = oracle.pwconv(oracle.dwconv3x3(X, Wdw, bdw), Wpw, bpw)
        return float((G * dG).sum())

    dX, dWdw, dbdw, dWpw, dbpw = oracle.cla_gate_backward(X, Wdw, bdw, Wpw, dG)
    _close(dX, _fd(loss, X))
    _close(dWdw, _fd(loss, Wdw))
    _close(dbdw, _fd(loss, bdw))
    _close(dWpw, _fd(loss, Wpw))
    _close(dbpw, _fd(loss, bpw))


@pytest.mark.parametrize("M,L", [(3, 2), (4, 1)])
def test_pos_features_backward_finite_differences(M, L):
    rng = np.random.default_rng(43 + M)
    heads, R, hidden = 2, 3, 5
    F = 2 + 4 * L
    Wh = rng.normal(size=(F, hidden))
    bh = rng.normal(size=hidden)
    Wpq = rng.normal(size=(hidden, heads * R))
    Wpk = rng.normal(size=(hidden, heads * R))
    N = M * M
    dQp = rng.normal(size=(heads, N, R))
    dKp = rng.normal(size=(heads, N, R))

    def loss():
        qp, kp = oracle.pos_features(M, L, Wh, bh, Wpq, Wpk, heads, R)
        return float((qp * dQp).sum() + (kp * dKp).sum())

    # no pre-activation within the step of the ReLU kink, so the
    # differences see one linear piece
    r = oracle.fourier_encode(oracle.window_coords(M), L)
    assert np.min(np.abs(r @ Wh + bh)) > 1e-4
    g = oracle.pos_features_backward(M, L, Wh, bh, Wpq, Wpk, heads, R, dQp, dKp)
    for name, arr in (("Wh", Wh), ("bh", bh), ("Wpq", Wpq), ("Wpk", Wpk)):
        _close(g[name], _fd(loss, arr))
