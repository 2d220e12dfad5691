"""Pins of the oracle's coordinate grid, Fourier encoding and coordinate MLP.

Cited passages: the RIB/SST write-up (omica.com.cn), section 2.2
"RIB的核心设计" (CoordinateEncoder with L=10 bands giving [N, 2+4L]; implicit
neural field h = ReLU(r Wh + bh), Qp = h Wp_q, Kp = h Wp_k); the French
summary, "Résumé technique" 2.A (normalised 2-D coordinates + Fourier features).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_encoding_width_matches_page():
    # tests/golden/page_constants.json: L=10 -> 2+4L = 42 columns (section 2.2).
    with open(os.path.join(GOLDEN, "page_constants.json")) as f:
        g = json.load(f)
    L = g["fourier_bands_L"]
    r = oracle.fourier_encode(oracle.window_coords(8), L)
    assert r.shape == (64, g["encoding_width"])
    assert g["encoding_width"] == 42


def test_grid_corners_and_token_order():
    M = 5
    c = oracle.window_coords(M)
    assert c.shape == (25, 2)
    # corners: t = i*M + j, (row y, column x), both in [-1, 1] with endpoints
    assert tuple(c[0]) == (-1.0, -1.0)
    assert tuple(c[M - 1]) == (-1.0, 1.0)
    assert tuple(c[M * (M - 1)]) == (1.0, -1.0)
    assert tuple(c[-1]) == (1.0, 1.0)
    # centre token of an odd window is the origin
    assert np.all(c[12] == 0.0)
    # equal spacing 2/(M-1)
    assert np.allclose(np.diff(c[:M, 1]), 0.5)
    assert np.allclose(np.diff(c[::M, 0]), 0.5)


def test_encoding_at_origin_fixes_column_order():
    # At (0,0): raw coords 0, every sine 0, every cosine 1 -> pins the order
    # [coords, sin pair, cos pair] per band.
    r = oracle.fourier_encode(np.zeros((1, 2)), 3)[0]
    expect = [0, 0] + [0, 0, 1, 1] * 3
    assert r.tolist() == expect


def test_encoding_first_band_textbook_values():
    # band 0 has frequency 2^0 = 1 (no pi): sin(1), cos(1), sin(-0.5), cos(-0.5)
    r = oracle.fourier_encode(np.array([[1.0, -0.5]]), 1)[0]
    assert r[0] == 1.0 and r[1] == -0.5
    assert abs(r[2] - 0.8414709848078965) < 1e-15
    assert abs(r[3] - (-0.479425538604203)) < 1e-15
    assert abs(r[4] - 0.5403023058681398) < 1e-15
    assert abs(r[5] - 0.8775825618903728) < 1e-15


@pytest.mark.parametrize("L", [6, 15])
def test_encoding_frequencies_double_per_band(L):
    # sin(2a) = 2 sin a cos a and cos(2a) = 1 - 2 sin^2 a pin freq_i = 2^i
    # (L = 15: the write-up's section 6 variant, arguments up to 2^14)
    rng = np.random.default_rng(0)
    c = rng.uniform(-1, 1, size=(50, 2))
    r = oracle.fourier_encode(c, L)
    assert r.shape == (50, 2 + 4 * L)
    for i in range(1, L):
        s_prev, c_prev = r[:, 2 + 4 * (i - 1):4 + 4 * (i - 1)], r[:, 4 + 4 * (i - 1):6 + 4 * (i - 1)]
        s_i, c_i = r[:, 2 + 4 * i:4 + 4 * i], r[:, 4 + 4 * i:6 + 4 * i]
        assert np.allclose(s_i, 2 * s_prev * c_prev, atol=1e-12)
        assert np.allclose(c_i, 1 - 2 * s_prev ** 2, atol=1e-12)
        assert np.allclose(s_i ** 2 + c_i ** 2, 1.0, atol=1e-12)


def _selector(rows, cols, picks):
    m = np.zeros((rows, cols))
    for r, c in picks:
        m[r, c] = 1.0
    return m


def test_coord_mlp_selection_weights():
    # Selection weights make every output a known entry of the encoding, which
    # pins operand orientation (r Wh, not Wh r), the bias add, the ReLU and
    # the head-major split of Wp's heads*R columns.
    L, heads, R, hidden = 2, 2, 3, 4
    M = 3
    r = oracle.fourier_encode(oracle.window_coords(M), L)   # [9, 10]
    e = r.shape[1]
    Wh = _selector(e, hidden, [(0, 0), (1, 1), (4, 2), (5, 3)])   # y, x, cos(y), cos(x)
    bh = np.array([0.0, 0.0, -0.5, 0.25])
    Wpq = _selector(hidden, heads * R, [(0, 0), (1, 1), (2, 2), (3, 3), (0, 4), (3, 5)])
    Wpk = 2.0 * _selector(hidden, heads * R, [(1, 0), (2, 4)])
    qp, kp, _, _ = oracle.coord_mlp(r, Wh, bh, Wpq, Wpk, heads, R)
    assert qp.shape == (heads, M * M, R) and kp.shape == (heads, M * M, R)
    g = [-1.0, 0.0, 1.0]
    for t in range(M * M):
        y, x = g[t // M], g[t % M]
        h0, h1 = max(y, 0.0), max(x, 0.0)
        h2, h3 = max(math.cos(y) - 0.5, 0.0), max(math.cos(x) + 0.25, 0.0)
        assert np.allclose(qp[0, t], [h0, h1, h2], atol=1e-15)
        assert np.allclose(qp[1, t], [h3, h0, h3], atol=1e-15)
        assert np.allclose(kp[0, t], [2 * h1, 0, 0], atol=1e-15)
        assert np.allclose(kp[1, t], [0, 2 * h2, 0], atol=1e-15)


def test_coord_mlp_relu_cuts_negative_trunk():
    L, heads, R, hidden = 1, 1, 2, 3
    r = oracle.fourier_encode(oracle.window_coords(4), L)
    rng = np.random.default_rng(1)
    Wh = rng.normal(size=(r.shape[1], hidden)) * 0.1
    bh = np.full(hidden, -100.0)
    qp, kp, _, _ = oracle.coord_mlp(r, Wh, bh, rng.normal(size=(hidden, R)), rng.normal(size=(hidden, R)), heads, R)
    assert np.all(qp == 0) and np.all(kp == 0)


def test_pos_features_shapes_for_page_windows():
    with open(os.path.join(GOLDEN, "page_constants.json")) as f:
        g = json.load(f)
    rng = np.random.default_rng(2)
    L, heads, R, hidden = g["fourier_bands_L"], g["lite"]["heads"], g["lite"]["R"], 8
    Wh = rng.normal(size=(2 + 4 * L, hidden))
    for M in sorted(set(g["cyclic_window_sizes"])):
        qp, kp = oracle.pos_features(M, L, Wh, np.zeros(hidden), rng.normal(size=(hidden, heads * R)),
                                     rng.normal(size=(hidden, heads * R)), heads, R)
        assert qp.shape == (heads, M * M, R) == kp.shape
