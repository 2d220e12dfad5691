"""Pins of the oracle's window partition/reverse, padding, CLA convs and LayerNorm.

Cited passages: RIB/SST write-up section 2.3 "卷积局部注意力(CLA)"
(X_2d = rearrange(X, 'b (h w) c -> b c h w'), G = PWConv(DWConv3x3(X_2d)),
O = softmax(S)V * sigma(G)); section 3.1 (LayerNorm before RIB attention).
"""
import numpy as np
import pytest
import torch

import oracle


def _payload(B, H, W, C):
    # integer payload that encodes (b, y, x, c) exactly in float64
    b, y, x, c = np.meshgrid(np.arange(B), np.arange(H), np.arange(W), np.arange(C), indexing="ij")
    return (((b * 1000 + y) * 1000 + x) * 100 + c).astype(np.float64)


@pytest.mark.parametrize("B,H,W,M", [(1, 32, 32, 16), (2, 18, 40, 8), (1, 5, 7, 4), (3, 96, 96, 96)])
def test_partition_reverse_bijection(B, H, W, M):
    X = _payload(B, H, W, 2)
    Xp = oracle.pad_to_windows(X, M)
    Hp, Wp = Xp.shape[1:3]
    assert Hp % M == 0 and Wp % M == 0 and Hp - H < M and Wp - W < M
    assert np.all(Xp[:, H:] == 0) and np.all(Xp[:, :, W:] == 0)
    win = oracle.window_partition(Xp, M)
    assert win.shape == (B * (Hp // M) * (Wp // M), M * M, 2)
    back = oracle.window_reverse(win, M, B, Hp, Wp)
    assert np.array_equal(back, Xp)
    # every position lands where window_token_index says, bit-exact
    for b in range(B):
        for y in range(0, H, max(1, H // 5)):
            for x in range(0, W, max(1, W // 5)):
                w, t = oracle.window_token_index(b, y, x, M, Hp, Wp)
                assert np.array_equal(win[w, t], X[b, y, x])
    # a permutation: all payload values appear exactly once
    vals = win[..., 0].reshape(-1)
    real = vals[vals != 0]
    assert len(np.unique(real)) == len(real) == B * H * W - (1 if np.any(X[..., 0] == 0) else 0)


def test_partition_matches_torch_rearrange():
    # rearrange 'b (ny M) (nx M) c -> (b ny nx) (M M) c' through torch views
    B, H, W, C, M = 2, 16, 24, 3, 8
    X = _payload(B, H, W, C)
    t = torch.tensor(X).view(B, H // M, M, W // M, M, C).permute(0, 1, 3, 2, 4, 5).reshape(-1, M * M, C)
    assert np.array_equal(oracle.window_partition(X, M), t.numpy())


@pytest.mark.parametrize("B,H,W,C", [(1, 9, 11, 5), (2, 4, 4, 3)])
def test_dwconv_matches_conv2d(B, H, W, C):
    rng = np.random.default_rng(0)
    X, Wd, bd = rng.normal(size=(B, H, W, C)), rng.normal(size=(C, 3, 3)), rng.normal(size=C)
    ref = torch.nn.functional.conv2d(torch.tensor(X).permute(0, 3, 1, 2), torch.tensor(Wd)[:, None],
                                     torch.tensor(bd), padding=1, groups=C).permute(0, 2, 3, 1).numpy()
    assert np.max(np.abs(oracle.dwconv3x3(X, Wd, bd) - ref)) < 1e-12


def test_dwconv_delta_filter_is_shift():
    # a filter with a single 1 at (ky,kx) shifts the map by (ky-1, kx-1)
    rng = np.random.default_rng(1)
    X = rng.normal(size=(1, 6, 7, 2))
    Wd = np.zeros((2, 3, 3))
    Wd[:, 0, 2] = 1.0      # out[y,x] = X[y-1, x+1]
    out = oracle.dwconv3x3(X, Wd, np.zeros(2))
    assert np.array_equal(out[0, 1:, :-1], X[0, :-1, 1:])
    assert np.all(out[0, 0] == 0) and np.all(out[0, :, -1] == 0)


def test_pwconv_matches_conv2d():
    rng = np.random.default_rng(2)
    B, H, W, Ci, Co = 2, 5, 6, 7, 4
    X, Wp, bp = rng.normal(size=(B, H, W, Ci)), rng.normal(size=(Ci, Co)), rng.normal(size=Co)
    ref = torch.nn.functional.conv2d(torch.tensor(X).permute(0, 3, 1, 2), torch.tensor(Wp).T[:, :, None, None],
                                     torch.tensor(bp)).permute(0, 2, 3, 1).numpy()
    assert np.max(np.abs(oracle.pwconv(X, Wp, bp) - ref)) < 1e-12


def test_sigmoid_values():
    s = oracle.sigmoid(np.array([0.0, 2.0, -2.0, 40.0, -40.0]))
    assert s[0] == 0.5
    assert abs(s[1] + s[2] - 1.0) < 1e-15
    assert abs(s[1] - 0.8807970779778823) < 1e-15
    assert s[3] > 1 - 1e-15 and s[4] < 1e-17


def test_cla_gate_range_and_composition():
    rng = np.random.default_rng(3)
    X = rng.normal(size=(1, 5, 5, 4))
    Wd, bd, Wp, bp = rng.normal(size=(4, 3, 3)), rng.normal(size=4), rng.normal(size=(4, 4)), rng.normal(size=4)
    g = oracle.cla_gate(X, Wd, bd, Wp, bp)
    assert np.all((g > 0) & (g < 1))
    ref = torch.sigmoid(torch.nn.functional.conv2d(
        torch.nn.functional.conv2d(torch.tensor(X).permute(0, 3, 1, 2), torch.tensor(Wd)[:, None], torch.tensor(bd),
                                   padding=1, groups=4),
        torch.tensor(Wp).T[:, :, None, None], torch.tensor(bp))).permute(0, 2, 3, 1).numpy()
    assert np.max(np.abs(g - ref)) < 1e-14


def test_layernorm_matches_torch():
    rng = np.random.default_rng(4)
    x = rng.normal(size=(2, 3, 4, 180)) * 3 + 1
    ref = torch.nn.functional.layer_norm(torch.tensor(x), (180,), eps=1e-5).numpy()
    assert np.max(np.abs(oracle.layernorm(x) - ref)) < 1e-12
