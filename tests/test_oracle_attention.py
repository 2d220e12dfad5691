"""Pins of the oracle's RIB score and per-window attention.

Cited passages: RIB/SST write-up section 2.2 "注意力计算重构" (RPB form
S = Qc Kc^T/sqrt(D) + B; RIB form Q = [Qc/sqrt(D), Qp/sqrt(R)], K = [Kc, Kp],
S = Q K^T equal to Qc Kc^T/sqrt(D) + Qp Kp^T/sqrt(R)); the French summary,
2.A, "[Qc,Qp][Kc,Kp]^T = QcKc^T + QpKp^T".
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _rand(rng, *shape):
    return rng.normal(size=shape)


@pytest.mark.parametrize("n,dh,R", [(16, 4, 3), (64, 30, 16), (33, 16, 16)])
def test_concatenation_identity(n, dh, R):
    rng = np.random.default_rng(n)
    qc, kc, qp, kp = _rand(rng, n, dh), _rand(rng, n, dh), _rand(rng, n, R), _rand(rng, n, R)
    a = oracle.rib_scores(qc, kc, qp, kp, dh, R)
    b = oracle.rib_scores_concat(qc, kc, qp, kp, dh, R)
    assert np.max(np.abs(a - b)) <= 1e-12 * max(1.0, np.max(np.abs(a)))


def test_zero_position_features_reduce_to_sdpa():
    # Qp = 0 -> plain scaled dot-product attention with scale 1/sqrt(dh).
    rng = np.random.default_rng(3)
    n, dh, R = 40, 8, 5
    qc, kc, v = _rand(rng, n, dh), _rand(rng, n, dh), _rand(rng, n, 7)
    kp = _rand(rng, n, R)
    o = oracle.attention_window(qc, kc, v, np.zeros((n, R)), kp, dh, R)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(qc)[None], torch.tensor(kc)[None], torch.tensor(v)[None]).numpy()[0]
    assert np.max(np.abs(o - ref)) < 1e-12


def test_positional_term_equals_explicit_bias():
    # The RPB form with B = Qp Kp^T / sqrt(R) as an additive mask.
    rng = np.random.default_rng(4)
    n, dh, R = 50, 6, 4
    qc, kc, v, qp, kp = (_rand(rng, n, dh), _rand(rng, n, dh), _rand(rng, n, 6),
                         _rand(rng, n, R), _rand(rng, n, R))
    bias = torch.tensor(qp) @ torch.tensor(kp).T / math.sqrt(R)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(qc)[None], torch.tensor(kc)[None], torch.tensor(v)[None],
        attn_mask=bias[None]).numpy()[0]
    o = oracle.attention_window(qc, kc, v, qp, kp, dh, R)
    assert np.max(np.abs(o - ref)) < 1e-12


def test_softmax_rows_sum_to_one_and_shift_invariant():
    rng = np.random.default_rng(5)
    S = rng.normal(size=(20, 31)) * 30
    P = oracle.softmax_rows(S)
    assert np.allclose(P.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(P >= 0)
    P2 = oracle.softmax_rows(S + rng.normal(size=(20, 1)) * 100)
    assert np.allclose(P, P2, atol=1e-13)


def test_two_keys_closed_form():
    # one query, two keys: O = (e^s1 v1 + e^s2 v2) / (e^s1 + e^s2)
    dh, R = 4, 2
    qc = np.array([[1.0, 0.0, 2.0, 0.0]])
    kc = np.array([[1.0, 1.0, 0.0, 0.0], [0.0, 0.0, 1.0, 0.0]])
    qp = np.array([[0.5, -1.0]])
    kp = np.array([[2.0, 0.0], [0.0, 1.0]])
    v = np.array([[1.0, -2.0], [3.0, 4.0]])
    s1 = 1.0 / 2.0 + 1.0 / math.sqrt(2)          # qc.kc1/sqrt(4) + qp.kp1/sqrt(2)
    s2 = 2.0 / 2.0 - 1.0 / math.sqrt(2)
    w1 = math.exp(s1) / (math.exp(s1) + math.exp(s2))
    expect = w1 * v[0] + (1 - w1) * v[1]
    o = oracle.attention_window(qc, kc, v, qp, kp, dh, R)
    assert np.allclose(o[0], expect, atol=1e-15)


def test_key_permutation_invariance_query_equivariance():
    # Attention inside a window does not depend on the order of its tokens,
    # which is what allows any tiling of a window.
    rng = np.random.default_rng(6)
    n, dh, R = 24, 5, 3
    qc, kc, v, qp, kp = (_rand(rng, n, dh), _rand(rng, n, dh), _rand(rng, n, 4),
                         _rand(rng, n, R), _rand(rng, n, R))
    o = oracle.attention_window(qc, kc, v, qp, kp, dh, R)
    pk = rng.permutation(n)
    o2 = oracle.attention_window(qc, kc[pk], v[pk], qp, kp[pk], dh, R)
    assert np.allclose(o, o2, atol=1e-13)
    pq = rng.permutation(n)
    o3 = oracle.attention_window(qc[pq], kc, v, qp[pq], kp, dh, R)
    assert np.allclose(o[pq], o3, atol=1e-13)


def test_constant_values_pass_through():
    rng = np.random.default_rng(7)
    n, dh, R = 16, 4, 4
    v = np.tile(np.array([[1.5, -2.0, 0.25]]), (n, 1))
    o = oracle.attention_window(_rand(rng, n, dh), _rand(rng, n, dh), v, _rand(rng, n, R), _rand(rng, n, R), dh, R)
    assert np.allclose(o, v, atol=1e-14)


def test_lse_matches_log_sum_exp():
    rng = np.random.default_rng(8)
    n, dh, R = 12, 3, 2
    qc, kc, v, qp, kp = (_rand(rng, n, dh), _rand(rng, n, dh), _rand(rng, n, 3),
                         _rand(rng, n, R), _rand(rng, n, R))
    _, P, lse = oracle.attention_window(qc, kc, v, qp, kp, dh, R, return_p=True)
    S = torch.tensor(qc) @ torch.tensor(kc).T / math.sqrt(dh) + torch.tensor(qp) @ torch.tensor(kp).T / math.sqrt(R)
    assert np.allclose(lse, torch.logsumexp(S, dim=1).numpy(), atol=1e-13)
    assert np.allclose(P, np.exp(S.numpy() - lse[:, None]), atol=1e-14)


# ------------------------------------------------------------------ optional key-padding mask
def test_key_mask_equals_attention_over_the_kept_keys():
    """Masking keys is the same as dropping them: attention over the kept
    rows of Kc, Kp and V only (a different formulation)."""
    rng = np.random.default_rng(7)
    N, dh, R = 36, 6, 4
    qc, kc, v = rng.standard_normal((N, dh)), rng.standard_normal((N, dh)), rng.standard_normal((N, 5))
    qp, kp = rng.standard_normal((N, R)), rng.standard_normal((N, R))
    mask = np.zeros(N, bool)
    mask[[3, 4, 10, 20, 35]] = True
    keep = ~mask
    got = oracle.attention_window(qc, kc, v, qp, kp, dh, R, key_mask=mask)
    ref = oracle.attention_window(qc, kc[keep], v[keep], qp, kp[keep], dh, R)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_padding_key_mask_marks_exactly_the_padded_tokens():
    H, W, M = 20, 13, 8          # padded to 24 x 16: 3 x 2 windows per image, 2 images
    Hp, Wp = 24, 16
    X = np.zeros((2, Hp, Wp, 1))
    X[:, :H, :W, 0] = 1.0        # 1 on real pixels
    xw = oracle.window_partition(X, M)
    for w in range(xw.shape[0]):
        m = oracle.padding_key_mask(w, M, H, W, Hp, Wp)
        assert np.array_equal(m, xw[w][:, 0] == 0.0)


def test_mask_padding_changes_only_windows_with_padding():
    rng = np.random.default_rng(8)
    B, H, W, C, heads, M, R = 1, 12, 20, 8, 2, 8, 4     # 2 x 3 windows, bottom row and right column padded
    X = rng.standard_normal((B, H, W, C))
    Wq, Wk, Wv = (rng.standard_normal((C, C)) / np.sqrt(C) for _ in range(3))
    qp, kp = rng.standard_normal((heads, M * M, R)), rng.standard_normal((heads, M * M, R))
    a = oracle.rib_attention(X, Wq, Wk, Wv, qp, kp, heads, M)
    b = oracle.rib_attention(X, Wq, Wk, Wv, qp, kp, heads, M, mask_padding=True)
    # window (0, 0) has no padding: identical; every padded window differs
    assert np.array_equal(a[0, :M, :M], b[0, :M, :M])
    assert not np.allclose(a[0, :M, 2 * M:3 * M], b[0, :M, 2 * M:3 * M])
    assert not np.allclose(a[0, M:2 * M, :M], b[0, M:2 * M, :M])
