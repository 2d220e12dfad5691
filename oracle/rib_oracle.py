"""Plain, slow, fp64 oracle of the RIB windowed-attention layer with CLA gate.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this module; it
shares no code, table or constant with the CUDA kernels. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use it.

Sources (the one page of the RIB/SST write-up that prints formulas and code,
"FlashAttention-accelerated super-resolution Transformer", omica.com.cn; its
sections are cited by number and Chinese heading):

* section 2.2 "RIB的核心设计" - the coordinate encoder (coords first, then per
  band i<L a sine and a cosine of 2^i * coords), the implicit neural field
  h = ReLU(r Wh + bh), Qp = h Wp_q, Kp = h Wp_k, and the score
  S = Qc Kc^T / sqrt(D) + Qp Kp^T / sqrt(R), written as one product of the
  concatenations Q = [Qc/sqrt(D), Qp/sqrt(R)], K = [Kc, Kp];
* section 2.3 "卷积局部注意力(CLA)" - the gate G = PWConv(DWConv3x3(X)) applied
  as O = softmax(S) V * sigmoid(G), with the image rearranged b (h w) c <->
  b c h w;
* section 3.1 "模型架构设计" - a block is LayerNorm -> RIB attention -> CLA
  -> ConvFFN (FFN expansion 1.25);
* section 3.2 "循环窗口策略" - window sizes cycled 16,32,64,16,32,64;
* section 5.2 "推理优化技巧" - Qp/Kp are precomputed once and reused.

The French summary of the same paper ("Résumé technique", 2. A, RIB) states
the concatenation identity [Qc,Qp][Kc,Kp]^T = Qc Kc^T + Qp Kp^T and that the
coordinates are normalised 2-D coordinates with Fourier features.

Readings where the pages are silent (each is listed in the design notes):
* D in 1/sqrt(D) is the per-head content dimension dh;
* the window grid is linspace(-1, 1, M) on both axes, token t = i*M + j,
  coordinate pair ordered (row y, column x);
* frequencies are 2^i without a factor pi, i = 0..L-1;
* one MLP trunk (Wh, bh) per layer; Wp_q, Wp_k map the hidden width to
  heads*R columns (head-major), no bias on Wp;
* Q/K/V projections are bias-free; the depthwise and pointwise convs have
  biases; there is no output projection after the gate;
* the map is zero-padded bottom/right to window multiples before the
  projections; padded tokens are unmasked keys (Kc = V = 0, Kp from the
  grid) and padded query rows are cropped; the convs see the unpadded map
  with zero borders;
* the gate reads the same X that feeds Q/K/V;
* a stack block is x <- x + Y(LayerNorm(x)), LayerNorm with unit gain,
  zero shift, eps 1e-5;
* ConvFFN (named, not defined, in section 3.1): hidden width 1.25 C, GELU
  in its erf form, h + DWConv3x3(h) on the hidden features, then the output
  linear map; the full SST block adds it as a second pre-norm residual,
  x <- x + ConvFFN(LayerNorm(x)).

Every function is pinned by ``tests/test_oracle_*.py`` against closed forms,
library routines used as textbook definitions (torch fp64 SDPA, conv2d,
layer_norm), identities and finite differences.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "window_coords", "fourier_encode", "coord_mlp", "pos_features",
    "pad_to_windows", "window_partition", "window_reverse", "window_token_index",
    "softmax_rows", "rib_scores", "rib_scores_concat", "attention_window", "padding_key_mask",
    "qkv_project", "rib_attention", "dwconv3x3", "pwconv", "sigmoid", "cla_gate",
    "layernorm", "rib_layer_forward", "rib_layer_backward", "rib_layer_forward_windows",
    "stack_forward", "attention_window_backward", "pos_features_backward",
    "qkv_project_backward", "cla_gate_backward",
    "gelu", "conv_ffn", "sst_block", "sst_stack_forward",
    "oracle_cores",
]


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# a1: window coordinate grid and Fourier encoding (section 2.2, CoordinateEncoder)
# --------------------------------------------------------------------------
def window_coords(M: int) -> np.ndarray:
    """Normalised 2-D coordinates of the M*M tokens of one window, [N, 2].

    Section 2.2 gives coords of shape [N, 2] in [-1, 1]; token t = i*M + j has
    (y_i, x_j) with y = x = linspace(-1, 1, M) (endpoints included)."""
    if M == 1:
        g = np.zeros(1)
    else:
        g = -1.0 + 2.0 * np.arange(M, dtype=np.float64) / (M - 1)
    yy, xx = np.meshgrid(g, g, indexing="ij")
    return np.stack([yy.reshape(-1), xx.reshape(-1)], axis=1)


def fourier_encode(coords: np.ndarray, L: int) -> np.ndarray:
    """Section 2.2 CoordinateEncoder: [coords, sin(2^0 c), cos(2^0 c), ...,
    sin(2^(L-1) c), cos(2^(L-1) c)] concatenated on the last axis, [N, 2+4L]."""
    c = _f64(coords)
    parts = [c]
    for i in range(L):
        freq = 2.0 ** i
        parts.append(np.sin(freq * c))
        parts.append(np.cos(freq * c))
    return np.concatenate(parts, axis=-1)


# --------------------------------------------------------------------------
# a2: implicit neural field (section 2.2 "隐式神经场")
# --------------------------------------------------------------------------
def coord_mlp(r, Wh, bh, Wpq, Wpk, heads: int, R: int):
    """h = ReLU(r Wh + bh); Qp = h Wp_q; Kp = h Wp_k, split per head.

    Returns (Qp, Kp, pre, h) with Qp, Kp of shape [heads, N, R] (unscaled;
    the 1/sqrt(R) of the score is applied where the score is formed)."""
    r, Wh, bh, Wpq, Wpk = map(_f64, (r, Wh, bh, Wpq, Wpk))
    pre = r @ Wh + bh
    h = np.maximum(pre, 0.0)
    qp = h @ Wpq
    kp = h @ Wpk
    n = r.shape[0]
    qp = qp.reshape(n, heads, R).transpose(1, 0, 2)
    kp = kp.reshape(n, heads, R).transpose(1, 0, 2)
    return qp, kp, pre, h


def pos_features(M: int, L: int, Wh, bh, Wpq, Wpk, heads: int, R: int):
    """Qp, Kp [heads, M*M, R] for window side M (computed once per size and
    reused, section 5.2 "位置表征缓存")."""
    r = fourier_encode(window_coords(M), L)
    qp, kp, _, _ = coord_mlp(r, Wh, bh, Wpq, Wpk, heads, R)
    return qp, kp


# --------------------------------------------------------------------------
# window partition / reverse (section 2.3 rearrange; zero padding to multiples)
# --------------------------------------------------------------------------
def pad_to_windows(X: np.ndarray, M: int) -> np.ndarray:
    """Zero-pad [B, H, W, C] at the bottom and right to multiples of M."""
    X = _f64(X)
    B, H, W, C = X.shape
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    out = np.zeros((B, Hp, Wp, C))
    out[:, :H, :W] = X
    return out


def window_partition(Xp: np.ndarray, M: int) -> np.ndarray:
    """[B, Hp, Wp, C] -> [B*nWy*nWx, M*M, C]; window index (b, wy, wx) row-major,
    token t = i*M + j inside a window."""
    B, Hp, Wp, C = Xp.shape
    ny, nx = Hp // M, Wp // M
    out = np.empty((B * ny * nx, M * M, C), dtype=Xp.dtype)
    w = 0
    for b in range(B):
        for wy in range(ny):
            for wx in range(nx):
                blk = Xp[b, wy * M:(wy + 1) * M, wx * M:(wx + 1) * M, :]
                out[w] = blk.reshape(M * M, C)
                w += 1
    return out


def window_reverse(win: np.ndarray, M: int, B: int, Hp: int, Wp: int) -> np.ndarray:
    """Inverse of :func:`window_partition`."""
    C = win.shape[-1]
    ny, nx = Hp // M, Wp // M
    out = np.empty((B, Hp, Wp, C), dtype=win.dtype)
    w = 0
    for b in range(B):
        for wy in range(ny):
            for wx in range(nx):
                out[b, wy * M:(wy + 1) * M, wx * M:(wx + 1) * M, :] = win[w].reshape(M, M, C)
                w += 1
    return out


def window_token_index(b: int, y: int, x: int, M: int, Hp: int, Wp: int) -> Tuple[int, int]:
    """(window id, token id) of image position (b, y, x) after partition."""
    ny, nx = Hp // M, Wp // M
    w = (b * ny + y // M) * nx + x // M
    return w, (y % M) * M + (x % M)


# --------------------------------------------------------------------------
# a4: RIB attention for one window and head (section 2.2 "注意力计算重构")
# --------------------------------------------------------------------------
def softmax_rows(S: np.ndarray) -> np.ndarray:
    """Row softmax with the row maximum subtracted first."""
    m = S.max(axis=-1, keepdims=True)
    e = np.exp(S - m)
    return e / e.sum(axis=-1, keepdims=True)


def rib_scores(Qc, Kc, Qp, Kp, D: float, R: float) -> np.ndarray:
    """S = Qc Kc^T / sqrt(D) + Qp Kp^T / sqrt(R): content term plus the
    rank-R positional term, formed explicitly as an N x N matrix."""
    Qc, Kc, Qp, Kp = map(_f64, (Qc, Kc, Qp, Kp))
    return (Qc @ Kc.T) / math.sqrt(D) + (Qp @ Kp.T) / math.sqrt(R)


def rib_scores_concat(Qc, Kc, Qp, Kp, D: float, R: float) -> np.ndarray:
    """Same score from one product of the concatenations
    Q = [Qc/sqrt(D), Qp/sqrt(R)], K = [Kc, Kp] ([N, D+R] each)."""
    Qc, Kc, Qp, Kp = map(_f64, (Qc, Kc, Qp, Kp))
    Q = np.concatenate([Qc / math.sqrt(D), Qp / math.sqrt(R)], axis=1)
    K = np.concatenate([Kc, Kp], axis=1)
    return Q @ K.T


def attention_window(Qc, Kc, V, Qp, Kp, D: float, R: float, return_p: bool = False, key_mask=None):
    """O = softmax(S) V for one window and head, S from :func:`rib_scores`.
    ``key_mask`` (bool [N], True = excluded) removes keys from every row's
    softmax (their scores become -inf).

    Returns O [N, dv] (and P, and the row log-sum-exp if ``return_p``)."""
    S = rib_scores(Qc, Kc, Qp, Kp, D, R)
    if key_mask is not None:
        S = np.where(np.asarray(key_mask, bool)[None, :], -np.inf, S)
    P = softmax_rows(S)
    O = P @ _f64(V)
    if return_p:
        m = S.max(axis=-1)
        lse = m + np.log(np.exp(S - m[:, None]).sum(axis=-1))
        return O, P, lse
    return O


def oracle_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# --------------------------------------------------------------------------
# a3 + a4 over a whole map
# --------------------------------------------------------------------------
def qkv_project(X, Wq, Wk, Wv):
    """Content features Qc = X Wq, Kc = X Wk, V = X Wv (bias-free), channels last."""
    X = _f64(X)
    return X @ _f64(Wq), X @ _f64(Wk), X @ _f64(Wv)


def padding_key_mask(w: int, M: int, H: int, W: int, Hp: int, Wp: int) -> np.ndarray:
    """Key-padding mask of window w (window order of :func:`window_partition`):
    True for the window's tokens that lie in the zero padding (row >= H or
    column >= W of the image)."""
    ny, nx = Hp // M, Wp // M
    rem = w % (ny * nx)
    wy, wx = divmod(rem, nx)
    i, j = np.divmod(np.arange(M * M), M)
    return (wy * M + i >= H) | (wx * M + j >= W)


def rib_attention(X, Wq, Wk, Wv, Qp, Kp, heads: int, M: int,
                  threads: Optional[int] = None, window_ids: Optional[Sequence[int]] = None,
                  return_lse: bool = False, mask_padding: bool = False):
    """Windowed RIB attention of a map X [B, H, W, C] (before the gate).

    Pads X to window multiples, projects, partitions, runs
    :func:`attention_window` for every (window, head) and reverses. Returns
    the padded output [B, Hp, Wp, C] (heads concatenated, channel
    = head*dh + j). With ``window_ids`` only those windows are computed (the
    rest of the output is NaN). ``threads`` parallelises over (window, head).
    ``mask_padding`` excludes the padded tokens from every softmax as keys
    (the masked reading of the padding; by default they are unmasked keys
    with Kc = V = 0).
    """
    X = _f64(X)
    B, H, W, C = X.shape
    dh = C // heads
    R = Qp.shape[-1]
    Xp = pad_to_windows(X, M)
    Hp, Wp = Xp.shape[1], Xp.shape[2]
    xw = window_partition(Xp, M)
    nwin = xw.shape[0]
    ids = list(range(nwin)) if window_ids is None else list(window_ids)
    Wq, Wk, Wv = _f64(Wq), _f64(Wk), _f64(Wv)
    out = np.full((nwin, M * M, C), np.nan)
    lse = np.full((nwin, heads, M * M), np.nan)

    def run(task):
        w, hd = task
        qc = xw[w] @ Wq[:, hd * dh:(hd + 1) * dh]
        kc = xw[w] @ Wk[:, hd * dh:(hd + 1) * dh]
        v = xw[w] @ Wv[:, hd * dh:(hd + 1) * dh]
        km = padding_key_mask(w, M, H, W, Hp, Wp) if mask_padding else None
        o, _, l = attention_window(qc, kc, v, Qp[hd], Kp[hd], dh, R, return_p=True, key_mask=km)
        out[w, :, hd * dh:(hd + 1) * dh] = o
        lse[w, hd] = l

    tasks = [(w, hd) for w in ids for hd in range(heads)]
    if threads and threads > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(run, tasks))
    else:
        for t in tasks:
            run(t)
    full = window_reverse(out, M, B, Hp, Wp)
    if return_lse:
        return full, lse
    return full


# --------------------------------------------------------------------------
# a5, a6: CLA gate (section 2.3)
# --------------------------------------------------------------------------
def dwconv3x3(X, Wdw, bdw) -> np.ndarray:
    """Depthwise 3x3 conv, zero padding 1, one filter and bias per channel:
    out[b,y,x,c] = bdw[c] + sum_{dy,dx in -1..1} Wdw[c,dy+1,dx+1] X[b,y+dy,x+dx,c]."""
    X, Wdw, bdw = _f64(X), _f64(Wdw), _f64(bdw)
    B, H, W, C = X.shape
    Xp = np.zeros((B, H + 2, W + 2, C))
    Xp[:, 1:H + 1, 1:W + 1] = X
    out = np.broadcast_to(bdw, (B, H, W, C)).copy()
    for ky in range(3):
        for kx in range(3):
            out += Xp[:, ky:ky + H, kx:kx + W, :] * Wdw[:, ky, kx]
    return out


def pwconv(Dw, Wpw, bpw) -> np.ndarray:
    """Pointwise (1x1) conv, channels last: G = Dw Wpw + bpw, Wpw [C_in, C_out]."""
    return _f64(Dw) @ _f64(Wpw) + _f64(bpw)


def sigmoid(x) -> np.ndarray:
    x = _f64(x)
    return 1.0 / (1.0 + np.exp(-x))


def cla_gate(X, Wdw, bdw, Wpw, bpw) -> np.ndarray:
    """sigma(PWConv(DWConv3x3(X))) [B, H, W, C]."""
    return sigmoid(pwconv(dwconv3x3(X, Wdw, bdw), Wpw, bpw))


# --------------------------------------------------------------------------
# a7: LayerNorm (section 3.1 block order)
# --------------------------------------------------------------------------
def layernorm(x, eps: float = 1e-5, gamma=None, beta=None) -> np.ndarray:
    """LayerNorm over the channel axis with biased variance."""
    x = _f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * _f64(gamma)
    if beta is not None:
        y = y + _f64(beta)
    return y


# --------------------------------------------------------------------------
# ConvFFN and the full SST block (section 3.1 "模型架构设计": each block is
# LayerNorm -> RIB attention -> CLA -> ConvFFN with FFN expansion 1.25)
# --------------------------------------------------------------------------
def gelu(x) -> np.ndarray:
    """GELU(x) = x * Phi(x) with Phi the standard normal CDF (the erf form)."""
    x = _f64(x)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def conv_ffn(x, W1, b1, Wf, bf, W2, b2) -> np.ndarray:
    """ConvFFN of one block (write-up section 3.1, expansion 1.25): the hidden
    features h = GELU(x W1 + b1) ([.., hidden], hidden = 1.25 C) get a
    depthwise 3x3 conv added to them, h' = h + DWConv3x3(h) (zero padding 1,
    one filter and bias per hidden channel), and out = h' W2 + b2."""
    h = gelu(_f64(x) @ _f64(W1) + _f64(b1))
    h = h + dwconv3x3(h, Wf, bf)
    return h @ _f64(W2) + _f64(b2)


def sst_block(x, p: Dict, f: Dict, heads: int, R: int, L: int, M: int,
              threads: Optional[int] = None, eps: float = 1e-5) -> np.ndarray:
    """One SST block with pre-norm residuals: x <- x + Y(LN(x)) (RIB attention
    gated by the CLA), then x <- x + ConvFFN(LN(x))."""
    x = _f64(x)
    y, _ = rib_layer_forward(layernorm(x, eps), p, heads, R, L, M, threads=threads)
    x = x + y
    return x + conv_ffn(layernorm(x, eps), f["W1"], f["b1"], f["Wf"], f["bf"], f["W2"], f["b2"])


def sst_stack_forward(x, blocks: List[Dict], ffns: List[Dict], windows: Sequence[int], heads: int, R: int, L: int,
                      threads: Optional[int] = None, eps: float = 1e-5):
    """The SST body: one :func:`sst_block` per window of the cycle."""
    x = _f64(x)
    for p, f, M in zip(blocks, ffns, windows):
        x = sst_block(x, p, f, heads, R, L, M, threads=threads, eps=eps)
    return x


# --------------------------------------------------------------------------
# one layer: Y = softmax(S) V * sigma(G), windows reversed and cropped
# --------------------------------------------------------------------------
def rib_layer_forward(X, p: Dict, heads: int, R: int, L: int, M: int,
                      threads: Optional[int] = None, window_ids=None, mask_padding: bool = False):
    """Full layer forward. ``p`` holds Wq, Wk, Wv, Wh, bh, Wpq, Wpk, Wdw, bdw,
    Wpw, bpw. Returns (Y [B,H,W,C], aux dict with the attention output O,
    the gate, Qp, Kp and the per-row LSE)."""
    X = _f64(X)
    B, H, W, C = X.shape
    qp, kp = pos_features(M, L, p["Wh"], p["bh"], p["Wpq"], p["Wpk"], heads, R)
    Ofull, lse = rib_attention(X, p["Wq"], p["Wk"], p["Wv"], qp, kp, heads, M,
                               threads=threads, window_ids=window_ids, return_lse=True,
                               mask_padding=mask_padding)
    O = Ofull[:, :H, :W, :]
    gate = cla_gate(X, p["Wdw"], p["bdw"], p["Wpw"], p["bpw"])
    Y = O * gate
    return Y, {"O": O, "gate": gate, "Qp": qp, "Kp": kp, "lse": lse}


def rib_layer_forward_windows(X, p: Dict, heads: int, R: int, L: int, M: int,
                              window_ids: Iterable[int], threads: Optional[int] = None):
    """Layer output on the tokens of selected windows only.

    Returns a list of (b, y0, x0, Y_block) with Y_block the cropped output of
    window (b, y0/M, x0/M) at rows y0.. and columns x0.. of the image. The gate
    is computed on the block plus a one-pixel halo, so this is exact."""
    X = _f64(X)
    B, H, W, C = X.shape
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    ny, nx = Hp // M, Wp // M
    ids = list(window_ids)
    qp, kp = pos_features(M, L, p["Wh"], p["bh"], p["Wpq"], p["Wpk"], heads, R)
    Ofull = rib_attention(X, p["Wq"], p["Wk"], p["Wv"], qp, kp, heads, M,
                          threads=threads, window_ids=ids)
    res = []
    for w in ids:
        b, rem = divmod(w, ny * nx)
        wy, wx = divmod(rem, nx)
        y0, x0 = wy * M, wx * M
        y1, x1 = min(y0 + M, H), min(x0 + M, W)
        hy0, hx0, hy1, hx1 = max(y0 - 1, 0), max(x0 - 1, 0), min(y1 + 1, H), min(x1 + 1, W)
        # halo block, zero outside the image as in the full conv
        blk = np.zeros((1, y1 - y0 + 2, x1 - x0 + 2, C))
        blk[0, hy0 - y0 + 1:hy1 - y0 + 1, hx0 - x0 + 1:hx1 - x0 + 1] = X[b, hy0:hy1, hx0:hx1]
        dw = dwconv3x3(blk, p["Wdw"], p["bdw"])[:, 1:-1, 1:-1]
        g = sigmoid(pwconv(dw, p["Wpw"], p["bpw"]))[0]
        res.append((b, y0, x0, Ofull[b, y0:y1, x0:x1] * g))
    return res


def stack_forward(x, blocks: List[Dict], windows: Sequence[int], heads: int, R: int, L: int,
                  threads: Optional[int] = None, eps: float = 1e-5):
    """Section 3.1/3.2 block stack: x <- x + Y_k(LayerNorm(x)), window windows[k]."""
    x = _f64(x)
    for p, M in zip(blocks, windows):
        y, _ = rib_layer_forward(layernorm(x, eps), p, heads, R, L, M, threads=threads)
        x = x + y
    return x


# --------------------------------------------------------------------------
# a8: backward (analytic, fp64; pinned by finite differences)
# --------------------------------------------------------------------------
def attention_window_backward(Qc, Kc, V, Qp, Kp, dO, D: float, R: float):
    """Gradients of O = softmax(Qc Kc^T/sqrt(D) + Qp Kp^T/sqrt(R)) V for one
    window and head: returns dQc, dKc, dV, dQp, dKp.

    dV = P^T dO; dP = dO V^T; dS = P * (dP - rowsum(dP * P)); the score's two
    terms then give dQc = dS Kc / sqrt(D), dKc = dS^T Qc / sqrt(D),
    dQp = dS Kp / sqrt(R), dKp = dS^T Qp / sqrt(R) - the split of
    dQ = dS K at the content/position boundary of the concatenation."""
    Qc, Kc, V, Qp, Kp, dO = map(_f64, (Qc, Kc, V, Qp, Kp, dO))
    S = rib_scores(Qc, Kc, Qp, Kp, D, R)
    P = softmax_rows(S)
    dV = P.T @ dO
    dP = dO @ V.T
    dS = P * (dP - (dP * P).sum(axis=1, keepdims=True))
    a, b = 1.0 / math.sqrt(D), 1.0 / math.sqrt(R)
    return a * dS @ Kc, a * dS.T @ Qc, dV, b * dS @ Kp, b * dS.T @ Qp


def pos_features_backward(M: int, L: int, Wh, bh, Wpq, Wpk, heads: int, R: int, dQp, dKp):
    """Gradients of the coordinate MLP weights from dQp, dKp [heads, N, R]."""
    r = fourier_encode(window_coords(M), L)
    _, _, pre, h = coord_mlp(r, Wh, bh, Wpq, Wpk, heads, R)
    n = r.shape[0]
    gq = _f64(dQp).transpose(1, 0, 2).reshape(n, heads * R)
    gk = _f64(dKp).transpose(1, 0, 2).reshape(n, heads * R)
    dWpq = h.T @ gq
    dWpk = h.T @ gk
    dh = gq @ _f64(Wpq).T + gk @ _f64(Wpk).T
    dpre = dh * (pre > 0)
    return {"Wh": r.T @ dpre, "bh": dpre.sum(axis=0), "Wpq": dWpq, "Wpk": dWpk}


def qkv_project_backward(X, Wq, Wk, Wv, gq, gk, gv):
    """Backward of Qc, Kc, V = X Wq, X Wk, X Wv for token rows X [T, C] and
    the gradients gq, gk, gv [T, C] of the three outputs:
    dX = gq Wq^T + gk Wk^T + gv Wv^T, dW_j = X^T g_j. Returns (dX, dWq, dWk, dWv)."""
    X = _f64(X)
    gq, gk, gv = _f64(gq), _f64(gk), _f64(gv)
    Wq, Wk, Wv = _f64(Wq), _f64(Wk), _f64(Wv)
    dX = gq @ Wq.T + gk @ Wk.T + gv @ Wv.T
    return dX, X.T @ gq, X.T @ gk, X.T @ gv


def cla_gate_backward(X, Wdw, bdw, Wpw, dG):
    """Backward of the CLA gate sigma(G), G = DWConv3x3(X) Wpw + bpw (section
    2.3), from dG, the gradient of G ([B, H, W, C]):
      dD = dG Wpw^T, dWpw = D^T dG, dbpw = sum dG,
      dWdw[c, ky, kx] = sum X[p + (ky-1, kx-1), c] dD[p, c], dbdw = sum dD,
      dX = the transposed depthwise conv of dD (zero outside the image).
    Returns (dX, dWdw, dbdw, dWpw, dbpw)."""
    X, dG = _f64(X), _f64(dG)
    B, H, W, C = X.shape
    D = dwconv3x3(X, Wdw, bdw)
    Wpw, Wdw = _f64(Wpw), _f64(Wdw)
    dWpw = D.reshape(-1, C).T @ dG.reshape(-1, C)
    dbpw = dG.reshape(-1, C).sum(axis=0)
    dD = dG @ Wpw.T
    dbdw = dD.reshape(-1, C).sum(axis=0)
    Xpad = np.zeros((B, H + 2, W + 2, C))
    Xpad[:, 1:H + 1, 1:W + 1] = X
    dWdw = np.zeros((C, 3, 3))
    dXpad = np.zeros_like(Xpad)
    for ky in range(3):
        for kx in range(3):
            dWdw[:, ky, kx] = (Xpad[:, ky:ky + H, kx:kx + W, :] * dD).reshape(-1, C).sum(axis=0)
            dXpad[:, ky:ky + H, kx:kx + W, :] += dD * Wdw[:, ky, kx]
    return dXpad[:, 1:H + 1, 1:W + 1], dWdw, dbdw, dWpw, dbpw


def rib_layer_backward(X, p: Dict, dY, heads: int, R: int, L: int, M: int,
                       threads: Optional[int] = None):
    """Gradients of sum(Y * dY) for Y = rib_layer_forward(X, p)[0].

    Returns (grads dict with keys X, Wq, Wk, Wv, Wh, bh, Wpq, Wpk, Wdw, bdw,
    Wpw, bpw; per-window content grads dict with Qc, Kc, V [nW, N, C] and
    dQp, dKp [heads, N, R])."""
    X, dY = _f64(X), _f64(dY)
    B, H, W, C = X.shape
    dh = C // heads
    qp, kp = pos_features(M, L, p["Wh"], p["bh"], p["Wpq"], p["Wpk"], heads, R)
    Wq, Wk, Wv = _f64(p["Wq"]), _f64(p["Wk"]), _f64(p["Wv"])
    Xp = pad_to_windows(X, M)
    Hp, Wp = Xp.shape[1], Xp.shape[2]
    xw = window_partition(Xp, M)
    nwin = xw.shape[0]
    # forward pieces needed by the backward
    Ofull = rib_attention(X, Wq, Wk, Wv, qp, kp, heads, M, threads=threads)
    O = Ofull[:, :H, :W]
    dw = dwconv3x3(X, p["Wdw"], p["bdw"])
    gate = sigmoid(pwconv(dw, p["Wpw"], p["bpw"]))
    # Y = O * gate
    dO_img = np.zeros((B, Hp, Wp, C))
    dO_img[:, :H, :W] = dY * gate
    dgate = dY * O
    dG = dgate * gate * (1.0 - gate)
    # attention backward per window and head
    dOw = window_partition(dO_img, M)
    dQc = np.zeros((nwin, M * M, C))
    dKc = np.zeros((nwin, M * M, C))
    dV = np.zeros((nwin, M * M, C))
    dQp = np.zeros_like(qp)
    dKp = np.zeros_like(kp)

    def run(task):
        w, hd = task
        sl = slice(hd * dh, (hd + 1) * dh)
        qc, kc, v = xw[w] @ Wq[:, sl], xw[w] @ Wk[:, sl], xw[w] @ Wv[:, sl]
        return attention_window_backward(qc, kc, v, qp[hd], kp[hd], dOw[w][:, sl], dh, R)

    tasks = [(w, hd) for w in range(nwin) for hd in range(heads)]
    if threads and threads > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            results = list(ex.map(run, tasks))
    else:
        results = [run(t) for t in tasks]
    # the position gradients are summed over the windows in window order,
    # whatever the order in which the tasks ran
    for (w, hd), (gqc, gkc, gv, gqp, gkp) in zip(tasks, results):
        sl = slice(hd * dh, (hd + 1) * dh)
        dQc[w][:, sl], dKc[w][:, sl], dV[w][:, sl] = gqc, gkc, gv
        dQp[hd] += gqp
        dKp[hd] += gkp
    g = {}
    # projection backward on the window tokens (padded tokens have X = 0 and
    # are cropped from dX)
    dxw, g["Wq"], g["Wk"], g["Wv"] = qkv_project_backward(
        xw.reshape(-1, C), Wq, Wk, Wv, dQc.reshape(-1, C), dKc.reshape(-1, C), dV.reshape(-1, C))
    dX = window_reverse(dxw.reshape(nwin, M * M, C), M, B, Hp, Wp)[:, :H, :W]
    g.update(pos_features_backward(M, L, p["Wh"], p["bh"], p["Wpq"], p["Wpk"], heads, R, dQp, dKp))
    dXg, g["Wdw"], g["bdw"], g["Wpw"], g["bpw"] = cla_gate_backward(X, p["Wdw"], p["bdw"], p["Wpw"], dG)
    g["X"] = dX + dXg
    inner = {"Qc": dQc, "Kc": dKc, "V": dV, "Qp": dQp, "Kp": dKp}
    return g, inner
