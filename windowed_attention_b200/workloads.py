"""Seeded synthetic workloads shared by the CUDA path's tests/bench and the oracle.

This module holds shapes and random numbers only: no step of the method's
arithmetic lives here. Both sides of every parity check draw their inputs from
:func:`make_inputs`, so the CUDA path and the oracle see bit-identical values.

Workloads (the shapes of the RIB/SST write-up, "Rank-Factorized Implicit
Neural Bias" summary, sections 2.1, 3.1, 3.2, 3.3 and 5.1):

* ``tiny``  - one layer, batch 1, 32x32 map, window 16, C=48, 3 heads, R=16,
  L=10, MLP hidden 64, fp32 inputs.
* ``lite``  - one layer, batch 1, 320x180 map (the lite model's LR input for a
  1280x720 output), C=48, 3 heads, R=16, L=10, hidden 64; windows 16/32/64.
* ``full``  - one layer, batch 1, 640x360 map (230,400 tokens), C=180,
  6 heads (dh=30), R=16, L=10, hidden 128, window 64.
* ``train`` - batch 16 patches of 96x96, C=180, 6 heads, R=16, window 96,
  forward + backward with an upstream gradient.
* ``stack`` - six blocks LN -> RIB attention -> CLA gate on the 640x360 map,
  windows cycled 16,32,64,16,32,64.
* ``sst``   - the same six blocks as full SST blocks (section 3.1): after the
  gated attention each block adds ConvFFN(LN(x)), FFN expansion 1.25
  (hidden 225 for C = 180).

Value recipe: feature maps ~ N(0,1); every weight and bias ~ N(0,1)/sqrt(fan_in)
with fan_in = 2+4L for the MLP trunk, hidden width for the rank projections,
C for Wq/Wk/Wv and the pointwise conv, 9 for the depthwise conv. Tensors that
the CUDA path consumes as bf16 (the feature map of bf16 workloads and the
tensor-core GEMM weights) are rounded to bf16 here, so both sides start from
the same representable values.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional, Tuple

import torch


@dataclass(frozen=True)
class LayerShape:
    """Shape of one windowed RIB attention + CLA gate layer."""

    B: int
    H: int            # image rows
    W: int            # image columns
    C: int            # channels (D in the write-up's model section)
    heads: int
    R: int            # rank of the positional features
    L: int            # Fourier frequency bands
    hidden: int       # coordinate-MLP hidden width
    window: int       # window side M (N = M*M tokens per window)
    dtype: str = "bf16"   # "bf16" or "f32": storage type of the feature map

    @property
    def dh(self) -> int:
        return self.C // self.heads

    @property
    def enc_dim(self) -> int:
        return 2 + 4 * self.L

    @property
    def Hp(self) -> int:
        return -(-self.H // self.window) * self.window

    @property
    def Wp(self) -> int:
        return -(-self.W // self.window) * self.window

    @property
    def n_windows(self) -> int:
        return self.B * (self.Hp // self.window) * (self.Wp // self.window)

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.W

    def attention_flops(self) -> float:
        """Algorithmic forward FLOPs of the attention: 2N^2(dh+R) + 2N^2 dh per
        window and head, unpadded head dims, padded windows counted in full."""
        n = self.window * self.window
        return float(self.n_windows * self.heads) * (2.0 * n * n * (self.dh + self.R) + 2.0 * n * n * self.dh)

    def attention_bwd_flops(self) -> float:
        """Algorithmic backward FLOPs: 2N^2(3(dh+R) + 2 dh) per window-head
        (recompute S, dP, dQ, dK over dh+R; dV over dh)."""
        n = self.window * self.window
        return float(self.n_windows * self.heads) * 2.0 * n * n * (3 * (self.dh + self.R) + 2 * self.dh)


@dataclass(frozen=True)
class Workload:
    name: str
    layer: LayerShape
    seed: int
    windows: Tuple[int, ...] = ()     # lite: separate runs; stack: one per block
    backward: bool = False
    blocks: int = 1
    ffn: bool = False                 # full SST blocks: a ConvFFN residual per block
    description: str = ""

    def layers(self) -> List[LayerShape]:
        if not self.windows:
            return [self.layer]
        return [replace(self.layer, window=w) for w in self.windows]


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload(
        "tiny", LayerShape(B=1, H=32, W=32, C=48, heads=3, R=16, L=10, hidden=64, window=16, dtype="f32"),
        seed=0, description="batch 1, 32x32, window 16, C=48, 3 heads, R=16, L=10, hidden 64, fp32"),
    "lite": Workload(
        "lite", LayerShape(B=1, H=180, W=320, C=48, heads=3, R=16, L=10, hidden=64, window=16),
        seed=1, windows=(16, 32, 64),
        description="batch 1, 320x180 LR map, C=48, 3 heads, R=16, L=10, hidden 64, windows 16/32/64, bf16"),
    "full": Workload(
        "full", LayerShape(B=1, H=360, W=640, C=180, heads=6, R=16, L=10, hidden=128, window=64),
        seed=2, description="batch 1, 640x360 LR map (230,400 tokens), C=180, 6 heads (dh=30), R=16, "
                            "L=10, hidden 128, window 64, bf16"),
    "train": Workload(
        "train", LayerShape(B=16, H=96, W=96, C=180, heads=6, R=16, L=10, hidden=128, window=96),
        seed=3, backward=True,
        description="batch 16 patches 96x96, C=180, 6 heads, R=16, window 96, bf16, forward + backward"),
    "stack": Workload(
        "stack", LayerShape(B=1, H=360, W=640, C=180, heads=6, R=16, L=10, hidden=128, window=16),
        seed=4, windows=(16, 32, 64, 16, 32, 64), blocks=6,
        description="six blocks LN -> RIB attention -> CLA gate, 640x360, C=180, windows 16,32,64,16,32,64"),
    "sst": Workload(
        "sst", LayerShape(B=1, H=360, W=640, C=180, heads=6, R=16, L=10, hidden=128, window=16),
        seed=5, windows=(16, 32, 64, 16, 32, 64), blocks=6, ffn=True,
        description="six full SST blocks (LN -> RIB attention -> CLA gate, LN -> ConvFFN x1.25), 640x360, "
                    "C=180, windows 16,32,64,16,32,64"),
}


def ffn_hidden(C: int) -> int:
    """ConvFFN hidden width: FFN expansion 1.25 (write-up section 3.1)."""
    return int(round(1.25 * C))


def bf16_round(t: torch.Tensor) -> torch.Tensor:
    """Round float32 values to the nearest bf16 value (returned as float32)."""
    return t.to(torch.bfloat16).to(torch.float32)


# Order in which the generator draws the tensors of one layer.
DRAW_ORDER = ("X", "Wq", "Wk", "Wv", "Wh", "bh", "Wpq", "Wpk", "Wdw", "bdw", "Wpw", "bpw")
# Tensors the CUDA path consumes as bf16 tensor-core operands.
BF16_WEIGHTS = ("Wq", "Wk", "Wv", "Wpw")


def _layer_params(s: LayerShape, g: torch.Generator, with_x: bool) -> Dict[str, torch.Tensor]:
    def randn(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32)

    out: Dict[str, torch.Tensor] = {}
    e, fh, hr, c = s.enc_dim, s.hidden, s.heads * s.R, s.C
    shapes = {
        "X": ((s.B, s.H, s.W, c), 1.0),
        "Wq": ((c, c), c), "Wk": ((c, c), c), "Wv": ((c, c), c),
        "Wh": ((e, fh), e), "bh": ((fh,), e),
        "Wpq": ((fh, hr), fh), "Wpk": ((fh, hr), fh),
        "Wdw": ((c, 3, 3), 9), "bdw": ((c,), 9),
        "Wpw": ((c, c), c), "bpw": ((c,), c),
    }
    for name in DRAW_ORDER:
        if name == "X" and not with_x:
            continue
        shape, fan = shapes[name]
        t = randn(*shape)
        if name != "X":
            t = t / float(fan) ** 0.5
        out[name] = t
    if s.dtype == "bf16":
        if "X" in out:
            out["X"] = bf16_round(out["X"])
        for name in BF16_WEIGHTS:
            out[name] = bf16_round(out[name])
    return out


# Order in which the generator draws one block's ConvFFN tensors (after every
# block's attention and gate tensors): W1 [C][hid], b1 [hid], Wf [hid][3][3],
# bf [hid], W2 [hid][C], b2 [C].
FFN_DRAW_ORDER = ("W1", "b1", "Wf", "bf", "W2", "b2")


def _ffn_params(s: LayerShape, g: torch.Generator) -> Dict[str, torch.Tensor]:
    c, hid = s.C, ffn_hidden(s.C)
    shapes = {"W1": ((c, hid), c), "b1": ((hid,), c), "Wf": ((hid, 3, 3), 9), "bf": ((hid,), 9),
              "W2": ((hid, c), hid), "b2": ((c,), hid)}
    out = {}
    for name in FFN_DRAW_ORDER:
        shape, fan = shapes[name]
        out[name] = torch.randn(*shape, generator=g, dtype=torch.float32) / float(fan) ** 0.5
    if s.dtype == "bf16":
        for name in ("W1", "W2"):
            out[name] = bf16_round(out[name])
    return out


def make_inputs(workload: str | Workload, layer: Optional[LayerShape] = None,
                with_grad: Optional[bool] = None) -> Dict[str, object]:
    """Draw the seeded inputs of a workload on the CPU (float32 tensors).

    Returns ``{"X": ..., "Wq": ..., ..., "dY": (if backward), "blocks": [...]}``.
    For the multi-block stack, ``blocks`` holds one parameter dict per block
    (drawn after X, in block order) and the top-level weights are block 0's.
    ``layer`` overrides the shape (used to draw small cases of a workload).
    """
    wl = WORKLOADS[workload] if isinstance(workload, str) else workload
    s = layer if layer is not None else wl.layer
    g = torch.Generator().manual_seed(wl.seed)
    first = _layer_params(s, g, with_x=True)
    out: Dict[str, object] = dict(first)
    blocks = [{k: v for k, v in first.items() if k != "X"}]
    for _ in range(1, wl.blocks):
        blocks.append(_layer_params(s, g, with_x=False))
    out["blocks"] = blocks
    if wl.ffn:
        out["ffns"] = [_ffn_params(s, g) for _ in range(wl.blocks)]
    grad = wl.backward if with_grad is None else with_grad
    if grad:
        dy = torch.randn(s.B, s.H, s.W, s.C, generator=g, dtype=torch.float32)
        out["dY"] = bf16_round(dy) if s.dtype == "bf16" else dy
    out["shape"] = s
    return out
