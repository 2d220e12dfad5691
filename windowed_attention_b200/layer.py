"""One windowed RIB attention + CLA gate layer driven through the C-ABI.

PyTorch only provides device memory and the stream here; every step runs in
librib's kernels, in this order (RIB/SST write-up sections 2.2-2.3):

    rib_pos_encode       once per window size (cached, section 5.2)
    rib_qkv_project      Qc (x 1/sqrt(dh)), Kc and V (bf16, ones columns)
                         in the window-padded, head-padded layout
    cla_gate             sigmoid(PWConv(DWConv3x3(X)))
    rib_window_attention fused scores/softmax/PV, gate multiply, window reverse

For the block stack (section 3.1/3.2) a block is x <- x + layer(LN(x)) with
the residual add fused into the attention store; the residual stream x is
kept in fp32 (LayerNorm reads it in fp32, the attention store adds into it in
fp32), so six blocks of bf16 rounding do not accumulate in x.
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import torch

from . import _lib
from .workloads import LayerShape


class RibLayer:
    """Device-resident weights, caches and activation buffers of one layer."""

    def __init__(self, shape: LayerShape, params: Dict[str, torch.Tensor], device="cuda",
                 windows: Optional[tuple] = None):
        _lib.load()
        self.s = shape
        self.device = torch.device(device)
        dev = self.device
        s = shape
        self.dh = s.C // s.heads
        self.DP = _lib.rib_head_pad(s.C, s.heads)
        bf = torch.bfloat16
        self.Wq = params["Wq"].to(dev, bf).contiguous()
        self.Wk = params["Wk"].to(dev, bf).contiguous()
        self.Wv = params["Wv"].to(dev, bf).contiguous()
        self.Wpw = params["Wpw"].to(dev, bf).contiguous()
        f32 = torch.float32
        self.Wh = params["Wh"].to(dev, f32).contiguous()
        self.bh = params["bh"].to(dev, f32).contiguous()
        self.Wpq = params["Wpq"].to(dev, f32).contiguous()
        self.Wpk = params["Wpk"].to(dev, f32).contiguous()
        self.Wdw = params["Wdw"].to(dev, f32).contiguous()
        self.bdw = params["bdw"].to(dev, f32).contiguous()
        self.bpw = params["bpw"].to(dev, f32).contiguous()
        self.mlp = _lib.mlp_desc(s.L, s.hidden, s.heads, s.R, self.Wh, self.bh, self.Wpq, self.Wpk)
        self.cache: Dict[int, tuple] = {}
        self.windows = tuple(windows or (s.window,))
        for M in self.windows:
            self.pos_cache(M)
        T = s.B * s.H * s.W
        Tp = max(self.padded_tokens(M) for M in self.windows)
        self.capacity = Tp
        self.Qc = torch.empty(Tp * s.heads * self.DP, dtype=bf, device=dev)
        self.Kc = torch.empty_like(self.Qc)
        self.V = torch.empty(Tp * s.heads * 32, dtype=_lib.v_dtype(), device=dev)
        self.gate = torch.empty(T * s.C, dtype=bf, device=dev)
        self.ws = torch.empty(_lib.cla_gate_workspace_size(s.B, s.H, s.W, s.C) // 2, dtype=bf, device=dev)
        self.Y = torch.empty(s.B, s.H, s.W, s.C, dtype=bf, device=dev)
        self.xbf = torch.empty(s.B, s.H, s.W, s.C, dtype=bf, device=dev) if s.dtype == "f32" else None

    def padded_tokens(self, M: int) -> int:
        s = self.s
        return s.B * (-(-s.H // M) * M) * (-(-s.W // M) * M)

    def pos_cache(self, M: int):
        if M not in self.cache:
            n = self.s.heads * M * M * self.s.R
            qp = torch.empty(n, dtype=torch.bfloat16, device=self.device)
            kp = torch.empty_like(qp)
            _lib.rib_pos_encode(self.mlp, M, qp, kp)
            self.cache[M] = (qp, kp)
        return self.cache[M]

    def forward(self, X: torch.Tensor, window: Optional[int] = None, residual: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                O_out: Optional[torch.Tensor] = None, gate: bool = True, mask_padding: bool = False,
                out_f32: bool = False, keep_depthwise: bool = False) -> torch.Tensor:
        """Y = attention(X) * sigmoid(gate(X)) (+ residual). keep_depthwise
        leaves the gate's depthwise output in self.ws (the backward reads it)."""
        s = self.s
        M = window or s.window
        if self.padded_tokens(M) > self.capacity:
            raise ValueError(f"window {M} pads the map beyond the buffers this layer was sized for")
        if X.dtype == torch.float32:
            _lib.rib_f32_to_bf16(X, self.xbf)
            X = self.xbf
        out_f16 = X.dtype == torch.float16 and not out_f32     # the fp16 path: fp16 in, fp16 Y out
        if out_f16 and out is None:
            if getattr(self, "Y16", None) is None:
                self.Y16 = torch.empty(s.B, s.H, s.W, s.C, dtype=torch.float16, device=self.device)
            out = self.Y16
        _lib.rib_qkv_project(X, s.B, s.H, s.W, s.C, s.heads, M, self.Wq, self.Wk, self.Wv, 1.0 / math.sqrt(self.dh),
                             self.Qc, self.Kc, self.V)
        if gate:
            _lib.cla_gate(X, s.B, s.H, s.W, s.C, self.Wdw, self.bdw, self.Wpw, self.bpw, self.gate,
                          self.ws if keep_depthwise else None)
        qp, kp = self.pos_cache(M)
        Y = self.Y if out is None else out
        desc = _lib.attn_desc(s.B, s.H, s.W, s.C, s.heads, s.R, M, 1.0, mask_padding=mask_padding, out_f32=out_f32,
                              out_f16=out_f16)
        _lib.rib_window_attention(desc, self.Qc, self.Kc, self.V, qp, kp, self.gate if gate else None, residual, Y,
                                  lse, O_out)
        return Y


    def backward(self, X: torch.Tensor, dY: torch.Tensor, window: Optional[int] = None) -> Dict[str, torch.Tensor]:
        """Forward (saving lse and the ungated output), then the backward chain
        through librib: rib_attention_bwd_prep -> rib_window_attention_bwd ->
        rib_pos_encode_bwd -> rib_qkv_project_bwd -> cla_gate_bwd. Returns the
        device gradients (see include/rib.h), dX and every weight's included."""
        s = self.s
        M = window or s.window
        dev = self.device
        Hp, Wp = -(-s.H // M) * M, -(-s.W // M) * M
        lse = torch.empty(s.B * s.heads * Hp * Wp, dtype=torch.float32, device=dev)
        O = torch.empty(s.B * s.H * s.W * s.heads * self.DP, dtype=torch.bfloat16, device=dev)
        Y = self.forward(X, window=M, lse=lse, O_out=O, keep_depthwise=True)
        desc = _lib.attn_desc(s.B, s.H, s.W, s.C, s.heads, s.R, M, 1.0)
        Tp = s.B * Hp * Wp
        g = {"Y": Y, "lse": lse, "O": O}
        g["dO"] = torch.empty(Tp * s.heads * 32, dtype=_lib.v_dtype(), device=dev)
        g["Dsum"] = torch.empty(s.B * s.heads * Hp * Wp, dtype=torch.float32, device=dev)
        g["dG"] = torch.empty(s.B, s.H, s.W, s.C, dtype=torch.bfloat16, device=dev)
        _lib.rib_attention_bwd_prep(desc, dY, self.gate, O, g["dO"], g["Dsum"], g["dG"])
        for k in ("dQc", "dKc", "dV"):
            g[k] = torch.empty(Tp * s.heads * 32, dtype=torch.float32, device=dev)
        for k in ("dQp", "dKp"):
            g[k] = torch.empty(s.heads * M * M * s.R, dtype=torch.float32, device=dev)
        g["ws"] = torch.empty(_lib.rib_window_attention_bwd_workspace_size(desc) // 4, dtype=torch.float32, device=dev)
        qp, kp = self.pos_cache(M)
        _lib.rib_window_attention_bwd(desc, self.Qc, self.Kc, self.V, qp, kp, lse, g["dO"], g["Dsum"], g["dQc"],
                                      g["dKc"], g["dV"], g["dQp"], g["dKp"], g["ws"])
        e = s.enc_dim
        g["dWh"] = torch.empty(e, s.hidden, dtype=torch.float32, device=dev)
        g["dbh"] = torch.empty(s.hidden, dtype=torch.float32, device=dev)
        g["dWpq"] = torch.empty(s.hidden, s.heads * s.R, dtype=torch.float32, device=dev)
        g["dWpk"] = torch.empty_like(g["dWpq"])
        pws = torch.empty(_lib.rib_pos_encode_bwd_workspace_size(self.mlp, M) // 4, dtype=torch.float32, device=dev)
        _lib.rib_pos_encode_bwd(self.mlp, M, g["dQp"], g["dKp"], g["dWh"], g["dbh"], g["dWpq"], g["dWpk"], pws)
        # content projections and CLA gate: dX and their weight gradients (from
        # the bf16 map the forward consumed)
        Xb = self.xbf if X.dtype == torch.float32 else X
        C = s.C
        g["dX"] = torch.empty(s.B, s.H, s.W, C, dtype=torch.float32, device=dev)
        for k in ("dWq", "dWk", "dWv", "dWpw"):
            g[k] = torch.empty(C, C, dtype=torch.float32, device=dev)
        g["dWdw"] = torch.empty(C, 3, 3, dtype=torch.float32, device=dev)
        g["dbdw"] = torch.empty(C, dtype=torch.float32, device=dev)
        g["dbpw"] = torch.empty(C, dtype=torch.float32, device=dev)
        pws = torch.empty(_lib.rib_qkv_project_bwd_workspace_size(s.B, s.H, s.W, C, s.heads), dtype=torch.uint8,
                          device=dev)
        _lib.rib_qkv_project_bwd(Xb, s.B, s.H, s.W, C, s.heads, M, self.Wq, self.Wk, self.Wv, 1 / math.sqrt(self.dh),
                                 g["dQc"], g["dKc"], g["dV"], g["dX"], g["dWq"], g["dWk"], g["dWv"], pws)
        gws = torch.empty(_lib.cla_gate_bwd_workspace_size(s.B, s.H, s.W, C) // 4, dtype=torch.float32, device=dev)
        _lib.cla_gate_bwd(Xb, s.B, s.H, s.W, C, self.Wdw, self.Wpw, self.ws, g["dG"], g["dX"], g["dWdw"], g["dbdw"],
                          g["dWpw"], g["dbpw"], gws)
        return g


class ConvFFN:
    """Device weights of one block's ConvFFN (section 3.1, expansion 1.25):
    x += (h + DWConv3x3(h)) W2 + b2 with h = GELU(LN(x) W1 + b1)."""

    def __init__(self, shape: LayerShape, f: Dict[str, torch.Tensor], device="cuda"):
        dev = torch.device(device)
        self.hidden = f["W1"].shape[1]
        self.W1 = f["W1"].to(dev, torch.bfloat16).contiguous()
        self.W2 = f["W2"].to(dev, torch.bfloat16).contiguous()
        self.b1, self.Wf, self.bf, self.b2 = (f[k].to(dev, torch.float32).contiguous() for k in ("b1", "Wf", "bf", "b2"))
        n = _lib.rib_conv_ffn_workspace_size(shape.B, shape.H, shape.W, self.hidden)
        self.ws = torch.empty(n // 2, dtype=torch.float16, device=dev)

    def __call__(self, xn: torch.Tensor, x: torch.Tensor, s: LayerShape) -> None:
        _lib.rib_conv_ffn(xn, x, s.B, s.H, s.W, s.C, self.hidden, self.W1, self.b1, self.Wf, self.bf, self.W2,
                          self.b2, self.ws)


class RibStack:
    """Block stack x <- x + layer_k(LN(x)) with cycled windows (sections 3.1,
    3.2); with ``ffns`` each block is the full SST block, which then adds
    x <- x + ConvFFN_k(LN(x)).

    The residual stream ``x`` is fp32 on the device; each LayerNorm output
    (the input of the attention layer and of the ConvFFN) is fp16: the
    normalised values are small, and fp16's finer steps keep the rounding of
    every block's input 8 times below bf16's, which would otherwise dominate
    the error of a deep stack (the pages train in fp16 mixed precision)."""

    def __init__(self, shape: LayerShape, blocks, windows, device="cuda", ffns=None):
        self.s = shape
        self.windows = tuple(windows)
        self.layers = [RibLayer(shape, p, device, windows=(w,)) for p, w in zip(blocks, windows)]
        self.ffns = [ConvFFN(shape, f, device) for f in ffns] if ffns else None
        dev = torch.device(device)
        self.ln = torch.empty(shape.B, shape.H, shape.W, shape.C, dtype=torch.float16, device=dev)
        self.x = torch.empty(shape.B, shape.H, shape.W, shape.C, dtype=torch.float32, device=dev)

    def load(self, x: torch.Tensor) -> None:
        """Start the residual stream from x (bf16 or fp32, [B, H, W, C])."""
        if x.data_ptr() == self.x.data_ptr():
            return
        if x.dtype == torch.bfloat16:
            _lib.rib_bf16_to_f32(x, self.x)
        else:
            self.x.copy_(x)

    def block(self, k: int, ffn: bool = True) -> torch.Tensor:
        """Block k in place on the residual stream: x <- x + layer_k(LN(x)),
        then (full SST blocks, unless ffn is False) x <- x + ConvFFN_k(LN(x))."""
        s = self.s
        _lib.rib_layernorm(self.x, self.ln, s.B * s.H * s.W, s.C, None, None, 1e-5)
        self.layers[k].forward(self.ln, window=self.windows[k], residual=self.x, out=self.x, out_f32=True)
        if self.ffns and ffn:
            self.ffn(k)
        return self.x

    def ffn(self, k: int) -> torch.Tensor:
        """The ConvFFN half of block k: x <- x + ConvFFN_k(LN(x))."""
        s = self.s
        _lib.rib_layernorm(self.x, self.ln, s.B * s.H * s.W, s.C, None, None, 1e-5)
        self.ffns[k](self.ln, self.x, s)
        return self.x

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        self.load(x)
        for k in range(len(self.layers)):
            self.block(k)
        return self.x
