"""ctypes binding of librib (the C-ABI declared in include/rib.h).

Argument marshalling only: tensors are passed as device pointers, the stream
is the caller's current torch stream, and every non-zero status raises
:class:`RibError` with the library's message. No step of the computation runs
here. There is no fallback: if librib.so is missing the import of the entry
points fails loudly.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librib.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "rib.h")

RIB_BF16, RIB_F32, RIB_F16 = 0, 1, 2
STATUS = {0: "RIB_OK", 1: "RIB_ERR_INVALID_ARG", 2: "RIB_ERR_UNSUPPORTED", 3: "RIB_ERR_ALIGNMENT",
          4: "RIB_ERR_CUDA", 5: "RIB_ERR_TIMEOUT"}


# kernel launches of one training step through these entry points: forward
# (projection 1, gate 1, attention 1), rib_attention_bwd_prep 1,
# rib_window_attention_bwd 4, rib_pos_encode_bwd 3, rib_qkv_project_bwd 4
# (weight re-layout, token GEMM, token reduction, partial sums), cla_gate_bwd
# 7 (weight re-layout, token GEMM, token reduction, transposed depthwise,
# partial sums of dWpw, depthwise reductions and their sums)
LAUNCHES = {"train_step": 22}


def v_dtype():
    """torch dtype of V and dO in the padded head-major layout (the operand
    type of the P.V product)."""
    import torch
    return torch.bfloat16


class RibError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class MlpDesc(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int), ("hidden", ctypes.c_int), ("heads", ctypes.c_int), ("R", ctypes.c_int),
                ("Wh", ctypes.c_void_p), ("bh", ctypes.c_void_p), ("Wpq", ctypes.c_void_p),
                ("Wpk", ctypes.c_void_p)]


class AttnDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int), ("C", ctypes.c_int),
                ("heads", ctypes.c_int), ("R", ctypes.c_int), ("window", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("mask_padding", ctypes.c_int), ("out_dtype", ctypes.c_int)]


_lib: Optional[ctypes.CDLL] = None
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

_SIGNATURES = {
    "rib_last_error": ([], ctypes.c_char_p),
    "rib_version": ([], _i),
    "rib_device_error": ([_vp], _i),
    "rib_head_pad": ([_i, _i], _i),
    "rib_pos_cache_bytes": ([ctypes.POINTER(MlpDesc), _i], _sz),
    "rib_pos_encode": ([ctypes.POINTER(MlpDesc), _i, _vp, _vp, _sz, _vp], _i),
    "rib_qkv_project": ([_vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp], _i),
    "cla_gate_workspace_size": ([_i, _i, _i, _i], _sz),
    "cla_gate": ([_vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _i),
    "cla_gate_static_scratch": ([_vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp], _i),
    "rib_window_attention": ([ctypes.POINTER(AttnDesc), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i),
    "rib_layernorm": ([_vp, _i, _vp, _i, _i, _i, _vp, _vp, _f, _vp], _i),
    "rib_attention_bwd_prep": ([ctypes.POINTER(AttnDesc), _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i),
    "rib_window_attention_workspace_size": ([ctypes.POINTER(AttnDesc)], _sz),
    "rib_window_attention_bwd_workspace_size": ([ctypes.POINTER(AttnDesc)], _sz),
    "rib_window_attention_bwd": ([ctypes.POINTER(AttnDesc)] + [_vp] * 14 + [_sz, _vp], _i),
    "rib_pos_encode_bwd_workspace_size": ([ctypes.POINTER(MlpDesc), _i], _sz),
    "rib_pos_encode_bwd": ([ctypes.POINTER(MlpDesc), _i] + [_vp] * 7 + [_sz, _vp], _i),
    "rib_f32_to_bf16": ([_vp, _vp, _sz, _vp], _i),
    "rib_bf16_to_f32": ([_vp, _vp, _sz, _vp], _i),
    "rib_qkv_project_bwd_workspace_size": ([_i, _i, _i, _i, _i], _sz),
    "rib_qkv_project_bwd": ([_vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _f] + [_vp] * 7 + [_vp, _sz, _vp], _i),
    "cla_gate_bwd_workspace_size": ([_i, _i, _i, _i], _sz),
    "cla_gate_bwd": ([_vp, _i, _i, _i, _i, _i] + [_vp] * 9 + [_vp, _sz, _vp], _i),
    "rib_selftest_wait_timeout": ([_i, _vp], _i),
    "rib_selftest_mma_rate": ([_i, _i, _i, _i, _vp, _vp, _vp], _i),
    "rib_conv_ffn_workspace_size": ([_i, _i, _i, _i], _sz),
    "rib_conv_ffn": ([_vp, _i, _vp, _i, _i, _i, _i, _i] + [_vp] * 7 + [_sz, _vp], _i),
}


def header_symbols() -> list:
    """Names of the functions include/rib.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = "\n".join(line for line in text.splitlines() if not line.lstrip().startswith("#"))
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)) - {"if", "sizeof"})


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load librib.so (building it first if the sources are newer)."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if path is None:
        from . import build as _build
        if not _build.up_to_date():
            _build.build()
    if not os.path.exists(p):
        raise ImportError(f"librib.so not found at {p}; run python -m windowed_attention_b200.build")
    lib = ctypes.CDLL(p)
    for name, (args, res) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != 0:
        raise RibError(status, _lib.rib_last_error().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("librib entry points take device tensors")
    if not t.is_contiguous():
        raise ValueError("librib entry points take contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _dtype_code(t) -> int:
    import torch
    return {torch.float32: RIB_F32, torch.float16: RIB_F16}.get(t.dtype, RIB_BF16)


# ----------------------------------------------------------------- entry points
def rib_version() -> int:
    return load().rib_version()


def rib_device_error(stream=None) -> None:
    load()
    _check(_lib.rib_device_error(_stream(stream)))


def rib_head_pad(C: int, heads: int) -> int:
    return load().rib_head_pad(C, heads)


def mlp_desc(L, hidden, heads, R, Wh, bh, Wpq, Wpk) -> MlpDesc:
    return MlpDesc(L, hidden, heads, R, _ptr(Wh), _ptr(bh), _ptr(Wpq), _ptr(Wpk))


def rib_pos_cache_bytes(desc: MlpDesc, window: int) -> int:
    return load().rib_pos_cache_bytes(ctypes.byref(desc), window)


def rib_pos_encode(desc: MlpDesc, window: int, qp_cache, kp_cache, stream=None) -> None:
    load()
    nbytes = min(qp_cache.numel() * qp_cache.element_size(), kp_cache.numel() * kp_cache.element_size())
    _check(_lib.rib_pos_encode(ctypes.byref(desc), window, _ptr(qp_cache), _ptr(kp_cache), nbytes,
                               _stream(stream)))


def rib_qkv_project(X, B, H, W, C, heads, window, Wq, Wk, Wv, q_scale, Qc, Kc, V, stream=None) -> None:
    load()
    _check(_lib.rib_qkv_project(_ptr(X), _dtype_code(X), B, H, W, C, heads, window, _ptr(Wq), _ptr(Wk), _ptr(Wv),
                                float(q_scale), _ptr(Qc), _ptr(Kc), _ptr(V), _stream(stream)))


def cla_gate_workspace_size(B, H, W, C) -> int:
    return load().cla_gate_workspace_size(B, H, W, C)


def cla_gate(X, B, H, W, C, Wdw, bdw, Wpw, bpw, sig_gate, workspace=None, stream=None) -> None:
    """sigmoid(PWConv(DWConv3x3(X))) into sig_gate; with a workspace, the
    depthwise output is left in it too (the backward's input)."""
    load()
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.cla_gate(_ptr(X), _dtype_code(X), B, H, W, C, _ptr(Wdw), _ptr(bdw), _ptr(Wpw), _ptr(bpw),
                         _ptr(sig_gate), _ptr(workspace), nbytes, _stream(stream)))


def cla_gate_static_scratch(X, B, H, W, C, Wdw, bdw, Wpw, bpw, sig_gate, stream=None) -> None:
    """cla_gate for callers that cannot allocate device memory: the depthwise
    intermediate lives in the library's fixed 16 MiB per-device array (see
    include/rib.h for the size limit and the sharing rules)."""
    load()
    _check(_lib.cla_gate_static_scratch(_ptr(X), _dtype_code(X), B, H, W, C, _ptr(Wdw), _ptr(bdw), _ptr(Wpw),
                                        _ptr(bpw), _ptr(sig_gate), _stream(stream)))


def attn_desc(B, H, W, C, heads, R, window, softmax_scale=1.0, mask_padding=False, out_f32=False,
              out_f16=False) -> AttnDesc:
    """Descriptor of one attention call; Y (and the residual) are bf16, or
    fp32 with out_f32, or fp16 with out_f16."""
    out = RIB_F32 if out_f32 else (RIB_F16 if out_f16 else RIB_BF16)
    return AttnDesc(B, H, W, C, heads, R, window, float(softmax_scale), 1 if mask_padding else 0, out)


def rib_window_attention(desc: AttnDesc, Qc, Kc, V, qp_cache, kp_cache, sig_gate, residual, Y, lse=None,
                         O_out=None, stream=None) -> None:
    load()
    _check(_lib.rib_window_attention(ctypes.byref(desc), _ptr(Qc), _ptr(Kc), _ptr(V), _ptr(qp_cache),
                                     _ptr(kp_cache), _ptr(sig_gate), _ptr(residual), _ptr(Y), _ptr(lse),
                                     _ptr(O_out), _stream(stream)))


def rib_attention_bwd_prep(desc: AttnDesc, dY, sig_gate, O, dO, Dsum, dG=None, stream=None) -> None:
    load()
    _check(_lib.rib_attention_bwd_prep(ctypes.byref(desc), _ptr(dY), _ptr(sig_gate), _ptr(O), _ptr(dO), _ptr(Dsum),
                                       _ptr(dG), _stream(stream)))


def rib_window_attention_workspace_size(desc: AttnDesc) -> int:
    return load().rib_window_attention_workspace_size(ctypes.byref(desc))


def rib_window_attention_bwd_workspace_size(desc: AttnDesc) -> int:
    return load().rib_window_attention_bwd_workspace_size(ctypes.byref(desc))


def rib_window_attention_bwd(desc: AttnDesc, Qc, Kc, V, qp_cache, kp_cache, lse, dO, Dsum, dQc, dKc, dV, dQp, dKp,
                             workspace, stream=None) -> None:
    load()
    _check(_lib.rib_window_attention_bwd(ctypes.byref(desc), _ptr(Qc), _ptr(Kc), _ptr(V), _ptr(qp_cache),
                                         _ptr(kp_cache), _ptr(lse), _ptr(dO), _ptr(Dsum), _ptr(dQc), _ptr(dKc),
                                         _ptr(dV), _ptr(dQp), _ptr(dKp), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)))


def rib_pos_encode_bwd_workspace_size(desc: MlpDesc, window: int) -> int:
    return load().rib_pos_encode_bwd_workspace_size(ctypes.byref(desc), window)


def rib_pos_encode_bwd(desc: MlpDesc, window, dqp_cache, dkp_cache, dWh, dbh, dWpq, dWpk, workspace,
                       stream=None) -> None:
    load()
    _check(_lib.rib_pos_encode_bwd(ctypes.byref(desc), window, _ptr(dqp_cache), _ptr(dkp_cache), _ptr(dWh),
                                   _ptr(dbh), _ptr(dWpq), _ptr(dWpk), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))


def rib_qkv_project_bwd_workspace_size(B, H, W, C, heads) -> int:
    return load().rib_qkv_project_bwd_workspace_size(B, H, W, C, heads)


def rib_qkv_project_bwd(X, B, H, W, C, heads, window, Wq, Wk, Wv, q_scale, dQc, dKc, dV, dX, dWq, dWk, dWv,
                        workspace=None, stream=None) -> None:
    """workspace: a device tensor of at least rib_qkv_project_bwd_workspace_size
    bytes (allocated here when None)."""
    load()
    if workspace is None:
        import torch
        workspace = torch.empty(rib_qkv_project_bwd_workspace_size(B, H, W, C, heads), dtype=torch.uint8,
                                device=X.device)
    _check(_lib.rib_qkv_project_bwd(_ptr(X), _dtype_code(X), B, H, W, C, heads, window, _ptr(Wq), _ptr(Wk), _ptr(Wv),
                                    float(q_scale), _ptr(dQc), _ptr(dKc), _ptr(dV), _ptr(dX), _ptr(dWq), _ptr(dWk),
                                    _ptr(dWv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)))


def cla_gate_bwd_workspace_size(B, H, W, C) -> int:
    return load().cla_gate_bwd_workspace_size(B, H, W, C)


def cla_gate_bwd(X, B, H, W, C, Wdw, Wpw, D, dG, dX, dWdw, dbdw, dWpw, dbpw, workspace, stream=None) -> None:
    load()
    _check(_lib.cla_gate_bwd(_ptr(X), _dtype_code(X), B, H, W, C, _ptr(Wdw), _ptr(Wpw), _ptr(D), _ptr(dG), _ptr(dX),
                             _ptr(dWdw), _ptr(dbdw), _ptr(dWpw), _ptr(dbpw), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)))


def rib_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Make one bounded device wait run out (see include/rib.h); the next
    rib_device_error() raises RibError with the timeout status."""
    load()
    _check(_lib.rib_selftest_wait_timeout(int(limit_us), _stream(stream)))


def rib_selftest_mma_rate(ctas_per_sm: int, issuers_per_cta: int, n: int, mmas: int, stream=None):
    """Issue rate of tcgen05.mma (see include/rib.h): every SM runs
    ctas_per_sm CTAs, each with issuers_per_cta threads issuing a chain of
    `mmas` M=128, K=16, width-n products. Returns a dict with the median
    clock64 cycles per MMA of one issuing thread (to its last issue and to
    the chain's completion), the SM's aggregate cycles per MMA, and
    `overlap`: over the SMs, the smallest ratio of the time all of an SM's
    CTAs ran together to the mean CTA's run time (1 when they ran side by
    side; the aggregate figure assumes they did)."""
    import torch
    load()
    dev = torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ctas = sms * ctas_per_sm
    cyc = torch.zeros(ctas * issuers_per_cta * 2, dtype=torch.int64, device=dev)
    spans = torch.zeros(ctas * 3, dtype=torch.int64, device=dev)
    _check(_lib.rib_selftest_mma_rate(int(ctas_per_sm), int(issuers_per_cta), int(n), int(mmas), _ptr(cyc),
                                      _ptr(spans), _stream(stream)))
    torch.cuda.synchronize(dev)
    rib_device_error()
    c = cyc.view(-1, 2).double().cpu()
    issue = float(c[:, 0].median()) / mmas
    done = float(c[:, 1].median()) / mmas
    sp = spans.view(-1, 3).cpu().tolist()
    by_sm = {}
    for smid, t0, t1 in sp:
        by_sm.setdefault(smid, []).append((t0, t1))
    overlap = 1.0
    for iv in by_sm.values():
        common = min(t1 for _, t1 in iv) - max(t0 for t0, _ in iv)
        mean = sum(t1 - t0 for t0, t1 in iv) / len(iv)
        overlap = min(overlap, max(0.0, common) / mean if mean > 0 else 0.0)
    return {"ctas_per_sm": ctas_per_sm, "issuers_per_cta": issuers_per_cta, "n": n, "mmas": mmas,
            "issue_cycles_per_mma": issue, "done_cycles_per_mma": done,
            "sm_cycles_per_mma": done / (ctas_per_sm * issuers_per_cta),
            "sms_used": len(by_sm), "max_ctas_on_an_sm": max(len(v) for v in by_sm.values()), "overlap": overlap}


def rib_layernorm(x, y, T, C, gamma=None, beta=None, eps=1e-5, stream=None) -> None:
    """y = LayerNorm(x) over C; x bf16, fp32 or fp16, y bf16 or fp16."""
    load()
    _check(_lib.rib_layernorm(_ptr(x), _dtype_code(x), _ptr(y), _dtype_code(y), T, C, _ptr(gamma), _ptr(beta),
                              float(eps), _stream(stream)))


def rib_f32_to_bf16(x, y, stream=None) -> None:
    load()
    _check(_lib.rib_f32_to_bf16(_ptr(x), _ptr(y), x.numel(), _stream(stream)))


def rib_bf16_to_f32(x, y, stream=None) -> None:
    load()
    _check(_lib.rib_bf16_to_f32(_ptr(x), _ptr(y), x.numel(), _stream(stream)))


def rib_conv_ffn_workspace_size(B, H, W, hidden) -> int:
    return load().rib_conv_ffn_workspace_size(B, H, W, hidden)


def rib_conv_ffn(xn, x, B, H, W, C, hidden, W1, b1, Wf, bf, W2, b2, workspace, stream=None) -> None:
    """x += ConvFFN(xn) (see include/rib.h): xn bf16 or fp16, x fp32 in place."""
    load()
    _check(_lib.rib_conv_ffn(_ptr(xn), _dtype_code(xn), _ptr(x), B, H, W, C, hidden, _ptr(W1), _ptr(b1), _ptr(Wf),
                             _ptr(bf), _ptr(W2), _ptr(b2), _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _stream(stream)))
