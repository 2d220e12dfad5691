"""Windowed RIB attention with CLA gate on B200 (sm_100a).

The computation lives in librib.so (hand-written CUDA behind the C-ABI of
include/rib.h); this package is its Python binding plus seeded synthetic
workloads. Importing the package does not load the library; the first entry
point call (or :func:`load`) does, and fails loudly if it is missing.
"""
from ._lib import (  # noqa: F401
    AttnDesc, MlpDesc, RibError, attn_desc, cla_gate, cla_gate_static_scratch, cla_gate_workspace_size, header_symbols, load, mlp_desc,
    rib_device_error, rib_f32_to_bf16, rib_bf16_to_f32, rib_head_pad, rib_layernorm, rib_pos_cache_bytes, rib_pos_encode,
    rib_qkv_project, rib_version, rib_window_attention, rib_attention_bwd_prep, rib_window_attention_bwd,
    rib_window_attention_workspace_size, rib_window_attention_bwd_workspace_size, rib_pos_encode_bwd, rib_pos_encode_bwd_workspace_size,
    rib_qkv_project_bwd, cla_gate_bwd, cla_gate_bwd_workspace_size, rib_qkv_project_bwd_workspace_size,
    rib_selftest_wait_timeout, rib_selftest_mma_rate, v_dtype,
    rib_conv_ffn, rib_conv_ffn_workspace_size,
)
from .workloads import WORKLOADS, LayerShape, Workload, make_inputs  # noqa: F401

__version__ = "0.1.0"
