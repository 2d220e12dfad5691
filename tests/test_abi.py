"""The C-ABI library builds, loads without a GPU, exports every symbol that
include/rib.h declares, and rejects bad arguments on the host before any
launch (no compute calls here)."""
import ctypes
import os

import pytest

import windowed_attention_b200 as rib
from windowed_attention_b200 import _lib


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_header_symbols_exported(lib):
    names = _lib.header_symbols()
    assert {"rib_window_attention", "rib_pos_encode", "cla_gate", "rib_qkv_project", "rib_layernorm"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib._SIGNATURES, f"binding lacks {n}"


def test_version_and_sizes(lib):
    assert rib.rib_version() >= 100
    assert rib.rib_head_pad(180, 6) == 32
    assert rib.rib_head_pad(48, 3) == 16
    assert rib.rib_head_pad(180, 7) == -1
    assert rib.cla_gate_workspace_size(1, 360, 640, 180) == 360 * 640 * 180 * 2
    d = _lib.MlpDesc(10, 128, 6, 16, 0, 0, 0, 0)
    assert rib.rib_pos_cache_bytes(d, 64) == 6 * 64 * 64 * 16 * 2
    a = _lib.attn_desc(1, 360, 640, 180, 6, 16, 64, 1.0)
    assert rib.rib_window_attention_workspace_size(a) == 0          # the forward keeps S and P on chip
    # per-window dQp/dKp partials, then (dh = 30: two spare columns) the folded
    # query operands, bf16 [640 x 384 padded tokens][6 heads][32 + 16]
    assert rib.rib_window_attention_bwd_workspace_size(a) == 2 * 60 * 6 * 64 * 64 * 16 * 4 + 640 * 384 * 6 * 48 * 2
    tiny = _lib.attn_desc(1, 32, 32, 48, 3, 16, 16, 1.0)     # dh = DP = 16: partials only
    assert rib.rib_window_attention_bwd_workspace_size(tiny) == 2 * 4 * 3 * 16 * 16 * 16 * 4


def _attn(lib, desc, ptr=256):
    return lib.rib_window_attention(ctypes.byref(desc), ptr, ptr, ptr, ptr, ptr, None, None, ptr, None, None, None)


def test_attention_argument_checks(lib):
    ok = _lib.AttnDesc(1, 360, 640, 180, 6, 16, 64, 1.0)
    assert lib.rib_window_attention(None, 256, 256, 256, 256, 256, None, None, 256, None, None, None) == 1
    bad_window = _lib.AttnDesc(1, 360, 640, 180, 6, 16, 24, 1.0)
    assert _attn(lib, bad_window) == 2
    assert b"window" in lib.rib_last_error()
    bad_rank = _lib.AttnDesc(1, 360, 640, 180, 6, 32, 64, 1.0)
    assert _attn(lib, bad_rank) == 2
    big_head = _lib.AttnDesc(1, 32, 32, 128, 4, 16, 16, 1.0)   # dh = 32
    assert _attn(lib, big_head) == 2
    bad_heads = _lib.AttnDesc(1, 32, 32, 48, 5, 16, 16, 1.0)
    assert _attn(lib, bad_heads) == 1
    assert _attn(lib, _lib.AttnDesc(1, 32, 32, 48, 3, 16, 16, 0.0)) == 1
    assert _attn(lib, ok, ptr=258) == 3        # misaligned pointer


def test_projection_and_gate_argument_checks(lib):
    assert lib.rib_qkv_project(None, 0, 1, 8, 8, 48, 3, 16, 256, 256, 256, 1.0, 256, 256, 256, None) == 1
    assert lib.rib_qkv_project(256, 0, 1, 8, 8, 50, 5, 16, 256, 256, 256, 1.0, 256, 256, 256, None) == 2   # dh odd
    assert lib.rib_qkv_project(256, 0, 1, 8, 8, 64, 2, 16, 256, 256, 256, 1.0, 256, 256, 256, None) == 2   # dh 32
    assert lib.rib_qkv_project(256, 1, 1, 8, 8, 48, 3, 16, 256, 256, 256, 1.0, 256, 256, 256, None) == 2   # f32 X
    assert lib.rib_qkv_project(256, 0, 1, 8, 8, 48, 3, 0, 256, 256, 256, 1.0, 256, 256, 256, None) == 1    # window
    assert lib.cla_gate(256, 0, 1, 8, 8, 46, 256, 256, 256, 256, 256, 256, 1 << 20, None) == 2          # C % 4
    assert lib.cla_gate(256, 0, 1, 8, 8, 48, 256, 256, 256, 256, 256, 256, 16, None) == 1               # workspace
    assert lib.rib_layernorm(256, 0, 256, 0, 10, 48, None, None, 0.0, None) == 1
    d = _lib.MlpDesc(10, 64, 3, 8, 256, 256, 256, 256)
    assert lib.rib_pos_encode(ctypes.byref(d), 16, 256, 256, 1 << 20, None) == 2


def test_window_tiling_rule():
    # windows the kernel tiles into 128-token rectangles: multiples of 16 up to 256
    from windowed_attention_b200.workloads import WORKLOADS
    sizes = {l.window for wl in WORKLOADS.values() for l in wl.layers()}
    assert sizes <= {16, 32, 64, 96}


def test_projection_and_gate_backward_argument_checks(lib):
    # X, xdtype, B, H, W, C, heads, window, Wq, Wk, Wv, q_scale, dQc, dKc, dV, dX, dWq, dWk, dWv, ws, ws_bytes,
    # stream
    a = [256, 0, 1, 8, 8, 48, 3, 16, 256, 256, 256, 1.0, 256, 256, 256, 256, 256, 256, 256, 256, 1 << 20, None]
    assert lib.rib_qkv_project_bwd(None, *a[1:]) == 1
    assert lib.rib_qkv_project_bwd(*a[:5], 50, 5, *a[7:]) == 2          # dh odd
    f32 = list(a)
    f32[1] = 1
    assert lib.rib_qkv_project_bwd(*f32) == 2                            # f32 X
    mis = list(a)
    mis[12] = 264
    assert lib.rib_qkv_project_bwd(*mis) == 3                            # dQc 8-byte aligned only
    small = list(a)
    small[20] = 16
    assert lib.rib_qkv_project_bwd(*small) == 1                          # workspace
    nows = list(a)
    nows[19] = None
    assert lib.rib_qkv_project_bwd(*nows) == 1                           # no workspace
    # re-laid weights (3 jobs x 2 two-head atoms x 64 rows x 128 B) + 144 partial [C][C] sums
    assert rib.rib_qkv_project_bwd_workspace_size(1, 8, 8, 48, 3) == 3 * 2 * 64 * 128 + 144 * 48 * 48 * 4
    # X, xdtype, B, H, W, C, Wdw, Wpw, D, dG, dX, dWdw, dbdw, dWpw, dbpw, ws, ws_bytes, stream
    b = [256, 0, 1, 8, 8, 48] + [256] * 9 + [256, 1 << 22, None]
    assert lib.cla_gate_bwd(*b[:5], 46, *b[6:]) == 2                    # C % 4
    small = list(b)
    small[16] = 16
    assert lib.cla_gate_bwd(*small) == 1                                 # workspace
    mis = list(b)
    mis[9] = 264
    assert lib.cla_gate_bwd(*mis) == 3                                   # dG 8-byte aligned only
    # dD fp32 + re-laid Wpw (one 64-channel atom x 64 rows x 128 B) + 144 partial [C][C]
    # sums + depthwise partials [C][11] per block of map rows (8 rows: one row per block)
    assert rib.cla_gate_bwd_workspace_size(1, 8, 8, 48) == 8 * 8 * 48 * 4 + 64 * 128 + 144 * 48 * 48 * 4 + 8 * 48 * 11 * 4


def test_key_padding_mask_is_forward_only(lib):
    d = _lib.attn_desc(1, 40, 72, 48, 3, 16, 16, 1.0, mask_padding=True)
    # rib_attention_bwd_prep(desc, dY, sig_gate, O, dO, Dsum, dG, stream)
    assert lib.rib_attention_bwd_prep(ctypes.byref(d), 256, 256, 256, 256, 256, 256, None) == 2
    assert b"forward only" in lib.rib_last_error()


def test_selftest_wait_limit_checked(lib):
    assert lib.rib_selftest_wait_timeout(0, None) == 1
    assert lib.rib_selftest_wait_timeout(2_000_000, None) == 1


def test_selftest_mma_rate_arguments_checked(lib):
    buf = ctypes.c_void_p(256)   # never dereferenced: every call below is refused before any launch
    for args in ((0, 1, 64, 16), (5, 1, 64, 16), (1, 0, 64, 16), (1, 5, 64, 16), (1, 1, 8, 16), (1, 1, 72, 16),
                 (1, 1, 272, 16), (1, 1, 64, 0), (1, 1, 64, 70000),
                 (4, 2, 128, 16),    # 2 x 128 columns > the 128 a CTA gets at four per SM
                 (2, 4, 128, 16)):   # 4 x 128 > 256
        assert lib.rib_selftest_mma_rate(*args, buf, None, None) == 1, args
    assert lib.rib_selftest_mma_rate(1, 1, 64, 16, None, None, None) == 1
    assert b"cycles is null" in lib.rib_last_error()


def test_natural_alignment_checked(lib):
    """A pointer that misses its element size (2 bytes for 16-bit data, 4 for
    fp32) is refused with RIB_ERR_ALIGNMENT before any launch."""
    odd2, odd4 = 257, 258          # not 2-byte aligned / 2- but not 4-byte aligned
    mlp_bad = _lib.MlpDesc(10, 64, 3, 16, odd4, 256, 256, 256)
    assert lib.rib_pos_encode(ctypes.byref(mlp_bad), 16, 256, 256, 1 << 24, None) == 3
    mlp = _lib.MlpDesc(10, 64, 3, 16, 256, 256, 256, 256)
    assert lib.rib_pos_encode_bwd(ctypes.byref(mlp), 16, odd4, 256, 256, 256, 256, 256, 256, 1 << 30, None) == 3
    assert lib.rib_pos_encode_bwd(ctypes.byref(mlp_bad), 16, *[256] * 7, 1 << 30, None) == 3
    assert lib.rib_qkv_project(256, 0, 1, 8, 8, 48, 3, 16, odd2, 256, 256, 1.0, 256, 256, 256, None) == 3
    gate = [256, 0, 1, 8, 8, 48, 256, 256, 256, 256, 256, 256, 1 << 20, None]
    for i, bad in ((6, odd4), (7, odd4), (8, odd2), (9, odd4)):     # Wdw, bdw, Wpw, bpw
        args = list(gate)
        args[i] = bad
        assert lib.cla_gate(*args) == 3, i
        assert lib.cla_gate_static_scratch(*args[:12]) == 3, i
    d = _lib.attn_desc(1, 40, 72, 48, 3, 16, 16, 1.0)
    assert lib.rib_attention_bwd_prep(ctypes.byref(d), odd2, 256, 256, 256, 256, 256, None) == 3
    assert lib.rib_attention_bwd_prep(ctypes.byref(d), 256, 256, 256, 256, odd4, 256, None) == 3
    a = [256, 0, 1, 8, 8, 48, 3, 16, 256, 256, 256, 1.0, 256, 256, 256, 256, 256, 256, 256, 256, 1 << 20, None]
    for i, bad in ((8, odd2), (16, odd4)):                           # Wq, dWq
        args = list(a)
        args[i] = bad
        assert lib.rib_qkv_project_bwd(*args) == 3, i
    b = [256, 0, 1, 8, 8, 48] + [256] * 9 + [256, 1 << 22, None]
    for i, bad in ((6, odd4), (7, odd2), (11, odd4), (14, odd4)):    # Wdw, Wpw, dWdw, dbpw
        args = list(b)
        args[i] = bad
        assert lib.cla_gate_bwd(*args) == 3, i
    assert lib.rib_layernorm(256, 0, 256, 0, 10, 48, odd4, None, 1e-5, None) == 3
    assert b"alignment" in lib.rib_last_error() or b"aligned" in lib.rib_last_error()


def test_empty_maps_are_refused(lib):
    """A map with no pixels (B, H or W = 0) is an invalid argument for every
    map-shaped entry point; nothing is launched."""
    for B, H, W in ((0, 8, 8), (1, 0, 8), (1, 8, 0)):
        assert lib.rib_qkv_project(256, 0, B, H, W, 48, 3, 16, 256, 256, 256, 1.0, 256, 256, 256, None) == 1
        assert lib.cla_gate(256, 0, B, H, W, 48, 256, 256, 256, 256, 256, 256, 1 << 20, None) == 1
        assert lib.cla_gate_static_scratch(256, 0, B, H, W, 48, 256, 256, 256, 256, 256, None) == 1
        d = _lib.attn_desc(B, H, W, 48, 3, 16, 16, 1.0)
        assert _attn(lib, d) == 1
        assert lib.rib_attention_bwd_prep(ctypes.byref(d), 256, 256, 256, 256, 256, 256, None) == 1
        assert lib.rib_qkv_project_bwd(256, 0, B, H, W, 48, 3, 16, 256, 256, 256, 1.0, *[256] * 7, 256, 1 << 20, None) == 1
        assert lib.cla_gate_bwd(256, 0, B, H, W, 48, *[256] * 9, 256, 1 << 22, None) == 1
    assert rib.cla_gate_workspace_size(0, 8, 8, 48) == 0
    assert lib.rib_layernorm(256, 0, 256, 0, -1, 48, None, None, 1e-5, None) == 1


def test_fp16_maps_are_forward_only(lib):
    """RIB_F16 maps go into the forward entry points; the backward refuses
    them on the host (RIB_ERR_UNSUPPORTED) before launching anything."""
    assert lib.rib_qkv_project_bwd(256, 2, 1, 8, 8, 48, 3, 16, 256, 256, 256, 1.0, *[256] * 7, 256, 1 << 20, None) == 2
    assert b"bf16" in lib.rib_last_error()
    assert lib.cla_gate_bwd(256, 2, 1, 8, 8, 48, *[256] * 9, 256, 1 << 22, None) == 2
    # an fp16 map whose W*C is not a multiple of 8 has no fused gate
    assert lib.cla_gate(256, 2, 1, 8, 9, 36, 256, 256, 256, 256, 256, 256, 1 << 20, None) == 2
    assert b"fp16" in lib.rib_last_error()
    # an out_dtype outside bf16 / fp32 / fp16
    d = _lib.attn_desc(1, 32, 32, 48, 3, 16, 16, 1.0)
    d.out_dtype = 7
    assert _attn(lib, d) == 1


C_PROGRAM = r"""
#include <stdio.h>
#include "rib.h"
int main(void) {
  rib_attn_desc d = {1, 360, 640, 180, 6, 16, 64, 1.0f, 0, RIB_BF16};
  rib_mlp_desc m = {10, 128, 6, 16, NULL, NULL, NULL, NULL};
  printf("%d %zu %zu %zu\n", rib_version(), rib_window_attention_workspace_size(&d),
         cla_gate_workspace_size(1, 8, 8, 48), rib_pos_cache_bytes(&m, 64));
  rib_status s = rib_window_attention(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0);
  printf("%d %s\n", (int)s, rib_last_error());
  return 0;
}
"""


def test_header_is_a_plain_c_interface(tmp_path):
    """include/rib.h compiles as C11 with warnings as errors, and a C program
    links against librib.so and calls it (host-side calls only)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda_inc = "/usr/local/cuda/include"
    if gcc is None or not os.path.isdir(cuda_inc):
        pytest.skip("gcc or the CUDA headers are not available")
    _lib.load()
    src = tmp_path / "t.c"
    src.write_text(C_PROGRAM)
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = tmp_path / "t"
    cc = subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.dirname(_lib.HEADER),
                         "-I", cuda_inc, str(src), "-L", libdir, "-lrib", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    first, second = run.stdout.splitlines()
    assert first.split() == [str(rib.rib_version()), "0", str(8 * 8 * 48 * 2), str(6 * 64 * 64 * 16 * 2)]
    assert second.startswith("1 rib_window_attention: null pointer")
