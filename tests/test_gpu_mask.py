"""GPU parity of the optional key-padding mask (rib_attn_desc.mask_padding):
padded pixels are excluded from every softmax instead of entering it as keys
with Kc = V = 0. Reference: the fp64 oracle with ``mask_padding=True``;
tolerance max abs 2e-2, mean abs 2e-3 (as the other parity tests)."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from windowed_attention_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN = 2e-2, 2e-3


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("H,W,C,heads,M", [
    (40, 72, 180, 6, 32),    # 64-key tiles, 32-wide heads; bottom and right padding
    (40, 40, 48, 3, 16),     # 64-key tiles, 16-wide heads
    (100, 96, 48, 3, 96),    # 128-key tiles; bottom padding only
], ids=["c180_m32", "c48_m16", "c48_m96"])
def test_key_padding_mask_matches_oracle(cuda_lib, H, W, C, heads, M):
    from windowed_attention_b200.layer import RibLayer
    layer = replace(WORKLOADS["tiny"].layer, H=H, W=W, C=C, heads=heads, window=M, dtype="bf16")
    inp = make_inputs("tiny", layer=layer)
    s = inp["shape"]
    lay = RibLayer(s, inp, "cuda")
    X = inp["X"].to("cuda", torch.bfloat16).contiguous()
    Ym = lay.forward(X, mask_padding=True).clone()
    Yu = lay.forward(X).clone()
    torch.cuda.synchronize()
    cuda_lib.rib_device_error()
    ref, _ = oracle.rib_layer_forward(inp["X"], inp, s.heads, s.R, s.L, M, threads=4, mask_padding=True)
    d = np.abs(_np(Ym) - ref)
    assert np.all(np.isfinite(_np(Ym)))
    assert d.max() <= TOL_MAX and d.mean() <= TOL_MEAN, f"max {d.max():.3e} mean {d.mean():.3e}"
    # the window at the origin has no padding: the masked kernel computes it as
    # the unmasked one does (to the bit when both run the safe softmax, dh ==
    # DP; with padded heads the unmasked kernel carries its softmax reference
    # in the score product, which rounds differently)
    if C // heads == cuda_lib.rib_head_pad(C, heads):
        assert torch.equal(Ym[:, :M, :M], Yu[:, :M, :M])
    else:
        d0 = np.abs(_np(Ym[:, :M, :M]) - _np(Yu[:, :M, :M]))
        assert d0.max() <= TOL_MAX and d0.mean() <= TOL_MEAN
    # and the mask matters where there is padding
    assert not torch.equal(Ym, Yu)
