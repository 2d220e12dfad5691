"""GPU parity of the full SST block (RIB/SST write-up section 3.1: LayerNorm ->
RIB attention -> CLA -> ConvFFN, FFN expansion 1.25) through the C-ABI against
the fp64 oracle: rib_conv_ffn alone (every element, ragged maps, the widest
hidden width), the six-block SST stack on a reduced map (every element) and
on the full 640x360 map (every block on sampled windows, from the GPU's own
input to that block). Tolerance: max abs 2e-2, mean abs 2e-3.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from windowed_attention_b200.workloads import WORKLOADS, ffn_hidden, make_inputs

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN = 2e-2, 2e-3
THREADS = max(1, min(16, oracle.oracle_cores()))


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _check(got, ref, what):
    d = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    print(f"{what}: max {d.max():.3e} mean {d.mean():.3e}")
    assert d.max() <= TOL_MAX and d.mean() <= TOL_MEAN, f"{what}: max {d.max():.3e} mean {d.mean():.3e}"


@pytest.mark.parametrize("B,H,W,C,xdt", [
    (1, 20, 36, 180, torch.bfloat16),   # hidden 225 (stored 232): three TMA boxes per row, two output products
    (1, 20, 36, 180, torch.float16),    # the same with an fp16 LayerNorm output (the stack's)
    (2, 9, 17, 48, torch.bfloat16),     # hidden 60 (stored 64), ragged 4x16 tiles
    (1, 8, 16, 160, torch.bfloat16),    # hidden 200: wide, both output products, L = 64 lines
    (1, 8, 16, 200, torch.bfloat16),    # hidden 250 (stored 256): the widest hidden width, first map with one accumulator
])
def test_conv_ffn_matches_oracle(cuda_lib, B, H, W, C, xdt):
    from windowed_attention_b200.layer import ConvFFN
    layer = replace(WORKLOADS["sst"].layer, B=B, H=H, W=W, C=C, heads=4 if C == 160 else WORKLOADS["sst"].layer.heads)
    inp = make_inputs("sst", layer=layer)
    s = inp["shape"]
    f = inp["ffns"][0]
    assert f["W1"].shape[1] == ffn_hidden(C)
    g = torch.Generator().manual_seed(31)
    xn = torch.randn(B, H, W, C, generator=g).to(xdt)
    x0 = torch.randn(B, H, W, C, generator=g)
    ffn = ConvFFN(s, f, "cuda")
    ffn.ws.fill_(float("nan"))
    x = x0.to("cuda").contiguous()
    ffn(xn.to("cuda").contiguous(), x, s)
    torch.cuda.synchronize()
    cuda_lib.rib_device_error()
    ref = x0.numpy().astype(np.float64) + oracle.conv_ffn(xn.float().numpy(), **{k: v.numpy() for k, v in f.items()})
    _check(_np(x), ref, f"ConvFFN C={C}")


def test_conv_ffn_refuses_what_does_not_fit(cuda_lib):
    """C = 256 with hidden 320: hidden widths above 256 (one MMA's N) are
    refused on the host before anything is launched."""
    from windowed_attention_b200.layer import ConvFFN
    layer = replace(WORKLOADS["sst"].layer, B=1, H=8, W=16, C=256, heads=8)
    inp = make_inputs("sst", layer=layer)
    s = inp["shape"]
    assert inp["ffns"][0]["W1"].shape[1] == ffn_hidden(256) == 320
    ffn = ConvFFN(s, inp["ffns"][0], "cuda")
    x = torch.zeros(1, 8, 16, 256, device="cuda")
    xn = torch.zeros(1, 8, 16, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.RibError) as e:
        ffn(xn, x, s)
    assert e.value.status == 2


def test_sst_stack_reduced_map_full_compare(cuda_lib):
    from windowed_attention_b200.layer import RibStack
    wl = WORKLOADS["sst"]
    small = replace(wl.layer, H=72, W=136)
    inp = make_inputs("sst", layer=small)
    st = RibStack(small, inp["blocks"], wl.windows, "cuda", ffns=inp["ffns"])
    out = st.forward(inp["X"].to("cuda", torch.bfloat16).contiguous())
    cuda_lib.rib_device_error()
    ref = oracle.sst_stack_forward(inp["X"], inp["blocks"], inp["ffns"], wl.windows, small.heads, small.R, small.L,
                                   threads=THREADS)
    _check(_np(out), ref, "SST stack (72x136)")


def _sample_window_ids(H, W, M):
    ny, nx = -(-H // M), -(-W // M)
    return sorted({0, nx - 1, nx, (ny // 2) * nx + nx // 2, (ny - 1) * nx, (ny - 1) * nx + nx // 2, ny * nx - 1})


def test_sst_stack_full_map_every_block_sampled_windows(cuda_lib):
    """Every block of the six-block SST stack on the full 640x360 map, in its
    two halves: the gated attention (as in the plain stack test) and the
    ConvFFN residual, each from the GPU's own input to that half; both are
    local (window plus a one-pixel halo), so the oracle computes them on
    sampled windows, including the padded bottom row of every window size."""
    from windowed_attention_b200.layer import RibStack
    wl = WORKLOADS["sst"]
    s = wl.layer
    inp = make_inputs("sst")
    st = RibStack(s, inp["blocks"], wl.windows, "cuda", ffns=inp["ffns"])
    st.load(inp["X"].to("cuda", torch.bfloat16).contiguous())
    for k, M in enumerate(wl.windows):
        xin = _np(st.x)
        xmid = _np(st.block(k, ffn=False))
        xout = _np(st.ffn(k))
        cuda_lib.rib_device_error()
        ids = _sample_window_ids(s.H, s.W, M)
        blocks = oracle.rib_layer_forward_windows(oracle.layernorm(xin), inp["blocks"][k], s.heads, s.R, s.L, M, ids,
                                                  threads=THREADS)
        f = {kk: v.numpy() for kk, v in inp["ffns"][k].items()}
        ea, ef = [], []
        for b, y0, x0, blk in blocks:
            h, w = blk.shape[0], blk.shape[1]
            ea.append(np.abs(xmid[b, y0:y0 + h, x0:x0 + w] - (xin[b, y0:y0 + h, x0:x0 + w] + blk)).reshape(-1))
            # the ConvFFN on the window plus a one-pixel halo of the GPU's x_mid
            hy0, hx0 = max(y0 - 1, 0), max(x0 - 1, 0)
            hy1, hx1 = min(y0 + h + 1, s.H), min(x0 + w + 1, s.W)
            patch = xmid[b:b + 1, hy0:hy1, hx0:hx1]
            ffn = oracle.conv_ffn(oracle.layernorm(patch), **f)[0]
            ref = xmid[b, y0:y0 + h, x0:x0 + w] + ffn[y0 - hy0:y0 - hy0 + h, x0 - hx0:x0 - hx0 + w]
            ef.append(np.abs(xout[b, y0:y0 + h, x0:x0 + w] - ref).reshape(-1))
        da, df = np.concatenate(ea), np.concatenate(ef)
        print(f"block {k} (M={M}): attention max {da.max():.3e} mean {da.mean():.3e}; "
              f"ConvFFN max {df.max():.3e} mean {df.mean():.3e}")
        assert da.max() <= TOL_MAX and da.mean() <= TOL_MEAN
        assert df.max() <= TOL_MAX and df.mean() <= TOL_MEAN
