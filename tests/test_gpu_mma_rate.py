"""The tcgen05.mma issue-rate diagnostic (rib_selftest_mma_rate) runs, returns
sane cycle counts and leaves no device error: its chains complete, each
thread's completion comes after its last issue, two issuing threads of one
CTA retire instructions at least as fast in aggregate as one, and the span
record reports how the CTAs of an SM overlapped."""
import math

import pytest

import windowed_attention_b200 as rib

pytestmark = pytest.mark.gpu


def test_mma_rate_probe(cuda_lib):
    one = rib.rib_selftest_mma_rate(1, 1, 64, 1024)
    two = rib.rib_selftest_mma_rate(1, 2, 64, 1024)
    pair = rib.rib_selftest_mma_rate(2, 2, 64, 1024)
    for r in (one, two, pair):
        print(r)
        assert math.isfinite(r["done_cycles_per_mma"]) and r["done_cycles_per_mma"] > 0
        assert r["done_cycles_per_mma"] >= r["issue_cycles_per_mma"] > 0
        # M = 128, N = 64, K = 16 is 262,144 flops: at most a few thousand cycles per instruction
        assert r["done_cycles_per_mma"] < 20000
        assert 0.0 <= r["overlap"] <= 1.0
    assert one["max_ctas_on_an_sm"] == 1 and two["max_ctas_on_an_sm"] == 1
    assert pair["max_ctas_on_an_sm"] <= 2 and pair["overlap"] > 0.5   # the two CTAs of an SM ran side by side
    assert two["sm_cycles_per_mma"] <= one["sm_cycles_per_mma"] * 1.05
