"""Failure detection on the GPU without a fault: one bounded device wait is
made to run out (a barrier nothing arrives on, 2 ms limit). The host must
read RIB_ERR_TIMEOUT with the wait's site, the error word must be cleared by
that read, and the context must stay usable (a layer forward still matches
its earlier result bit for bit)."""
import pytest
import torch

from windowed_attention_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_the_context_survives(cuda_lib):
    from windowed_attention_b200 import _lib
    from windowed_attention_b200.layer import RibLayer
    inp = make_inputs("tiny")
    s = inp["shape"]
    lay = RibLayer(s, inp, "cuda")
    X = inp["X"].to("cuda", torch.float32).contiguous()
    before = lay.forward(X).clone()
    cuda_lib.rib_device_error()                      # clean state

    cuda_lib.rib_selftest_wait_timeout(2000)
    with pytest.raises(_lib.RibError) as exc:
        cuda_lib.rib_device_error()
    assert exc.value.status == 5                     # RIB_ERR_TIMEOUT
    assert "901" in str(exc.value) and "self-test" in str(exc.value)
    cuda_lib.rib_device_error()                      # the read cleared the word

    after = lay.forward(X)
    cuda_lib.rib_device_error()
    assert torch.equal(before, after)
