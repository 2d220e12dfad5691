import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built C-ABI library bound through the Python binding (GPU tests only)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import windowed_attention_b200 as rib
    from windowed_attention_b200 import _lib
    lib = rib.load()
    # the kernels under test are the in-tree build, not a copy found elsewhere
    assert os.path.samefile(lib._name, _lib.LIB_PATH), lib._name
    print(f"librib loaded from {lib._name}")
    return rib
