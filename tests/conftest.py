import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def gpu_lib():
    """The C-ABI library through its Python binding; a GPU test fails (not skips)
    when the extension or the device is missing."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for tests marked gpu")
    import mxfp8_grouped_gemm_moe_b200 as mx
    mx.load()
    return mx
