import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a); run with -m gpu")


@pytest.fixture(scope="session")
def ref():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def gpu():
    """The CUDA library on cuda:0; GPU tests fail (not skip) if it is missing."""
    import torch
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    import microscaling_fp4_quantization_bf16_b200 as fp4q
    fp4q.load()
    return fp4q
