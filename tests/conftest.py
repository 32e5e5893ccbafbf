import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def moe_gpu():
    """The CUDA library, built in-tree if needed, on a visible GPU."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    from mxfp4_expert_ffn_moe_b200 import build as moe_build
    moe_build.build()
    import mxfp4_expert_ffn_moe_b200 as moe
    moe.load_library()
    moe.moe_get_device_error()  # start from a clear error word
    return moe
