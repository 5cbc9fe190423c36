import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU oracle case")


@pytest.fixture(scope="session")
def nclib():
    """The package with its CUDA library built in-tree (fails, never skips, if it cannot be)."""
    from decoder_only_transformer_nc_b200 import build as ncbuild
    ncbuild.build_library()
    import decoder_only_transformer_nc_b200 as nc
    nc.lib()
    return nc


@pytest.fixture(scope="session")
def gpu(nclib):
    """Requires a CUDA sm_100 device; a missing device is a failure, not a skip."""
    import torch
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    major, minor = torch.cuda.get_device_capability(0)
    assert (major, minor) == (10, 0), f"expected sm_100, got sm_{major}{minor}"
    torch.cuda.set_device(0)
    return nclib
