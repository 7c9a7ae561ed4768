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
def oracle_lib():
    import oracle
    return oracle.lib()


def pytest_collection_modifyitems(config, items):
    """GPU tests need a CUDA device; on a machine without one they are skipped
    (the CPU suite is run with -m "not gpu" anyway)."""
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session")
def hq():
    """The product library, built in-tree if the sources are newer."""
    from nvfp4_quantization_group_b200 import _build
    _build.build()
    import nvfp4_quantization_group_b200 as m
    m.lib()
    return m
