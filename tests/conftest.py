import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running CPU oracle work")


def pytest_collection_modifyitems(config, items):
    # GPU tests fail loudly (not skip) when selected with -m gpu on a machine without a GPU,
    # so that a missing device or library is never mistaken for a pass.
    pass


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA C-ABI library, loaded for GPU tests; raises if missing."""
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test selected but no CUDA device is visible")
    import exact_io_aware_98_b200 as fa
    fa.load()
    return fa
