import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")
    # The C ABI library is built in-tree; build it once if this checkout has not yet.
    from block_sparse_video_tile3d_b200 import build as _build
    if not os.path.exists(_build.LIB):
        _build.build()


@pytest.fixture(scope="session")
def cuda_available():
    import torch
    return torch.cuda.is_available()
