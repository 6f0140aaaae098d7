import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


@pytest.fixture(scope="session")
def gpu_lib():
    """The CUDA library through its Python binding; fails loudly if it is missing."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_attention_46_b200 as lf
    from block_sparse_attention_46_b200 import build
    build.build()      # rebuilds if a source is newer than liblf.so; raises if nvcc fails
    lf.load()          # raises if liblf.so is absent or does not load
    return lf
