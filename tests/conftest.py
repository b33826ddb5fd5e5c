import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def gpu():
    """The CUDA path: libcsa2.so built in-tree and a CUDA device. Never falls back."""
    import torch
    import sparse_attention_decode_kv_b200 as csa2
    from sparse_attention_decode_kv_b200 import build as csa2_build
    if not torch.cuda.is_available():
        pytest.fail("a gpu-marked test ran without a CUDA device")
    csa2_build.build()
    csa2.lib()
    return torch.device("cuda:0")
