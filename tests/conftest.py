import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload (minutes of CPU oracle work)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built C-ABI library (built in-tree on first use); GPU tests only."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import attention_dit_attn_b200 as dit
    dit.ensure_built()
    return dit
