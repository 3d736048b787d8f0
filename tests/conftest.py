import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload; minutes of CPU time")


@pytest.fixture(scope="session")
def gpu_lib():
    """The compiled library, loaded; skips nothing -- a GPU test must fail loudly."""
    import paged_kv_attention_37_b200 as pkv
    return pkv
