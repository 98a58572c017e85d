import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running check")


@pytest.fixture(scope="session")
def cuda_lib():
    """The product library, built in-tree; skips nothing: a GPU test fails loudly
    if the CUDA extension is missing."""
    import gated_delta_rule_134_b200 as kda
    kda.load()
    return kda
