import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session", autouse=True)
def _built_helpers():
    """The oracle and the input generator are plain C/C++ built with the host compiler."""
    from oracle import build_oracle
    from quantized_attention_kvq_b200 import build

    build_oracle.build()
    build.build_gen()
    yield
