import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle

    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def semkv():
    """The library's Python binding (builds libsemkv.so first if it is stale; loads without a GPU)."""
    from mixed_precision_kv_semkv_b200 import build

    build.build()
    import mixed_precision_kv_semkv_b200 as m

    return m
