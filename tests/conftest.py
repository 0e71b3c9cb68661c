"""Shared test set-up: the `gpu` marker, import paths, and the oracle fixture."""
import os
import sys

import pytest

_TESTS = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_TESTS)
for p in (_ROOT, _TESTS):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()


@pytest.fixture(scope="session")
def libttt():
    """The CUDA library, built in-tree for sm_100a if it is missing (nvcc needs no GPU)."""
    from test_rnn_layers_b200 import build
    build.build()
    import test_rnn_layers_b200 as ttt
    return ttt
