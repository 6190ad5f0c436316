import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # The expert-parallel tests run the single-GPU layer inside every rank, so
    # they come after every test of the layer's own entry points (a layer
    # failure is reported as such first).  The entry point without a caller
    # workspace comes last of all: a run that stops at its first failure has
    # then run everything else.
    rank = {"test_gpu_ep": 1, "test_zz_no_alloc": 2}
    items.sort(key=lambda it: rank.get(getattr(it.module, "__name__", ""), 0))


@pytest.fixture(scope="session")
def olib():
    import oracle
    return oracle.load()


@pytest.fixture(scope="session")
def moelib():
    """The CUDA library, built in place if missing (nvcc cross-compiles here)."""
    from moe_expert_layer_08_b200 import build
    build.build()
    import moe_expert_layer_08_b200 as m
    return m.load()
