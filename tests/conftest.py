import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built libminf.so")


@pytest.fixture(scope="session")
def orc():
    import oracle

    return oracle.get()


@pytest.fixture(scope="session")
def minf_lib():
    """The built product library (compiled here if missing); no GPU call is made."""
    from dynamic_sparse_attention_est_b200 import build_lib

    return build_lib.ensure_built()


def pytest_collection_modifyitems(config, items):
    import torch

    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device here")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
