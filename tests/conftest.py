import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an sm_100a GPU (B200)")
    config.addinivalue_line("markers", "slow: long-running CPU case")


def pytest_collection_modifyitems(config, items):
    # GPU tests are never silently skipped on a GPU machine: they fail loudly if the
    # CUDA extension cannot be loaded.  On a CPU-only machine they are skipped.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture
def few_token_kernel():
    """Run every forward with M <= 16 tokens on the few-token kernel, whatever
    the weight's size (the library's default sends small weights to the
    mid-size kernel); restores the previous setting afterwards."""
    import bit_nf4_quantized_26_b200 as lib
    prev = lib.qlora_set_few_token_threshold(0)
    yield
    lib.qlora_set_few_token_threshold(prev)
