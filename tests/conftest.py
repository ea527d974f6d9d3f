import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(params=["single", "heads"])
def prefill_kernel(request):
    """Runs a test under each work unit of the prefill kernel (two query tiles of one head;
    one query tile of two heads of one kv group), restoring the default afterwards."""
    import bf16_causal_prefill_attn_b200 as pkg
    k = {"single": pkg.ATTN_KERNEL_SINGLE, "heads": pkg.ATTN_KERNEL_HEADS}[request.param]
    pkg.attn_select_prefill_kernel(k)
    yield request.param
    pkg.attn_select_prefill_kernel(pkg.ATTN_KERNEL_SINGLE)
