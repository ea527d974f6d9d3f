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


KERNELS = {"single": "ATTN_KERNEL_SINGLE", "heads": "ATTN_KERNEL_HEADS",
           "k64": "ATTN_KERNEL_K64", "k64heads": "ATTN_KERNEL_K64_HEADS"}


@pytest.fixture(params=list(KERNELS))
def prefill_kernel(request):
    """Runs a test under each prefill kernel (128-key tiles with two query tiles of one head
    or one query tile of two heads of one kv group per CTA; 64-key tiles with either unit),
    restoring the default afterwards."""
    import bf16_causal_prefill_attn_b200 as pkg
    pkg.attn_select_prefill_kernel(getattr(pkg, KERNELS[request.param]))
    yield request.param
    pkg.attn_select_prefill_kernel(pkg.ATTN_KERNEL_SINGLE)


@pytest.fixture
def key_tile(prefill_kernel):
    """Keys per tile of the selected prefill kernel: the FP8 lean-P reference max is updated
    once per key tile, so the emulator replays the kernel with this tile."""
    return 64 if prefill_kernel.startswith("k64") else 128
