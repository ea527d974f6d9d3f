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


# prefill kernel settings: (unit and schedule flags, cap on the persistent grid).  The caps
# make the small test problems run several units per CTA on the persistent schedule.
KERNELS = {"single": (("ATTN_KERNEL_SINGLE",), 0),
           "heads": (("ATTN_KERNEL_HEADS",), 0),
           "persistent": (("ATTN_KERNEL_SINGLE", "ATTN_KERNEL_PERSISTENT"), 5),
           "heads_persistent": (("ATTN_KERNEL_HEADS", "ATTN_KERNEL_PERSISTENT"), 3),
           "dynamic": (("ATTN_KERNEL_SINGLE", "ATTN_KERNEL_DYNAMIC"), 0),
           # both BF16 pipelines on every shape (without a flag the pipeline follows Hq / Hkv)
           "dynamic_bf16_s_ahead": (("ATTN_KERNEL_SINGLE", "ATTN_KERNEL_DYNAMIC",
                                     "ATTN_KERNEL_BF16_S_AHEAD"), 0),
           "persistent_bf16_p_over_s": (("ATTN_KERNEL_SINGLE", "ATTN_KERNEL_PERSISTENT",
                                         "ATTN_KERNEL_BF16_P_OVER_S"), 5),
           "auto": (("ATTN_KERNEL_AUTO",), 0)}


def select_kernel(pkg, name):
    flags, cap = KERNELS[name]
    k = 0
    for f in flags:
        k |= getattr(pkg, f)
    pkg.attn_select_prefill_kernel(k)
    pkg.attn_selftest_max_ctas(cap)


@pytest.fixture(params=list(KERNELS))
def prefill_kernel(request):
    """Runs a test under each work unit (two query tiles of one head; one query tile of two
    heads of one kv group) and schedule (one CTA per unit; a static persistent grid, capped
    so that CTAs run several units; dynamic take-over of units) of the prefill kernel,
    restoring the default afterwards."""
    import bf16_causal_prefill_attn_b200 as pkg
    select_kernel(pkg, request.param)
    yield request.param
    pkg.attn_select_prefill_kernel(pkg.ATTN_KERNEL_AUTO)
    pkg.attn_selftest_max_ctas(0)


@pytest.fixture
def key_tile(prefill_kernel):
    """Keys per tile of the selected prefill kernel: the FP8 lean-P reference max is updated
    once per key tile, so the emulator replays the kernel with this tile."""
    return 128
