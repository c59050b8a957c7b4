import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_cuda = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_cuda = False
    if has_cuda:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(params=[1, 2], ids=["one_kernel", "two_kernels"])
def chunk_schedule(request):
    """Runs a prefill test under each schedule of the tensor-core path (gdr_debug_set_chunk_schedule): 1 the
    one-kernel schedule, 2 the WY pass plus chain kernel.  Shapes the tensor cores do not take run the CUDA-core
    kernel under both."""
    import gated_deltanet_gdr_b200 as gdr
    gdr.set_chunk_schedule(request.param)
    try:
        yield request.param
    finally:
        gdr.set_chunk_schedule(0)
