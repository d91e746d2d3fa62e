import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


def pytest_collection_modifyitems(config, items):
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


@pytest.fixture(scope="module")
def torch_cuda():
    """torch with a CUDA device, the library loaded (it fails loudly when its
    build is missing) and the device input generator built."""
    import torch
    assert torch.cuda.is_available()
    import moe_inputs as mi
    import sparse_mixture_experts_rmsnorm_b200  # noqa: F401
    if not os.path.exists(mi.CUDA_LIB):
        mi.build(cuda=True)
    return torch
