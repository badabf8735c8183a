"""pytest configuration: the `gpu` marker and shared helpers."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


@pytest.fixture(autouse=True)
def _device_status(request):
    """After every GPU test: no kernel may have recorded an error in its
    workspace's status word (a bounded wait that ran out, or a failed internal
    consistency check) -- those results would otherwise pass unnoticed."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from long_context_sparse_rtp_b200.rtp import rtp_check_device
    rtp_check_device()
