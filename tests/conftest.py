import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: statistical pins that take tens of seconds")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(autouse=True)
def _device_status_after_gpu_tests(request):
    """After every GPU test, read the status word of each workspace the binding
    holds: a tcgen05 or fused kernel whose bounded wait ran out records it
    there, and its output would otherwise look like a result."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    from activation_perturbation_es_b200 import dust
    if dust._lib is None:
        return
    import torch
    if not torch.cuda.is_available() or not torch.cuda.is_initialized():
        return
    assert dust.poll_all() == "ok"
