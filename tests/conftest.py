import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


@pytest.fixture(autouse=True)
def _device_error_word_stays_clear(request):
    """With the bounds-checked build loaded (TCQ_LIBRARY=debug), every GPU test
    must leave the device error word clear: no index of any instrumented kernel
    went out of its buffer and no bounded wait gave up."""
    yield
    if os.environ.get("TCQ_LIBRARY") != "debug" or request.node.get_closest_marker("gpu") is None:
        return
    from trellis_coded_weight_tcq_b200 import tcq

    if tcq._lib is None:  # the test never loaded the library
        return
    flags = tcq.device_errors()
    assert flags == 0, f"device error flags {flags:#x} after {request.node.nodeid}"
