import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "device_error_expected: the test itself sets and clears "
                                       "bits of the library's device error word")


@pytest.fixture(autouse=True)
def _device_error_word_stays_clear(request):
    """After every GPU test: no staged kernel recorded a wait that gave up, a
    bounds violation (the bounds-checking build) or an out-of-range input,
    unless the test plants one and clears the word itself."""
    yield
    if "gpu" not in request.keywords or "device_error_expected" in request.keywords:
        return
    import structured_sparse_attention_fibonacci_b200 as sa
    word = sa.device_error(clear=True)
    assert word == 0, f"device error word {word:#x} after {request.node.name}"


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this environment")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
