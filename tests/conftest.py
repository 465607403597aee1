import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size cases (minutes of CPU oracle time)")


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


@pytest.fixture(autouse=True)
def _library_status_word_stays_clean(request):
    """After every GPU test, the library's own device status word (where
    kernels called with dev_status=None report a wait that gave up) must
    still read 0: no call in the test timed out unnoticed."""
    yield
    if "gpu" not in request.keywords:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import bit_w4a4_diffusion_b200 as B
    torch.cuda.synchronize()
    code = B.device_status(clear=True)
    assert code == 0, f"a kernel called without dev_status reported a timeout (code {code})"
