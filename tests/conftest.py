import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def no_device_error_left(request):
    """After every GPU test, no bounded in-kernel wait may have run out unnoticed:
    the device error flags must be clear (a test that provokes a timeout reads
    and clears them itself)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import scaled_dot_product_14_b200 as S
    torch.cuda.synchronize()
    st, code = S.sdpa_check_device_error()
    assert code == 0, f"a bounded in-kernel wait ran out during this test (device error code {code})"
