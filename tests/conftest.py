import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size inputs, takes more than a few seconds")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle

    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _no_failed_index_checks(request):
    """Under the checked build (CK_LIBRARY=libck_checked.so), every GPU test
    must also leave no failed device-side index check behind."""
    yield
    if "gpu" in request.keywords and os.environ.get("CK_LIBRARY", "").endswith("libck_checked.so"):
        import int8_quantized_linear_convrot256_b200 as ck

        bits = ck.checked_violations()
        assert bits == 0, f"failed index checks in the checked build, class bits {bits:#x}"
