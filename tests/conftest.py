import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle():
    from oracle import oracle as O
    O.build()
    return O


@pytest.fixture(scope="session")
def ans_lib():
    """The product C-ABI library (built in-tree if missing or stale)."""
    from rans_decode_gemm_b200 import ans
    ans.load()
    return ans


@pytest.fixture(scope="session")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture
def plan_limits():
    """plan_limits(max_ctas=, max_producers=, schedule="local"|"central"):
    limits on the fused-GEMM launch plans of this test (the library's internal
    test hook), restored to the defaults afterwards."""
    from rans_decode_gemm_b200 import ans
    state = {"max_ctas": 0, "max_producers": 0, "schedule": "local"}

    def set_limits(**kw):
        state.update(kw)
        ans._set_plan_limits(state["max_ctas"], state["max_producers"],
                             state["schedule"] == "central")
    yield set_limits
    ans._set_plan_limits(0, 0, False)
