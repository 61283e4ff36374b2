import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large oracle computation")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


@pytest.fixture(autouse=True)
def _checked_build_plan_status():
    """Under the bounds-checked library (BFA_LIBRARY=checked), every plan a test
    creates is verified after the test: bfa_plan_device_status checks the guard
    bytes around its arrays and the kernels' index-check flag (BFA_ERR_BOUNDS)."""
    if os.environ.get("BFA_LIBRARY") != "checked":
        yield
        return
    import mask_skipping_flashattention_b200 as bfa
    made = []
    orig = bfa.Plan.__init__

    def init(self, *a, **k):
        orig(self, *a, **k)
        made.append(self)

    bfa.Plan.__init__ = init
    try:
        yield
    finally:
        bfa.Plan.__init__ = orig
    for P in made:
        if P._h is not None:
            P.device_status()
