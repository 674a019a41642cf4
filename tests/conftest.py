import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


def pytest_sessionfinish(session, exitstatus):
    """With RPTQ_PARITY_REPORT set, write the measured agreement of the GPU comparisons."""
    path = os.environ.get("RPTQ_PARITY_REPORT")
    if not path:
        return
    mod = sys.modules.get("tests.gpu_common")
    if mod is None:
        return
    import json
    with open(path, "w") as f:
        json.dump(mod.REPORT, f, indent=1, sort_keys=True)
