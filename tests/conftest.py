import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle


def pytest_sessionfinish(session, exitstatus):
    """With GEMM_EPI_DBIAS_LOG=<path>, write the worst dbias error ratios the
    parity checks saw (against the stated bound and against the full bound)."""
    path = os.environ.get("GEMM_EPI_DBIAS_LOG")
    if not path:
        return
    mod = sys.modules.get("_parity")
    if mod is None or not getattr(mod, "DBIAS_RATIOS", None):
        return
    import json

    with open(path, "w") as f:
        json.dump(mod.DBIAS_RATIOS, f, indent=1, sort_keys=True)
