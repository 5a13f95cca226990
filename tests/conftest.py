import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle


def pytest_sessionfinish(session, exitstatus):
    """With DMOE_PARITY_LOG set, write every float comparison of the session (what, relative
    L2, max-abs / RMS, bound) to that JSON file."""
    path = os.environ.get("DMOE_PARITY_LOG")
    if not path:
        return
    try:
        import helpers
    except Exception:
        return
    import json

    with open(path, "w") as fh:
        json.dump([{"what": w, "rel_l2": r, "max_abs_rms": m, "bound": b}
                   for w, r, m, b in helpers.RECORD], fh, indent=1)
