import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.load()


def pytest_terminal_summary(terminalreporter):
    """How many attention outputs passed only through the |ref| >= 4 allowance
    of the parity bound (see mg_testlib.elementwise_bound)."""
    try:
        from mg_testlib import WIDENED
    except Exception:
        return
    if WIDENED["checked"]:
        terminalreporter.write_line(
            f"parity bound: {WIDENED['checked']} output elements compared with the oracle; "
            f"{WIDENED['over_plain_bound']} above a plain 1e-2 (allowed only where |ref| >= 4, "
            f"worst |err| {WIDENED['worst_over']:.4e}); smallest slack to the bound {WIDENED['min_slack']:.4e} "
            f"at {WIDENED['min_slack_at']}")
