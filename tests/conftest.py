import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """One line with every near-tie the parity tests excused (accept flips with
    |u - r| < 1e-6, draw picks within 1e-6 R, Viterbi paths within the score
    band), per kind, beside the number of decisions compared."""
    try:
        from parity import SESSION_COMPARED, SESSION_NEAR_TIES
    except Exception:
        return
    if not SESSION_COMPARED and not SESSION_NEAR_TIES:
        return
    kinds = sorted(set(SESSION_COMPARED) | set(SESSION_NEAR_TIES))
    terminalreporter.write_line(
        "near-ties excused: " + ", ".join(
            "%s %d of %d" % (k, SESSION_NEAR_TIES.get(k, 0), SESSION_COMPARED.get(k, 0))
            for k in kinds))
