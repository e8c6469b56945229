import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU-side check")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.lib()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """One line on the near-tie mask differences of the calibrated-tau cases."""
    from tests import parity
    if parity.TIE_LOG:
        ties = sum(t for _, t, _ in parity.TIE_LOG)
        valid = sum(v for _, _, v in parity.TIE_LOG)
        worst = max(parity.TIE_LOG, key=lambda x: x[1])
        terminalreporter.write_line(
            f"calibrated-tau parity: {len(parity.TIE_LOG)} cases, {ties} near-tie mask differences in {valid} "
            f"compared entries (most: {worst[1]} in {worst[0]})")
