import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()


def pytest_terminal_summary(terminalreporter):
    """The parity report: one line per comparison the tests made against a reference."""
    import harness
    if not harness.PARITY_LOG:
        return
    tr = terminalreporter
    tr.section("parity report: max|err|/RMS(ref), beyond bf16 output rounding, RMS(err)/RMS(ref), bound")
    for what, mx, arith, rmse, tol in harness.PARITY_LOG:
        tr.write_line(f"{mx:9.2e} {arith:9.2e} {rmse:9.2e}  <= {tol:g}   {what}")
