import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.get()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    import util
    if not util.PARITY_STATS:
        return
    tr = terminalreporter
    tr.section("parity against the oracle (O: fp32 output; P codes: 8-bit codes of the softmax)")
    tr.write_line(f"{'case':58s} {'max-abs':>10s} {'mean-abs':>10s} {'P-code mismatches':>22s}")
    for case, mx, mean, pm, pt in util.PARITY_STATS:
        pstr = "-" if pm is None else f"{pm} of {pt}"
        tr.write_line(f"{case[:58]:58s} {mx:10.3e} {mean:10.3e} {pstr:>22s}")
