import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


# Parity margins measured by the full-size GPU tests: (test, quantity, value, bar). They are
# printed at the end of the run so that the margin to each bar shows in the run's summary.
MARGINS = []


def record_margin(test: str, quantity: str, value: float, bar: float) -> None:
    MARGINS.append((test, quantity, float(value), float(bar)))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if not MARGINS:
        return
    terminalreporter.section("parity margins (rel-L2 against the fp64 oracle)")
    for test, quantity, value, bar in MARGINS:
        terminalreporter.write_line(f"{test:44s} {quantity:34s} {value:.3e}  bar {bar:.0e}  "
                                    f"margin {bar / max(value, 1e-300):6.1f}x")


def rel_l2(x, ref):
    import numpy as np
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.load()
