import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case (minutes)")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Outputs where |y| >= 32, whose per-output bound is half an fp16 spacing (plus fp32
    accumulation slack) instead of 1e-2: how many there were and how many needed it."""
    try:
        from tests.owq_checks import RELAXED_REPORT
    except Exception:
        return
    if not RELAXED_REPORT:
        return
    terminalreporter.write_sep("-", "outputs with |y| >= 32 (relaxed per-output bound)")
    for where, info in RELAXED_REPORT:
        terminalreporter.write_line(
            f"{where}: {info['n_big']} outputs with |y| >= 32 (max |y| {info['max_abs_y']:.1f}), "
            f"{info['n_relaxed']} over 1e-2, worst {info['worst_relaxed_ulp']:.3f} fp16 spacings")
