import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running full-size case")


def pytest_terminal_summary(terminalreporter):
    """Largest observed error per test against its tolerance (GPU parity checks)."""
    try:
        from tests.parity import OBSERVED
    except ImportError:
        return
    if not OBSERVED:
        return
    worst = {}
    for test, what, err, tol in OBSERVED:
        k = (test, tol)
        if k not in worst or err > worst[k][1]:
            worst[k] = (what, err)
    terminalreporter.section("observed parity errors (largest per test)")
    for (test, tol), (what, err) in sorted(worst.items()):
        terminalreporter.write_line(f"{err:10.3e} / {tol:.0e}  {test}  [{what}]")
