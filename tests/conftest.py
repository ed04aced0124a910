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
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session")
def oracle():
    from oracle import Oracle
    return Oracle()


def pytest_terminal_summary(terminalreporter):
    """Per mask comparison: rows checked, rows the 1e-3 gap rule exempts, and
    rows identical to the oracle's (printed even under -q)."""
    try:
        import parity_helpers
    except Exception:
        return
    if not parity_helpers.MASK_REPORT:
        return
    terminalreporter.write_line("mask rows (label: rows, exempt by the gap rule, identical):")
    for label, rows, n_ex, n_exact in parity_helpers.MASK_REPORT:
        terminalreporter.write_line(f"  {label}: {rows}, {n_ex} ({100.0 * n_ex / rows:.1f}%), "
                                    f"{n_exact} ({100.0 * n_exact / rows:.2f}%)")
