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
    from oracle import oracle
    oracle.build()
    return oracle


_PARITY_REPORT = []


@pytest.fixture(scope="session")
def parity_report():
    """Rows (workload, sequences, max-abs, rel-L2, max-abs / max|oracle|)
    collected by the full-size parity tests, printed at the end of the run."""
    return _PARITY_REPORT


def pytest_terminal_summary(terminalreporter):
    if not _PARITY_REPORT:
        return
    terminalreporter.write_line("parity against the fp64 oracle (whole outputs):")
    terminalreporter.write_line(f"  {'workload':<20} {'seqs':>5} {'max_abs':>10} {'rel_l2':>10} {'abs/max':>10}")
    for name, n, max_abs, rel, frac in _PARITY_REPORT:
        terminalreporter.write_line(f"  {name:<20} {n:>5} {max_abs:>10.3e} {rel:>10.3e} {frac:>10.3e}")
