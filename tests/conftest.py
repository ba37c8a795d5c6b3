import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Per-element error statistics of the feature checks against the oracle
    (|err| / sum of |terms| per element: median, 99th percentile, maximum)."""
    from tests.util import ERROR_LOG
    if not ERROR_LOG:
        return
    tr = terminalreporter
    tr.section("error statistics vs the oracle (|err| / sum|terms| per element)")
    tr.write_line(f"{'check':<72} {'dtype':<9} {'max/max|ref|':>12} {'p50':>10} {'p99':>10} {'max':>10}")
    for r in ERROR_LOG:
        name = f"{r['test'].split('::')[-1]} {r['what']}"[:72]
        tr.write_line(f"{name:<72} {r['dtype']:<9} {r['max_err_over_max_ref']:>12.3e} {r['rel_terms_p50']:>10.3e} "
                      f"{r['rel_terms_p99']:>10.3e} {r['rel_terms_max']:>10.3e}")
