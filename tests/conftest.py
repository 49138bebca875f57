import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle():
    import oracle as o
    o.build()
    return o


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Per comparison of GPU outputs with the oracle: the normalised max error
    (bf16 output rounding included), the arithmetic error beyond each
    output's half-ulp (both relative to the largest output), and the share
    of outputs that differ from the correctly rounded oracle value."""
    try:
        import pw_testutil
    except ImportError:
        return
    rows = pw_testutil.RECORDED
    if not rows:
        return
    tr = terminalreporter
    tr.section("output errors against the oracle")
    tr.write_line("%-72s %12s %12s %9s" % ("test", "norm_max", "arith", "rne_diff"))
    for test, e in rows:
        tr.write_line("%-72s %12.3e %12.3e %8.1f%%" % (test[-72:], e["norm_max_rel"],
                                                     e["arith_excess"], 100 * e["rne_mismatch"]))
    worst = max(e["arith_excess"] for _, e in rows)
    tr.write_line("largest arithmetic error beyond the output rounding: %.3e of scale "
                  "(budget 2e-3)" % worst)
