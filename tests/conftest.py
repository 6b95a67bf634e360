import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    # tests/test_zz_* files run last, whatever the collection order
    items.sort(key=lambda it: os.path.basename(str(it.fspath)).startswith("test_zz_"))


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _name_reports(request):
    import tolerance
    tolerance.CURRENT_TEST[0] = request.node.nodeid
    yield


def pytest_terminal_summary(terminalreporter):
    """The error report of every bf16 output checked in this session."""
    import tolerance
    if not tolerance.REPORTS:
        return
    terminalreporter.section("bf16 output errors (plain / floor / relaxed / excess)")
    for test, what, rep in tolerance.REPORTS:
        terminalreporter.write_line("%s [%s] %s" % (test, what, tolerance.fmt_report(rep)))
