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
    import oracle as _oracle
    _oracle.build()
    mutant = os.environ.get("SSD_ORACLE_MUTANT_LIB")
    if mutant:  # set only by tests/test_oracle_mutations.py for its child runs
        _oracle.use_library(_oracle.bind(mutant))
    return _oracle


def pytest_terminal_summary(terminalreporter):
    """Print the error figures tests recorded with record_property (the parity
    metric and the elementwise diagnostic), one line per test."""
    rows = []
    for rep in terminalreporter.stats.get("passed", []):
        props = [(k, v) for k, v in getattr(rep, "user_properties", []) if isinstance(v, float)]
        if props and rep.when == "call":
            rows.append(rep.nodeid.split("::")[-1] + "  " +
                        "  ".join(f"{k}={v:.3g}" for k, v in props))
    if rows:
        terminalreporter.write_sep("-", "recorded errors")
        for r in rows:
            terminalreporter.write_line(r)
