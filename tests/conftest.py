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
