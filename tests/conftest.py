import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle():
    import oracle as _oracle

    # tests/test_oracle_mutants.py runs the pins against deliberately broken builds of the
    # oracle, compiled elsewhere; this variable names such a library
    mutant = os.environ.get("ORACLE_MUTANT_LIB")
    if mutant:
        _oracle._LIB = mutant
        _oracle._lib = None
    _oracle.build()
    return _oracle
