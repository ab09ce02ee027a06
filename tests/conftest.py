import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: larger CPU cases")
    mutant = os.environ.get("FT_ORACLE_MUTANT")
    if mutant:  # a child run of test_oracle_mutants.py: plant one mistake in the oracle
        sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
        import _oracle_mutants
        _oracle_mutants.apply(mutant)


@pytest.fixture(scope="session")
def has_gpu():
    import torch
    return torch.cuda.is_available()
