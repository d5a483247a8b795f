import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


# Planted oracle slips (tests/test_oracle_mutants.py runs the pins in a
# subprocess with this variable set; it is never set otherwise).
if os.environ.get("SFX_ORACLE_MUTANT"):
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    import oracle_mutants

    oracle_mutants.apply(os.environ["SFX_ORACLE_MUTANT"])
