import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session")
def orc():
    """The CPU oracle, on every host thread this process may use (its OpenMP build
    splits independent rows and entries only, so the results are those of the serial
    build)."""
    import oracle
    oracle.build()
    n = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    oracle.set_threads(n)
    return oracle
