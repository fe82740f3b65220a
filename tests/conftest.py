"""Shared pytest configuration.

Markers:
  gpu  -- needs a CUDA device (a B200); run with ``-m gpu``.  Everything else
          runs on a CPU-only machine with ``-m "not gpu"``.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: test needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case, minutes of CPU time")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle
