"""Shared pytest configuration.

Markers:
  gpu -- needs a CUDA device (B200, sm_100a) and the built CUDA library; these
         are the parity tests of the CUDA path against the CPU oracle.
Everything unmarked runs on a CPU-only machine.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU and the built CUDA library")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle
