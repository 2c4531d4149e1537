"""Shared pytest configuration.

Markers:
  gpu -- needs a CUDA device; these are the parity tests proper, calling the
         CUDA library through its C ABI.  Everything else runs on the CPU.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (parity tests through the C ABI)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle
