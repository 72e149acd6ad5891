"""Shared pytest setup: the `gpu` marker and session fixtures.

Tests marked `gpu` need a CUDA device and the built CUDA library; everything else
runs on the CPU (oracle pins, host-side argument checks, symbol exports).
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle

    oracle.build()
    return oracle
