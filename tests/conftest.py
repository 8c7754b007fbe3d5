"""Shared test configuration.

``-m gpu`` tests need a B200 and the built CUDA library; everything else runs
on CPU.  The CPU oracle (``oracle/``) is test infrastructure and is imported
only from tests, the smoke check and the benchmark's CPU arms.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an NVIDIA B200 (sm_100a) and the built libtfq.so")
    config.addinivalue_line("markers", "slow: full-size parity cases (minutes)")
