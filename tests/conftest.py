"""Shared test configuration.

Markers: ``gpu`` tests need a CUDA device (a B200) and the built library; all
other tests run on the CPU.  The oracle under ``oracle/`` is imported only by
tests (and by the benchmark's CPU-baseline leg).
"""
import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and libw4a.so")
    config.addinivalue_line("markers", "slow: long-running (full-size) case")


@pytest.fixture(scope="session")
def built_lib():
    """Build libw4a.so if it is missing or stale (nvcc cross-compiles on a host)."""
    from w4_weight_only_b200 import build
    return build.build()


@pytest.fixture(scope="session")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("gpu test selected but no CUDA device is visible")
    return torch.device("cuda:0")
