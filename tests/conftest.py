import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


def pytest_sessionstart(session):
    """Build libkronq.so in-tree when it is absent (a fresh checkout): the CPU
    tests load it for its exports and host-side checks."""
    lib = os.path.join(ROOT, "post_weight_quantization_syrk_b200", "libkronq.so")
    if not os.path.exists(lib):
        from post_weight_quantization_syrk_b200 import build
        build.build()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
