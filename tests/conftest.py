import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    # Rebuild libqk.so when a CUDA source is newer than it (no-op otherwise),
    # so no test runs against a library built from older sources.
    from block_quantized_expert_mxfp4_b200 import build

    build.build()


def golden(name):
    return os.path.join(ROOT, "tests", "golden", name)
