import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large CPU work (oracle at full size)")
    # The binding loads libsalad.so at import; build it first if it is stale.
    from sparse_linear_hybrid_top_b200 import build as _build
    _build.build()
