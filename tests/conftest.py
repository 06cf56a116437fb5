import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


@pytest.fixture(scope="session", autouse=True)
def _built_libraries():
    """Both native libraries are built (incrementally) before any test."""
    from shared_context_decode_b200 import build as ppbuild
    from oracle import build as obuild
    ppbuild.build()
    obuild.build()
