import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _ensure_library():
    """Builds libwkv7.so in-tree when it is missing or older than its sources.
    The build script is loaded by path because importing the package loads the
    library (and fails loudly while it does not exist)."""
    import importlib.util

    path = os.path.join(ROOT, "linear_recurrent_lm_wkv7_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_wkv7_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


def pytest_configure(config):
    _ensure_library()
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle
