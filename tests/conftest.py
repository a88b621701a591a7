import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")
    # Test modules import the binding, which loads libpa.so: make sure it is
    # built (nvcc cross-compiles for sm_100a without a GPU). build.py is loaded
    # by path because importing the package would load the library first.
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "pa_build", os.path.join(ROOT, "paged_kv_cache_475_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
