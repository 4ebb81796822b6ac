import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _library_build_module():
    """ragged_reduce_b200/build.py, loaded without importing the package (the
    package loads the library this may rebuild)."""
    import importlib.util

    path = os.path.join(ROOT, "ragged_reduce_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_h3rr_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # Test the library built from the sources in the tree: rebuild when the
    # recorded source digest differs (or the library is missing).
    build = _library_build_module()
    if build.is_stale():
        build.build()


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.load()
