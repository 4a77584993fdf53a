import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # Both libraries build in-tree on demand (gcc for the oracle, nvcc for libipe).
    import importlib.util
    from oracle import build as obuild
    obuild.build()
    # by path: importing the package needs the library it would build
    path = os.path.join(ROOT, "interpolated_position_encoding_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_ipe_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.get()
