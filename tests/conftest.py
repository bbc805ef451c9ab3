import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes of oracle time)")


def build_cuda_library() -> str:
    """Build libw8a8.so (by file path: importing the package needs the .so)."""
    import importlib.util
    path = os.path.join(ROOT, "w8a8_linear_layers_b200", "build.py")
    spec = importlib.util.spec_from_file_location("w8a8_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle
