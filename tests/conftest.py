import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library's Python binding (only for tests marked gpu)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_int4_a16w4_b200 as w4
    return w4


def build_library():
    """Build (or refresh) the in-tree library without importing the package,
    which would load a stale library first."""
    import importlib.util
    path = os.path.join(ROOT, "weight_only_int4_a16w4_b200", "build.py")
    spec = importlib.util.spec_from_file_location("w4a16_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()
