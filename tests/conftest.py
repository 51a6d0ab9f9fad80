import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def splitkv():
    """The Python binding with libsplitkv.so built in-tree (nvcc cross-compiles; no GPU needed)."""
    _build = load_build_module()
    if not os.path.exists(_build.LIB):
        _build.build()
    import context_block_sparse_b200 as skv
    return skv


def load_build_module():
    """context_block_sparse_b200/build.py, loaded by path (importing the package needs the built library)."""
    import importlib.util
    path = os.path.join(ROOT, "context_block_sparse_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_splitkv_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def gpu_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False
