"""Shared pytest setup: the `gpu` marker and on-demand builds of the small C libraries."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def build_cuda_library():
    """Build libvtattn.so if stale (nvcc cross-compiles without a GPU); loads build.py by
    path because importing the package loads the library."""
    import importlib.util
    path = os.path.join(ROOT, "flash_attention_varlen_b200", "build.py")
    spec = importlib.util.spec_from_file_location("vt_attn_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="session", autouse=True)
def _c_libs_built():
    import oracle
    import workloads
    oracle.build()
    workloads.build()
    build_cuda_library()
    yield
