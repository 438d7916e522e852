import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle


def build_library():
    """Builds libbsa.so through the package's build.py loaded by path (importing
    the package would load a possibly stale or missing library first)."""
    import importlib.util

    path = os.path.join(ROOT, "block_sparse_attention_19_b200", "build.py")
    spec = importlib.util.spec_from_file_location("bsa_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="session", autouse=True)
def _library_present():
    """Builds libbsa.so in-tree when it is missing (a GPU-only selection skips
    the CPU tests whose fixture builds it); an existing library is used as is."""
    if not os.path.exists(os.path.join(ROOT, "block_sparse_attention_19_b200", "libbsa.so")):
        build_library()
