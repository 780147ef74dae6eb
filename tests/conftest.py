import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def build_library() -> str:
    """Build librope_store.so if it is missing or stale (rope_paged_kv_b200/build.py, loaded
    from its file: importing the package needs the library) and return its path."""
    import importlib.util
    path = os.path.join(ROOT, "rope_paged_kv_b200", "build.py")
    spec = importlib.util.spec_from_file_location("rope_paged_kv_b200_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="session", autouse=True)
def _built_oracle():
    from oracle import build as ob
    ob.build()
