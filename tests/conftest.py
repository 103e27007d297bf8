import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _load_build_module():
    """Import the build script by path, without importing the package (which
    needs the built library)."""
    path = os.path.join(ROOT, "exact_attention_156_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_attn156_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_sessionstart(session):
    # (Re)build the libraries if a source is newer than the built .so files.
    _load_build_module().build()
