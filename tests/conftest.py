import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_sessionstart(session):
    """Bring libgqa.so up to date before any test imports the package."""
    import importlib.util
    import shutil
    path = os.path.join(ROOT, "grouped_query_softmax_b200", "_build.py")
    spec = importlib.util.spec_from_file_location("gqa_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    if mod.stale() and (shutil.which("nvcc") or os.path.exists(mod.NVCC)):
        mod.build()
