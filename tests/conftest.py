import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_sessionstart(session):
    """Build libtps.so in-tree if it is missing (fresh checkout): the host and GPU
    tests call the library through its C ABI. The build script is loaded by path
    so that the package (which loads the library) is not imported first."""
    lib = os.path.join(ROOT, "tensor_sharded_linear_columnparallel_b200", "libtps.so")
    if os.path.exists(lib):
        return
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "tps_build", os.path.join(ROOT, "tensor_sharded_linear_columnparallel_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
