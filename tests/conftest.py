import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # The library is built in-tree; (re)build it when a source is newer than
    # it.  build.py is loaded by path: importing the package would load the
    # library before it exists.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_inkling_moe_build", os.path.join(ROOT, "mixture_experts_feed_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
