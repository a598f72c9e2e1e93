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
    # The library is built in-tree; build it once if this checkout has none.
    lib = os.path.join(ROOT, "mixture_experts_feed_b200", "libinklingmoe.so")
    if not os.path.exists(lib):
        from mixture_experts_feed_b200.build import build
        build()
