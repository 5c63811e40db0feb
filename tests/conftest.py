import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_library():
    """Compile librq.so in-tree when missing or older than its sources (the
    package loads it at import and has no fallback)."""
    import importlib.util
    path = os.path.join(ROOT, "decode_attention_14_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_rq_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


_build_library()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(autouse=True)
def _guard_bands(request):
    """After every GPU test: the guard bands around the harness's cache arenas
    and decode outputs are intact."""
    yield
    if request.node.get_closest_marker("gpu") is not None:
        import rqharness
        rqharness.check_guards()
