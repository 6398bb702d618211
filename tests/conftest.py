import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")
    _build_library_if_missing()


def _build_library_if_missing():
    """A fresh checkout has no libbq.so (built files are not committed):
    compile it with the package's own build script before any test imports
    the package. nvcc cross-compiles for sm_100a without a GPU."""
    import importlib.util
    pkg = os.path.join(ROOT, "dequantize_absmax_reduce_b200")
    if os.path.exists(os.path.join(pkg, "libbq.so")):
        return
    spec = importlib.util.spec_from_file_location("_bq_build", os.path.join(pkg, "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(autouse=True)
def _no_abandoned_waits(request):
    """After every GPU test: no kernel took its bounded-wait exit (which
    returns without finishing its work)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import dequantize_absmax_reduce_b200 as m
    st = m._bq.bq_check_device_error()
    assert st == m._bq.BQ_OK, f"device error flag after the test: {m._bq.bq_status_string(st)}"
