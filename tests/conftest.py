import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


def _stale(out, srcs):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in srcs)


def _ensure_built():
    """Builds any missing or stale library (the driver's build() normally did it)."""
    from oracle import build as ob
    from inputgen import build as ib
    if _stale(os.path.join(ROOT, "oracle", "liboracle.so"),
              [os.path.join(ROOT, "oracle", f) for f in ("oracle.c", "oracle.h")] +
              [os.path.join(ROOT, "inputgen", "sa_inputgen.h")]):
        ob.build()
    if _stale(os.path.join(ROOT, "inputgen", "libsa_inputgen.so"),
              [os.path.join(ROOT, "inputgen", f) for f in ("inputgen.cu", "sa_inputgen.h")]):
        ib.build()
    try:
        from rolling_kv_cache_sa_b200 import build as pb
    except ImportError:
        return
    if pb.is_stale():
        pb.build()


_ensure_built()


@pytest.fixture(scope="session")
def has_gpu():
    import torch
    return torch.cuda.is_available()


@pytest.fixture(autouse=True)
def _debug_bounds_words(request):
    """Under the debug build (SA_LIBRARY_VARIANT=debug), every GPU test ends by
    reading the kernels' index-check words: a failed check fails the test."""
    yield
    if os.environ.get("SA_LIBRARY_VARIANT") != "debug" or request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from rolling_kv_cache_sa_b200 import _lib
    st = _lib.lib().sa_debug_bounds_status(None)
    assert st == _lib.SA_OK, _lib.lib().sa_last_error_string().decode()
