"""The debug build (libsa_debug.so): every kernel range-checks the buffer
indexes it computes (cache rows, raw-sink rows, refresh rows, query and
key/value tile coordinates, partial-result slots and arrival counters of
split attention units, GDN workspace blocks and state slices) and records a
failed check in a device word instead of faulting. With compute-sanitizer
closed on this pool, this is the in-kernel evidence that the indexes stay in
bounds.

Each test runs in a child process with SA_LIBRARY_VARIANT=debug (the library
is loaded once per process):
  * the recording path works: a kernel that fails a check on purpose without
    touching memory is reported, and reading the words clears them;
  * the small-case GPU parity tests pass under the debug build with every
    index check holding after every test (tests/conftest.py reads the words),
    covering ragged tails, split attention units (the 512p stream and the
    split-unit case below), refreshes, sink updates, uncommitted steps, the
    e4m3 cache, the allocation-free entry and the GDN block."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")


def _child_env():
    env = dict(os.environ)
    env["SA_LIBRARY_VARIANT"] = "debug"
    return env


def test_debug_build_records_and_clears_a_failed_check():
    code = r"""
import sys
sys.path.insert(0, %r)
from rolling_kv_cache_sa_b200 import _lib
L = _lib.lib()
assert _lib.LIB_PATH.endswith("libsa_debug.so"), _lib.LIB_PATH
assert L.sa_debug_bounds_status(None) == _lib.SA_OK
assert L.sa_debug_bounds_selftest(None) == _lib.SA_OK
st = L.sa_debug_bounds_status(None)
msg = L.sa_last_error_string().decode()
assert st == _lib.SA_ERR_DEVICE_BOUNDS, (st, msg)
assert "attend_tc sites 0x80000000" in msg, msg
assert L.sa_debug_bounds_status(None) == _lib.SA_OK   # read clears
print("debug bounds ok")
""" % ROOT
    r = subprocess.run([sys.executable, "-c", code], env=_child_env(), capture_output=True,
                       text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug bounds ok" in r.stdout


SUBSET = ("tiny_fp32_every or edge_cases or fp32_d128 or inactive or 512p_full or split_units "
          "or gdn_small or gdn_token or gdn_special or sink_update_and or uncommitted_steps "
          "or e4m3_small or e4m3_sink or noalloc_ragged or noalloc_every_row")


def test_small_parity_suite_under_the_debug_build():
    files = ["tests/test_gpu_parity.py", "tests/test_gpu_gdn.py", "tests/test_gpu_sink.py",
             "tests/test_gpu_uncommitted.py", "tests/test_gpu_fp8.py", "tests/test_zz_no_alloc.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p",
                        "no:cacheprovider", "-k", SUBSET, *files],
                       env=_child_env(), capture_output=True, text=True, timeout=1200, cwd=ROOT)
    tail = r.stdout[-3000:] + r.stderr[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail
