"""Failure detection on the GPU without any fault: a bounded device wait on a
barrier that nothing completes runs out, the host reads SA_ERR_DEVICE_TIMEOUT,
a second waiter leaves through the abort flag, and the CUDA context stays
usable (a cache created afterwards still matches the oracle). Host-injected
failures (SA_FAULT) take the allocation and launch error paths: the status is
reported, nothing changes, and the next call succeeds."""
import pytest
import torch

from gpu_harness import assert_rows
from inputgen.workloads import TINY_F32

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000  # 2 ms


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")


def test_bounded_wait_expires_and_context_survives():
    from rolling_kv_cache_sa_b200 import sa_wait_probe
    from rolling_kv_cache_sa_b200._lib import SA_ERR_DEVICE_TIMEOUT
    from gpu_harness import Runner

    st, waited = sa_wait_probe(LIMIT_NS)
    assert st == SA_ERR_DEVICE_TIMEOUT
    # warp 0 gave up after its own limit (allow scheduling slack)
    assert LIMIT_NS <= waited[0] < LIMIT_NS + 50_000_000
    # warp 1 (limit 40 ms) left through the abort flag, well before its limit
    assert waited[1] < 10 * LIMIT_NS
    assert waited[1] >= waited[0] - 1_000_000

    # the context is intact: a fresh cache still computes the right answer
    w = TINY_F32
    r = Runner(w)
    try:
        for g in range(3):
            chunks, _ = r.step(g)
        torch.cuda.synchronize()
        assert r.cache.device_status() == 0
        out = r.out.float().cpu()
        assert_rows(w, 0, chunks[0], out[0], list(range(w.Lc)))
    finally:
        r.close()


def test_injected_allocation_failure(monkeypatch):
    from rolling_kv_cache_sa_b200 import SACache, SAError, config_for
    from rolling_kv_cache_sa_b200._lib import SA_ERR_OOM
    monkeypatch.setenv("SA_FAULT", "alloc")
    with pytest.raises(SAError) as e:
        SACache(config_for(TINY_F32))
    assert e.value.status == SA_ERR_OOM


def test_injected_launch_failure_leaves_state_and_recovers(monkeypatch):
    from gpu_harness import Runner
    from rolling_kv_cache_sa_b200 import SAError
    from rolling_kv_cache_sa_b200._lib import SA_ERR_CUDA
    monkeypatch.setenv("SA_FAULT", "launch_once")
    w = TINY_F32
    r = Runner(w)
    monkeypatch.delenv("SA_FAULT")
    try:
        with pytest.raises(SAError) as e:
            r.step(0)
        assert e.value.status == SA_ERR_CUDA
        assert r.cache.state(0) == (0, 0)
        for g in range(3):
            chunks, _ = r.step(g)
        torch.cuda.synchronize()
        assert r.cache.state(0)[0] == 3 * w.C
        assert_rows(w, 0, chunks[0], r.out.float().cpu()[0], list(range(w.Lc)))
    finally:
        r.close()
