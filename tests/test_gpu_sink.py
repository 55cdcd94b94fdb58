"""Adaptive sink update and the re-pinned sink (StreamDiffusionV2, section
2.A.2) on the GPU against the oracle: two streams at different fill levels,
RoPE refreshes, a half-weight sink update every 4 chunks, both sink position
modes; every output row per chunk and the cache after each chunk."""
import pytest
import torch

import inputgen as IG
from gpu_harness import Runner, assert_cache, assert_rows
from inputgen.workloads import Workload
from rolling_kv_cache_sa_b200._lib import SA_ERR_INVALID_ARG, SA_ERR_STATE, SA_SINK_REPIN, \
    SA_SINK_SHIFT, SAError

pytestmark = pytest.mark.gpu

SINK_BF16 = Workload("sink_update_bf16_8x12", B=2, H=4, D=128, fh=8, fw=12, C=1, S=2, W=3,
                     n_chunks=10, dtype="bf16", refresh_period=3, starts=(0, 2),
                     sink_update_period=4, sink_alpha=0.5)
SINK_F32 = Workload("sink_update_f32_8x8", B=1, H=2, D=64, fh=8, fw=8, C=2, S=1, W=2,
                    n_chunks=9, dtype="f32", refresh_period=2, sink_update_period=3,
                    sink_alpha=1.0)


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")


def _update_due(w, c):
    return c > 0 and c % w.sink_update_period == 0 and c * w.C >= w.S


SINK_E4M3 = SINK_BF16.with_(name="sink_update_e4m3_8x12", cache="e4m3")


@pytest.mark.parametrize("repin", [False, True], ids=["shift", "repin"])
@pytest.mark.parametrize("w0", [SINK_BF16, SINK_F32, SINK_E4M3], ids=lambda w: w.name)
def test_sink_update_and_modes_match_oracle(w0, repin):
    w = w0.with_(sink_repin=repin)
    r = Runner(w)
    r.cache.set_sink_mode(SA_SINK_REPIN if repin else SA_SINK_SHIFT)
    shape = (w.B, w.S * w.F, w.H, w.D)
    kn = torch.empty(shape, dtype=r.q.dtype, device="cuda")
    vn = torch.empty_like(kn)
    st = torch.cuda.current_stream().cuda_stream
    toks = list(range(w.Lc))
    n_upd = 0
    try:
        for g in range(w.n_steps):
            chunks = w.local_chunks(g)
            upd = [c >= 0 and _update_due(w, c) for c in chunks]
            if any(upd):
                coords = [IG.sink_update_chunk(c) if u else -1 for c, u in zip(chunks, upd)]
                IG.fill_device(w, list(range(w.B)), coords, IG.K, kn.data_ptr(), st, n_tok=w.S * w.F)
                IG.fill_device(w, list(range(w.B)), coords, IG.V, vn.data_ptr(), st, n_tok=w.S * w.F)
                r.cache.sink_update(kn, vn, w.sink_alpha, upd)
                n_upd += sum(upd)
            r.step(g)
            torch.cuda.synchronize()
            out = r.out.float().cpu()
            for b, c in enumerate(chunks):
                if c < 0:
                    continue
                assert_rows(w, b, c, out[b], toks)
                assert_cache(w, r, b, c, sink_ulps=1 if w.dtype == "bf16" else 0)
        assert n_upd >= 2
        assert r.device_status() == 0
    finally:
        r.close()


def test_sink_update_refusals():
    w = SINK_BF16
    r = Runner(w)
    try:
        kn = torch.zeros((w.B, w.S * w.F, w.H, w.D), dtype=r.q.dtype, device="cuda")
        with pytest.raises(SAError) as e:  # sink not complete: nothing written yet
            r.cache.sink_update(kn, kn, 1.0)
        assert e.value.status == SA_ERR_STATE
        for g in range(4):
            r.step(g)
        with pytest.raises(SAError) as e:
            r.cache.sink_update(kn, kn, 1.5)
        assert e.value.status == SA_ERR_INVALID_ARG
        with pytest.raises(SAError) as e:
            r.cache.set_sink_mode(7)
        assert e.value.status == SA_ERR_INVALID_ARG
    finally:
        r.close()
