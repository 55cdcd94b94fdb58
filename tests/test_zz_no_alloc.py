"""The allocation-free entry point, sa_append_attend_noalloc.

It serves callers that may not call the CUDA allocator (engines and plugin
hosts that own all device memory through their own pool, real-time frame
loops that cannot afford a device-synchronising cudaMalloc/cudaFree): they
pass the cache memory themselves and the library uses a fixed 16 MiB static
device scratch instead of allocating a workspace. This test streams the same
chunks through it and through the handle-based sa_append_attend and checks
the outputs agree within the bf16 tolerance used by the parity tests, on
consecutive calls. The file sorts last so that a failure here comes after
every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

import inputgen as IG
from inputgen.workloads import P512
from rolling_kv_cache_sa_b200 import (SACache, SAError, config_for, sa_append_attend_noalloc)
from rolling_kv_cache_sa_b200._lib import SA_ERR_UNSUPPORTED

pytestmark = pytest.mark.gpu

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")


def test_noalloc_matches_handle_entry_on_consecutive_calls():
    w = P512
    cfg = config_for(w)
    cache = SACache(cfg)
    shape = (w.B, w.Lc, w.H, w.D)
    q = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    k, v = torch.empty_like(q), torch.empty_like(q)
    out_ref, out_na = torch.zeros_like(q), torch.zeros_like(q)
    ntok = (w.S + w.R) * w.F
    # caller-owned cache memory for the allocation-free entry point
    k_cache = torch.zeros((w.B, w.H, ntok, w.D), dtype=torch.bfloat16, device="cuda")
    v_cache = torch.zeros_like(k_cache)
    k_raw = torch.zeros((w.B, w.H, w.S * w.F, w.D), dtype=torch.bfloat16, device="cuda")
    frames_written = (ctypes.c_int64 * w.B)(*([0] * w.B))
    pos_base = (ctypes.c_int64 * w.B)(*([0] * w.B))
    st = torch.cuda.current_stream().cuda_stream
    try:
        for c in range(4):  # consecutive calls: sink + growing window + steady state
            for t, buf in ((IG.Q, q), (IG.K, k), (IG.V, v)):
                IG.fill_device(w, list(range(w.B)), [c] * w.B, t, buf.data_ptr(), st)
            cache.append_attend(q, k, v, out_ref)
            sa_append_attend_noalloc(cfg, k_cache, v_cache, k_raw, frames_written, pos_base,
                                     q, k, v, out_na)
            torch.cuda.synchronize()
            assert list(frames_written) == [(c + 1) * w.C] * w.B
            err = (out_na.float() - out_ref.float()).abs()
            assert torch.isfinite(out_na.float()).all()
            assert float(err.max()) <= BF16_MAX_ABS, (c, float(err.max()))
            assert float(err.mean()) <= BF16_MEAN_ABS, (c, float(err.mean()))
            k_ref, v_ref = cache.copy_out(0)
            np.testing.assert_array_equal(
                (v_cache[0].view(torch.int16).cpu().numpy().astype(np.uint16).astype(np.uint32)
                 << 16).view(np.float32), v_ref)
    finally:
        cache.close()


def test_noalloc_rejects_configurations_beyond_the_scratch():
    w = P512.with_(B=2)  # rotated queries alone need 25 MB > 16 MiB
    cfg = config_for(w)
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    fw = (ctypes.c_int64 * 2)(0, 0)
    pb = (ctypes.c_int64 * 2)(0, 0)
    with pytest.raises(SAError) as e:
        sa_append_attend_noalloc(cfg, dummy, dummy, dummy, fw, pb, dummy, dummy, dummy, dummy)
    assert e.value.status == SA_ERR_UNSUPPORTED
    assert "scratch" in str(e.value)
    assert list(fw) == [0, 0]
