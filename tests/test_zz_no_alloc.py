"""The allocation-free entry point, sa_append_attend_noalloc.

It serves callers that may not call the CUDA allocator: engines and plugin
hosts that own all device memory through their own pool and do not let a
library allocate, and real-time frame loops that cannot afford a
cudaMalloc/cudaFree (either may synchronise the whole device and miss the
frame deadline). They pass the cache memory themselves and the library uses
a fixed 16 MiB static device scratch instead of allocating a workspace.

These tests stream chunks through it on consecutive calls, past the point
where the ring evicts its oldest frames, and check:
  * every output row of every active stream against the fp64 oracle, within
    the tolerance of the parity tests (bf16 and fp32);
  * the caller-owned K'/V cache of every stream against the oracle's cache
    contents (V bit-exact, K' within one storage ulp plus the fp32 rotation
    term: no refresh exists on this path, so every key is rounded once);
  * the outputs and caches against the handle entry sa_append_attend;
  * the device status word after every call.
The file sorts last so that a failure here comes after every other test."""
import ctypes

import numpy as np
import pytest
import torch

from inputgen.workloads import P512, Workload
from rolling_kv_cache_sa_b200 import (SACache, config_for, sa_append_attend_noalloc,
                                      sa_noalloc_device_status)
from rolling_kv_cache_sa_b200._lib import SA_ERR_UNSUPPORTED

import inputgen as IG
from gpu_harness import assert_cache, assert_rows, sample_tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")


class _CallerCache:
    """Caller-owned cache memory and stream state for the allocation-free
    entry, with the views the cache checks of the parity harness read."""

    def __init__(self, w):
        self.w = w
        dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        ntok = (w.S + w.R) * w.F
        self.k_cache = torch.zeros((w.B, w.H, ntok, w.D), dtype=dt, device="cuda")
        self.v_cache = torch.zeros_like(self.k_cache)
        self.k_raw = (torch.zeros((w.B, w.H, w.S * w.F, w.D), dtype=dt, device="cuda")
                      if w.S > 0 else None)
        self.frames_written = (ctypes.c_int64 * w.B)(*([0] * w.B))
        self.pos_base = (ctypes.c_int64 * w.B)(*([0] * w.B))
        self.scales = np.ones((3, w.H))
        self.cache = self  # assert_cache reads runner.cache.copy_out / state

    def state(self, b):
        return self.frames_written[b], self.pos_base[b]

    def copy_out(self, b):
        torch.cuda.synchronize()
        return self.k_cache[b].float().cpu().numpy(), self.v_cache[b].float().cpu().numpy()

    def call(self, cfg, q, k, v, out, active):
        sa_append_attend_noalloc(cfg, self.k_cache, self.v_cache, self.k_raw,
                                 self.frames_written, self.pos_base, q, k, v, out, active)
        sa_noalloc_device_status()  # raises if a bounded wait gave up


def _stream(w, check_every_row, handle=None, n_chunks=None):
    cfg = config_for(w)
    caller = _CallerCache(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    shape = (w.B, w.Lc, w.H, w.D)
    q = torch.empty(shape, dtype=dt, device="cuda")
    k, v = torch.empty_like(q), torch.empty_like(q)
    out_na = torch.full(shape, 7.0, dtype=dt, device="cuda")
    out_ref = torch.zeros_like(q)
    st = torch.cuda.current_stream().cuda_stream
    worst = 0.0
    for g in range(n_chunks if n_chunks is not None else w.n_steps):
        chunks = w.local_chunks(g)
        active = [c >= 0 for c in chunks]
        if not any(active):
            continue
        for t, buf in ((IG.Q, q), (IG.K, k), (IG.V, v)):
            IG.fill_device(w, list(range(w.B)), chunks, t, buf.data_ptr(), st)
        before = out_na.clone()
        fw_before = list(caller.frames_written)
        caller.call(cfg, q, k, v, out_na, active)
        if handle is not None:
            handle.append_attend(q, k, v, out_ref, active)
        torch.cuda.synchronize()
        got = out_na.float().cpu()
        for b, c in enumerate(chunks):
            if c < 0:
                # an inactive stream's rows are left as they were
                assert torch.equal(out_na[b], before[b]), (b, g)
                assert caller.frames_written[b] == fw_before[b], (b, g)
                continue
            assert caller.frames_written[b] == (c + 1) * w.C
            toks = list(range(w.Lc)) if check_every_row else sample_tokens(w, n_random=6)
            heads = None if check_every_row else [0, w.H // 2, w.H - 1]
            mx, _ = assert_rows(w, b, c, got[b], toks, heads)
            worst = max(worst, mx)
            assert_cache(w, caller, b, c)
        if handle is not None:
            err = (out_na.float() - out_ref.float()).abs()
            assert float(err.max()) <= 2e-2 and float(err.mean()) <= 2e-3, (g, float(err.max()))
            for b in range(w.B):
                kh, vh = handle.copy_out(b)
                kn, vn = caller.copy_out(b)
                np.testing.assert_array_equal(vn, vh)
                # the spatial RoPE tables are built on the device here and on
                # the host for a handle: one storage rounding apart at most
                ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(kh), 2.0 ** -126))) - 7)
                assert (np.abs(kn - kh) <= ulp + np.abs(kh).max(-1, keepdims=True) * 2.0 ** -21
                        ).all(), (g, b)
    return worst


def test_noalloc_512p_consecutive_calls_past_eviction_vs_oracle_and_handle():
    # 512p stream shape, 6 consecutive calls: the ring (W + C = 6 frames = 3
    # chunks) wraps at the 4th call, so eviction and slot reuse are covered;
    # no refresh falls in this range (every 32 chunks)
    w = P512.with_(n_chunks=6, refresh_period=0)
    handle = SACache(config_for(w))
    try:
        _stream(w, check_every_row=False, handle=handle)
    finally:
        handle.close()


def test_noalloc_ragged_streams_every_row_vs_oracle_bf16():
    # three streams starting at different steps (ragged fill, inactive
    # streams on the first calls), ragged last query tile (160 rows), ring
    # wrap after 3 calls; every output row and every cache row checked
    w = Workload("noalloc_ragged_bf16", B=3, H=2, D=128, fh=8, fw=20, C=1, S=1, W=2, n_chunks=6,
                 dtype="bf16", starts=(0, 1, 3))
    _stream(w, check_every_row=True)


def test_noalloc_every_row_vs_oracle_fp32():
    w = Workload("noalloc_fp32", B=2, H=2, D=64, fh=8, fw=8, C=1, S=1, W=2, n_chunks=6,
                 dtype="f32", starts=(0, 2))
    _stream(w, check_every_row=True)


def test_noalloc_rejects_configurations_beyond_the_scratch():
    w = P512.with_(B=2)  # rotated queries alone need 25 MB > 16 MiB
    cfg = config_for(w)
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    fw = (ctypes.c_int64 * 2)(0, 0)
    pb = (ctypes.c_int64 * 2)(0, 0)
    from rolling_kv_cache_sa_b200 import lib
    st = lib().sa_append_attend_noalloc(ctypes.byref(cfg), dummy.data_ptr(), dummy.data_ptr(),
                                        dummy.data_ptr(), fw, pb, dummy.data_ptr(),
                                        dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
                                        None, None)
    assert st == SA_ERR_UNSUPPORTED
    assert b"scratch" in lib().sa_last_error_string()
    assert list(fw) == [0, 0]


def test_noalloc_binding_refuses_wrong_buffers_before_the_call():
    # the C side cannot see buffer sizes; the binding checks them first
    w = Workload("noalloc_small", B=2, H=2, D=128, fh=8, fw=8, C=1, S=1, W=2, n_chunks=2,
                 dtype="bf16")
    cfg = config_for(w)
    caller = _CallerCache(w)
    q = torch.zeros((w.B, w.Lc, w.H, w.D), dtype=torch.bfloat16, device="cuda")
    short = torch.zeros((w.B, w.H, w.R * w.F, w.D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="k_cache"):  # cache sized without the sink rows
        sa_append_attend_noalloc(cfg, short, caller.v_cache, caller.k_raw, caller.frames_written,
                                 caller.pos_base, q, q, q, q)
    with pytest.raises(ValueError, match="q must"):  # fp32 tensors for a bf16 configuration
        sa_append_attend_noalloc(cfg, caller.k_cache, caller.v_cache, caller.k_raw,
                                 caller.frames_written, caller.pos_base, q.float(), q, q, q)
    with pytest.raises(ValueError, match="k_raw"):
        sa_append_attend_noalloc(cfg, caller.k_cache, caller.v_cache, None,
                                 caller.frames_written, caller.pos_base, q, q, q, q)
    assert list(caller.frames_written) == [0, 0]
