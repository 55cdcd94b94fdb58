"""Attention of a chunk without committing it (sa_attend): the non-final
denoising steps of a chunk. Each uncommitted step is compared with the oracle's
uncommitted-chunk attention (context from the stream's own draw, the chunk's
queries, keys and values from the step's draw); the final, committing step
with the oracle's committed path; the cache after each chunk with the oracle's
storage model, so the uncommitted steps leave no trace. Ragged tiles, two
streams at different fill levels, refreshes, bf16 (tcgen05) and fp32 (SIMT)."""
import dataclasses

import numpy as np
import pytest
import torch

import inputgen as IG
import oracle as O
from gpu_harness import (BF16_MAX_ABS, BF16_MEAN_ABS, E4M3_MAX_ABS, E4M3_MEAN_ABS, F32_MAX_ABS,
                         Runner, assert_cache, assert_rows, log_line)
from inputgen import spec_for
from inputgen.workloads import Workload

pytestmark = pytest.mark.gpu

UNC_BF16 = Workload("uncommitted_bf16_8x12", B=2, H=4, D=128, fh=8, fw=12, C=2, S=1, W=4,
                    n_chunks=9, dtype="bf16", refresh_period=4, starts=(0, 3))
UNC_E4M3 = UNC_BF16.with_(name="uncommitted_e4m3_8x12", cache="e4m3",
                          fp8_scales=((1.0, 2.0, 0.5, 4.0), (2.0, 1.0, 4.0, 0.25),
                                      (1.0, 8.0, 0.5, 2.0)))
UNC_F32 = Workload("uncommitted_f32_8x8", B=1, H=2, D=64, fh=8, fw=8, C=1, S=1, W=2,
                   n_chunks=8, dtype="f32", refresh_period=4)


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")


def _fill(r, w_draw, chunks):
    st = torch.cuda.current_stream().cuda_stream
    for t, buf in ((IG.Q, r.q), (IG.K, r.k), (IG.V, r.v)):
        IG.fill_device(w_draw, list(range(r.w.B)), chunks, t, buf.data_ptr(), st)


@pytest.mark.parametrize("w", [UNC_BF16, UNC_F32, UNC_E4M3], ids=lambda w: w.name)
def test_uncommitted_steps_then_commit(w):
    draws = [dataclasses.replace(w, seed=w.seed + 101 + i) for i in range(2)]
    cfg = O.cfg_for(w)
    r = Runner(w)
    toks = list(range(w.Lc))
    tt = np.repeat(np.asarray(toks), w.H)
    hh = np.tile(np.arange(w.H), len(toks))
    try:
        for g in range(w.n_steps):
            chunks = w.local_chunks(g)
            active = [c >= 0 for c in chunks]
            if not any(active):
                continue
            for wd in draws:
                _fill(r, wd, chunks)
                r.sess.step_uncommitted(r.q, r.k, r.v, r.out, active)
                torch.cuda.synchronize()
                out = r.out.float().cpu()
                for b, c in enumerate(chunks):
                    if c < 0:
                        continue
                    assert r.cache.state(b)[0] == c * w.C  # nothing committed
                    ref = O.attend_rows_uncommitted(cfg, spec_for(w), spec_for(wd), b, c, tt, hh)
                    got = out[b][torch.as_tensor(tt), torch.as_tensor(hh)].double().numpy()
                    err = np.abs(got - ref)
                    log_line(f"{w.name} uncommitted stream {b} chunk {c}: max_abs {err.max():.3e} "
                             f"mean_abs {err.mean():.3e}")
                    if w.cache == "e4m3":
                        assert err.max() <= E4M3_MAX_ABS and err.mean() <= E4M3_MEAN_ABS, (b, c)
                    elif w.dtype == "bf16":
                        assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS, (b, c)
                    else:
                        assert err.max() <= F32_MAX_ABS, (b, c, err.max())
            # the final step commits the stream's own draw
            r.step(g)
            torch.cuda.synchronize()
            out = r.out.float().cpu()
            for b, c in enumerate(chunks):
                if c < 0:
                    continue
                assert_rows(w, b, c, out[b], toks)
                assert_cache(w, r, b, c)
        assert r.device_status() == 0
    finally:
        r.close()


def test_uncommitted_step_with_final_inputs_equals_commit():
    """An uncommitted step on the inputs the commit then uses gives the
    commit's output bit for bit (same rows written, same context)."""
    w = UNC_BF16
    r = Runner(w)
    try:
        for g in range(6):
            chunks = w.local_chunks(g)
            active = [c >= 0 for c in chunks]
            _fill(r, w, chunks)
            r.sess.step_uncommitted(r.q, r.k, r.v, r.out, active)
            torch.cuda.synchronize()
            first = r.out.clone()
            r.sess.step(r.q, r.k, r.v, r.out, active)
            torch.cuda.synchronize()
            for b, c in enumerate(chunks):
                if c >= 0:
                    assert torch.equal(first[b], r.out[b]), (g, b)
    finally:
        r.close()
