"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, at the full workload sizes (sampled rows) and on small
edge cases (every row). Tolerances: fp32 max abs 1e-4; bf16 max abs 2e-2 and
mean abs 2e-3; cache indexing (V bytes, slot map, metadata) bit-exact; rotated
keys within the storage rounding (see gpu_harness.assert_cache)."""
import numpy as np
import pytest
import torch

from gpu_harness import Runner, assert_cache, assert_rows, sample_tokens
from inputgen.workloads import (BATCHED_480, LONG_STRESS, P512, SANA_1280, TINY_F32, Workload,
                                NORMAL, UNIFORM)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")


def _run(w, checks, rows=None, cache_checks=(), n_steps=None, heads=None):
    """Streams w; at each global step in `checks` compares every active
    stream's sampled rows (or all rows when rows == 'all')."""
    r = Runner(w)
    worst = (0.0, 0.0)
    try:
        steps = w.n_steps if n_steps is None else n_steps
        for g in range(steps):
            chunks, active = r.step(g)
            if g in checks:
                torch.cuda.synchronize()
                out = r.out.float().cpu()
                for b, c in enumerate(chunks):
                    if c < 0:
                        continue
                    toks = list(range(w.Lc)) if rows == "all" else sample_tokens(w, seed=g * 31 + b)
                    mx, mean = assert_rows(w, b, c, out[b], toks, heads)
                    worst = (max(worst[0], mx), max(worst[1], mean))
            if g in cache_checks:
                torch.cuda.synchronize()
                for b, c in enumerate(chunks):
                    if c >= 0:
                        assert_cache(w, r, b, c)
        assert r.device_status() == 0
    finally:
        r.close()
    return worst


def test_tiny_fp32_every_chunk_every_row():
    steps = set(range(TINY_F32.n_steps))
    _run(TINY_F32, steps, rows="all", cache_checks=steps)


def test_tiny_fp32_alternative_rope_split():
    w = TINY_F32.with_(rope_dims=(22, 22, 20))
    steps = set(range(w.n_steps))
    _run(w, steps, rows="all", cache_checks={0, 3, 4, 7})


def test_512p_full_stream():
    w = P512
    _run(w, {0, 1, 2, 3, 31, 32, 33, 63}, cache_checks={0, 2, 32, 63})


def test_480x832_ragged_batched_streams():
    w = BATCHED_480
    _run(w, {0, 3, 7, 12, 13, 40, 127, 130, 139}, cache_checks={12, 139}, heads=[0, 5, 11])


def test_1280x704_sink_plus_window():
    w = SANA_1280
    _run(w, {0, 1, 2, 3, 4, 128, 255}, cache_checks={3, 255}, heads=[0, 7, 15])


def test_long_stress_10000_chunks():
    w = LONG_STRESS
    # stream 0 at chunks 0, 255, 256 (first refresh), 5000, 9984 (last refresh), 9999 (last)
    checks = {0, 255, 256, 5000, 9984, 9999, w.n_steps - 1}
    _run(w, checks, cache_checks={256, 9999}, heads=[0, 9, 15])


@pytest.mark.parametrize("name,kw", [
    ("window0", dict(W=0)),
    ("sink_eq_chunk", dict(S=2, C=2, W=2)),
    ("no_sink", dict(S=0, W=3)),
    ("sink_gt_chunk", dict(S=3, C=2, W=2)),
    ("d64", dict(D=64)),
    ("odd_frame_tails", dict(fh=5, fw=7, C=3, S=1, W=3)),
    ("single_partial_tile", dict(fh=4, fw=5, C=1, S=1, W=1)),
    # 64 streams (the handle's maximum), ragged: several append and refresh
    # launches per call, stream-K units spanning many streams
    ("max_streams_64", dict(B=64, H=2, fh=4, fw=8, C=1, S=1, W=2, n_chunks=6,
                            starts=tuple(i % 5 for i in range(64)))),
    ("multi_frame_chunk", dict(C=4, S=2, W=4, fh=8, fw=8)),
    ("many_heads", dict(H=32, fh=8, fw=8)),
])
def test_bf16_edge_cases_every_row(name, kw):
    base = Workload("edge_" + name, B=2, H=3, D=128, fh=16, fw=12, C=1, S=1, W=2, n_chunks=9,
                    dtype="bf16", refresh_period=3, starts=(0, 2))
    w = base.with_(**kw)
    steps = set(range(w.n_steps))
    _run(w, steps, rows="all", cache_checks=steps)


def test_split_units_every_row():
    # 2 streams x 8 heads x 2 query-tile pairs = 32 units of up to 14 key tiles
    # (448 >= the SM count): the persistent attention kernel splits units
    # between CTAs and merges their partial results; every row is checked,
    # across ring wrap, refreshes and a ragged start
    w = Workload("split_units", B=2, H=8, D=128, fh=16, fw=16, C=2, S=1, W=4, n_chunks=5,
                 dtype="bf16", refresh_period=3, starts=(0, 1))
    steps = set(range(w.n_steps))
    _run(w, steps, rows="all", cache_checks={1, 3, 5})


def test_fp32_d128():
    w = Workload("fp32_d128", B=2, H=2, D=128, fh=6, fw=10, C=2, S=1, W=4, n_chunks=7,
                 dtype="f32", refresh_period=3, starts=(0, 1), dist=(NORMAL, NORMAL, UNIFORM))
    steps = set(range(w.n_steps))
    _run(w, steps, rows="all", cache_checks={0, 3, 7})


def test_inactive_streams_untouched_and_empty_call():
    w = Workload("inactive", B=3, H=2, D=128, fh=8, fw=16, C=1, S=1, W=2, n_chunks=4,
                 dtype="bf16", starts=(0, 2, 100))
    r = Runner(w)
    try:
        sentinel = torch.full_like(r.out, 7.0)
        for g in range(4):
            chunks = w.local_chunks(g)
            active = [c >= 0 for c in chunks]
            r.out.copy_(sentinel)
            r.fill(chunks)
            before = [r.cache.state(b) for b in range(w.B)]
            r.sess.step(r.q, r.k, r.v, r.out, active)
            torch.cuda.synchronize()
            for b, c in enumerate(chunks):
                if c < 0:
                    assert torch.equal(r.out[b], sentinel[b])
                    assert r.cache.state(b) == before[b]
                else:
                    assert r.cache.state(b)[0] == before[b][0] + w.C
        # an all-inactive call changes nothing
        r.out.copy_(sentinel)
        st = [r.cache.state(b) for b in range(w.B)]
        r.cache.append_attend(r.q, r.k, r.v, r.out, [False] * w.B)
        torch.cuda.synchronize()
        assert torch.equal(r.out, sentinel)
        assert [r.cache.state(b) for b in range(w.B)] == st
        assert r.device_status() == 0
    finally:
        r.close()


def test_host_buffer_entry_matches_device_entry():
    w = P512.with_(n_chunks=4)
    a, b = Runner(w), Runner(w)
    try:
        qh = torch.empty(a.q.shape, dtype=a.q.dtype).pin_memory()
        kh, vh = torch.empty_like(qh).pin_memory(), torch.empty_like(qh).pin_memory()
        oh = torch.empty_like(qh).pin_memory()
        for g in range(4):
            chunks, active = a.step(g)
            qh.copy_(a.q)
            kh.copy_(a.k)
            vh.copy_(a.v)
            b.sess.step_host(qh, kh, vh, oh, active)
            torch.cuda.synchronize()
            assert torch.equal(oh, a.out.cpu())
    finally:
        a.close()
        b.close()


def test_pipelined_host_entry_matches_device_entry():
    """The queued host path (three staging slots in rotation, copies on their
    own streams) gives the device path's outputs bit for bit, across a
    refresh and with every chunk's host buffers queued before one wait."""
    w = Workload("pipe", B=2, H=4, D=128, fh=8, fw=16, C=2, S=1, W=4, n_chunks=9, dtype="bf16",
                 refresh_period=4, starts=(0, 1))
    a, b = Runner(w), Runner(w)
    try:
        n = w.n_steps
        shape = (n,) + tuple(a.q.shape)
        qh = torch.empty(shape, dtype=a.q.dtype).pin_memory()
        kh, vh = torch.empty_like(qh).pin_memory(), torch.empty_like(qh).pin_memory()
        oh = torch.zeros_like(qh).pin_memory()
        ref = torch.zeros(shape, dtype=a.q.dtype)
        acts = []
        for g in range(n):
            chunks, active = a.step(g)
            acts.append(active)
            torch.cuda.synchronize()
            qh[g].copy_(a.q)
            kh[g].copy_(a.k)
            vh[g].copy_(a.v)
            ref[g].copy_(a.out.cpu())
        for g in range(n):
            b.sess.step_host_async(qh[g], kh[g], vh[g], oh[g], acts[g])
        b.cache.host_wait()
        for g in range(n):
            for s_, on in enumerate(acts[g]):
                if on:
                    assert torch.equal(oh[g][s_], ref[g][s_]), (g, s_)
        assert b.device_status() == 0
    finally:
        a.close()
        b.close()


def test_invalid_arguments_leave_state_unchanged():
    from rolling_kv_cache_sa_b200 import SAError, sa_append_attend
    w = Workload("inv", B=1, H=2, D=128, fh=8, fw=16, C=1, S=1, W=2, n_chunks=2, dtype="bf16")
    r = Runner(w)
    try:
        r.step(0)
        st = r.cache.state(0)
        flat = r.q.view(-1)
        with pytest.raises(SAError) as e:
            sa_append_attend(r.cache.h, flat[1:], r.k, r.v, r.out, None, None, 1)  # misaligned
        assert e.value.status == 1
        assert r.cache.state(0) == st
    finally:
        r.close()
