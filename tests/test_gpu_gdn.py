"""GPU parity of sa_gdn_chunk (Gated DeltaNet block) against the fp64 oracle.

The oracle (orc_gdn_chunk) runs the gated delta rule token by token; the
kernels run its chunkwise form, their products as three-term bf16 split
products on the tensor cores (x = hi + lo, about 2^-16 relative per product,
fp32 accumulation) and the rest in fp32 (D = 64 with the key dims padded to
128). Tolerances:
  * fp32 inputs and outputs: max abs 1e-4 on outputs and on the state, the
    bar the fp32 attention path is held to. Per sub-chunk the split products
    err by about 2^-16 relative on values |S|, |o| <~ 4 through dot products
    of <= 128 terms and a 64 x 64 triangular inverse: a few 1e-6 measured;
    the decay damps older errors, so it does not grow over a stream (a
    32-call stream is checked without re-synchronising with the oracle).
  * bf16 inputs and outputs: the same fp32 arithmetic on the same (bf16)
    input values, then one rounding of o to bf16 (relative 2^-9): the
    attention bar, max abs 2e-2 and mean abs 2e-3 on outputs; the fp32 state
    within 1e-4.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import inputgen as IG
import oracle as O
from inputgen.workloads import P512, Workload

pytestmark = pytest.mark.gpu

F32_MAX = 1e-4
BF16_MAX, BF16_MEAN = 2e-2, 2e-3
STATE_MAX = 1e-4


def _gdn():
    from rolling_kv_cache_sa_b200 import sa_gdn_chunk
    return sa_gdn_chunk


def _tdt(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def _block(w, b, c, tensor):
    a = IG.fill_host(w, b, c, tensor)
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    return t.view(torch.bfloat16) if a.dtype == np.uint16 else t


def _inputs(w, chunks, g_scale):
    """Device inputs [B, Lc, H, D] / [B, Lc, H] for local chunk chunks[b] of
    each stream (chunks[b] < 0: zeros, the stream is inactive)."""
    B = len(chunks)
    z = torch.zeros(w.Lc, w.H, w.D, dtype=_tdt(w))
    zg = torch.zeros(w.Lc, w.H, dtype=torch.float32)
    qs, ks, vs, gs, bs = [], [], [], [], []
    for b in range(B):
        c = chunks[b]
        if c < 0:
            qs.append(z), ks.append(z), vs.append(z), gs.append(zg), bs.append(zg)
            continue
        qs.append(_block(w, b, c, IG.Q))
        ks.append(_block(w, b, c, IG.K))
        vs.append(_block(w, b, c, IG.V))
        g, beta = IG.fill_gates_host(w, b, c, g_scale)
        gs.append(torch.from_numpy(g))
        bs.append(torch.from_numpy(beta))
    dev = lambda xs: torch.stack(xs).cuda().contiguous()   # noqa: E731
    return dev(qs), dev(ks), dev(vs), dev(gs), dev(bs)


def _check(w, out, ref, what):
    err = np.abs(out - ref)
    if w.dtype == "bf16":
        assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN, \
            f"{what}: max {err.max():.3g} mean {err.mean():.3g}"
    else:
        assert err.max() <= F32_MAX, f"{what}: max {err.max():.3g}"
    return err.max()


def _run_streams(w, schedule, g_scale, scale, check_state=True):
    """Calls sa_gdn_chunk once per entry of `schedule` (a list of per-stream
    active flags); every output row of every active stream and every state
    is compared with the oracle after each call."""
    gdn = _gdn()
    B = w.B
    state = torch.zeros(B, w.H, w.D, w.D, dtype=torch.float32, device="cuda")
    ref_state = [np.zeros((w.H, w.D, w.D)) for _ in range(B)]
    local = [0] * B
    out = torch.full((B, w.Lc, w.H, w.D), 7.0, dtype=_tdt(w), device="cuda")
    worst = 0.0
    for act in schedule:
        chunks = [local[b] if act[b] else -1 for b in range(B)]
        q, k, v, g, beta = _inputs(w, chunks, g_scale)
        prev_out = out.clone()
        gdn(state, q, k, v, g, beta, out, scale, active=act)
        torch.cuda.synchronize()
        o = out.float().cpu().numpy()
        st = state.cpu().numpy()
        for b in range(B):
            if not act[b]:
                assert torch.equal(out[b], prev_out[b]), "inactive stream's out was written"
                np.testing.assert_array_equal(st[b], ref_state[b].astype(np.float32))
                continue
            qq, kk, vv, gg, bb = O.gdn_inputs(w, b, local[b], g_scale)
            ref = O.gdn_chunk(scale if scale > 0 else 1 / np.sqrt(w.D), ref_state[b], qq, kk,
                              vv, gg, bb)
            worst = max(worst, _check(w, o[b], ref, f"stream {b} chunk {local[b]}"))
            if check_state:
                serr = np.abs(st[b] - ref_state[b]).max()
                assert serr <= STATE_MAX, f"state of stream {b} after chunk {local[b]}: {serr:.3g}"
                # continue from the GPU's own state so errors are judged per call
                ref_state[b] = st[b].astype(np.float64)
            local[b] += 1
    return worst


def _w(D, dtype, fh, fw, B=3, H=2, seed=0):
    return Workload(f"gdn_{fh}x{fw}_d{D}_{dtype}", B=B, H=H, D=D, fh=fh, fw=fw, C=1, S=1, W=0,
                    n_chunks=4, dtype=dtype, seed=seed)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("g_scale,scale", [(0.3, 1.0), (0.002, 0.0)])
def test_gdn_small_ragged(dtype, D, g_scale, scale):
    # 150 tokens per call: two full 64-token sub-chunks and a ragged tail of 22
    w = _w(D, dtype, 10, 15)
    sched = [(1, 1, 0), (1, 0, 1), (1, 1, 1), (0, 1, 1)]
    _run_streams(w, sched, g_scale, scale)


@pytest.mark.parametrize("fh,fw", [(1, 1), (8, 8), (5, 13), (16, 16)])
def test_gdn_token_counts(fh, fw):
    # T = 1, exactly one sub-chunk, 65 (one token into a second), 256
    w = _w(128, "f32", fh, fw, B=1, H=3, seed=3)
    _run_streams(w, [(1,), (1,)], 0.05, 1.0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
def test_gdn_pieces_with_ragged_tail(dtype, D):
    # 2,107 tokens per call: 33 sub-chunks, the last of 59 tokens. With few
    # heads a call runs in pieces of sub-chunks (the prep of one piece
    # overlapping the sequential pass of the previous, which hands its state
    # on through global memory); an inactive stream in one call. D = 64 runs
    # with its key dims padded to 128.
    w = _w(D, dtype, 43, 49, B=2, H=3, seed=5)
    _run_streams(w, [(1, 1), (1, 0), (1, 1)], 0.02, 0.0)


def test_gdn_many_heads_one_piece():
    # 2,048 tokens per call (32 sub-chunks) over 4 streams x 12 heads: the
    # pass needs 96 CTAs, more than half of the SMs, so a call runs as one
    # piece; then a call with one active stream (24 CTAs), which is split.
    w = _w(128, "bf16", 32, 64, B=4, H=12, seed=7)
    _run_streams(w, [(1, 1, 1, 1), (0, 0, 1, 0)], 0.002, 0.0)


def test_gdn_zero_tokens_and_no_active_stream_are_no_ops():
    gdn = _gdn()
    st0 = torch.randn(2, 2, 64, 64, device="cuda")
    st = st0.clone()
    x = torch.randn(2, 0, 2, 64, device="cuda")
    g = torch.zeros(2, 0, 2, device="cuda")
    gdn(st, x, x, x, g, g, x.clone())
    x1 = torch.randn(2, 5, 2, 64, device="cuda")
    g1 = torch.zeros(2, 5, 2, device="cuda")
    out = torch.zeros_like(x1)
    gdn(st, x1, x1, x1, g1, g1, out, active=[0, 0])
    torch.cuda.synchronize()
    assert torch.equal(st, st0) and torch.all(out == 0)


def test_gdn_special_inputs():
    """Zero key rows write nothing; beta = 0 is pure decay; beta = 1 with a
    repeated key overwrites; all against the oracle."""
    gdn = _gdn()
    T, H, D = 100, 2, 128
    gen = torch.Generator().manual_seed(5)
    q = torch.randn(1, T, H, D, generator=gen)
    k = torch.randn(1, T, H, D, generator=gen)
    v = torch.randn(1, T, H, D, generator=gen)
    k[0, 10:20] = 0.0
    q[0, 30] = 0.0
    k[0, 40:80, 1] = k[0, 40, 1]          # one key repeated 40 times on head 1
    g = -0.05 * torch.rand(1, T, H, generator=gen)
    beta = torch.rand(1, T, H, generator=gen)
    beta[0, :, 0] = 0.0                   # head 0: pure decay of the initial state
    beta[0, 40:80, 1] = 1.0
    g[0, 40:80, 1] = 0.0
    s0 = 0.5 * torch.randn(1, H, D, D, generator=gen)
    state = s0.cuda()
    out = torch.empty(1, T, H, D, device="cuda")
    gdn(state, q.cuda(), k.cuda(), v.cuda(), g.cuda(), beta.cuda(), out, 1.0)
    torch.cuda.synchronize()
    rs = s0[0].double().numpy().copy()
    ref = O.gdn_chunk(1.0, rs, q[0].double().numpy(), k[0].double().numpy(),
                      v[0].double().numpy(), g[0].double().numpy(), beta[0].double().numpy())
    assert np.abs(out[0].cpu().numpy() - ref).max() <= F32_MAX
    assert np.abs(state[0].cpu().numpy() - rs).max() <= STATE_MAX
    assert torch.all(out[0, 30] == 0)


def test_gdn_512p_sampled_heads():
    """The 512p stream (B=1, H=24, D=128, 2048 tokens per chunk, bf16) in the
    launch configuration the benchmark times: every output of three sampled
    heads over two chunks, and their states."""
    w = P512
    gdn = _gdn()
    heads = [0, 11, 23]
    g_scale = 0.002
    state = torch.zeros(1, w.H, w.D, w.D, dtype=torch.float32, device="cuda")
    out = torch.empty(1, w.Lc, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    ref_state = np.zeros((len(heads), w.D, w.D))
    for c in range(2):
        q, k, v, g, beta = _inputs(w.with_(B=1), [c], g_scale)
        gdn(state, q, k, v, g, beta, out)
        torch.cuda.synchronize()
        qq, kk, vv, gg, bb = O.gdn_inputs(w, 0, c, g_scale)
        ref = O.gdn_chunk(1 / np.sqrt(w.D), ref_state, qq[:, heads], kk[:, heads], vv[:, heads],
                          gg[:, heads], bb[:, heads])
        o = out[0][:, heads].float().cpu().numpy()
        _check(w, o, ref, f"512p chunk {c}")
        serr = np.abs(state[0, heads].cpu().numpy() - ref_state).max()
        assert serr <= STATE_MAX, f"512p state after chunk {c}: {serr:.3g}"


def test_gdn_long_stream_no_drift():
    """32 calls of 1,024 tokens (fp32): the state is never reset to the
    oracle's, so an error that compounded would show at the late checks."""
    w = Workload("gdn_long_32x32", B=1, H=2, D=128, fh=32, fw=32, C=1, S=1, W=0, n_chunks=32,
                 dtype="f32")
    gdn = _gdn()
    g_scale = 0.002
    state = torch.zeros(1, w.H, w.D, w.D, dtype=torch.float32, device="cuda")
    out = torch.empty(1, w.Lc, w.H, w.D, dtype=torch.float32, device="cuda")
    ref_state = np.zeros((w.H, w.D, w.D))
    errs = []
    for c in range(32):
        q, k, v, g, beta = _inputs(w, [c], g_scale)
        gdn(state, q, k, v, g, beta, out, 1.0)
        qq, kk, vv, gg, bb = O.gdn_inputs(w, 0, c, g_scale)
        ref = O.gdn_chunk(1.0, ref_state, qq, kk, vv, gg, bb)
        if c in (0, 15, 31):
            torch.cuda.synchronize()
            e = np.abs(out[0].cpu().numpy() - ref).max()
            se = np.abs(state[0].cpu().numpy() - ref_state).max()
            errs.append((c, e, se))
            assert e <= F32_MAX and se <= STATE_MAX, f"chunk {c}: out {e:.3g} state {se:.3g}"
    print("gdn long stream (chunk, out max, state max):", errs)
