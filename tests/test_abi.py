"""The C ABI on the host (no GPU needed): exports, validation, host planner.

The planner's slot map, visible-key count, positions and refresh offset are
compared bit for bit with the oracle's independent closed forms."""
import ctypes
import os
import re

import pytest
import torch

import oracle as O
import rolling_kv_cache_sa_b200 as S
from rolling_kv_cache_sa_b200 import _lib
from inputgen.workloads import ALL, Workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    txt = open(os.path.join(ROOT, "include", "sa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    L = _lib.lib()
    declared = _declared_symbols()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(_lib.EXPORTED) == declared
    assert S.sa_abi_version() == 1


def test_debug_build_exports_every_declared_symbol():
    # the debug build (index checks in every kernel) has the same ABI
    from rolling_kv_cache_sa_b200 import build as B
    assert os.path.exists(B.DEBUG_LIB)
    D = ctypes.CDLL(B.DEBUG_LIB)
    for name in _declared_symbols():
        assert hasattr(D, name), name


def test_debug_entries_refused_by_the_normal_build():
    # outside the debug build the bounds calls say so, before touching a device
    L = _lib.lib()
    if _lib.LIB_PATH.endswith("libsa_debug.so"):
        pytest.skip("running against the debug build")
    assert L.sa_debug_bounds_status(None) == _lib.SA_ERR_UNSUPPORTED
    assert L.sa_debug_bounds_selftest(None) == _lib.SA_ERR_UNSUPPORTED
    assert b"debug build" in L.sa_last_error_string()


def test_invalid_configs_are_rejected():
    base = S.config_for(ALL[1])
    bad = []
    for field, val in [("batch", 0), ("batch", 65), ("heads", 0), ("head_dim", 96),
                       ("frame_h", 0), ("chunk_frames", 0), ("chunk_frames", 33),
                       ("sink_frames", -1), ("window_frames", -1), ("rope_base", 0.0),
                       ("softmax_scale", -1.0), ("dtype", 7)]:
        c = S.config_for(ALL[1])
        setattr(c, field, val)
        bad.append(c)
    c = S.config_for(ALL[1]); c.rope_dims[0] = 43; c.rope_dims[1] = 43; bad.append(c)  # odd
    c = S.config_for(ALL[1]); c.rope_dims[0] = 40; bad.append(c)  # sum != D
    for c in bad:
        with pytest.raises(S.SAError) as e:
            S.sa_plan_chunk(c, 0, 0)
        assert e.value.status == _lib.SA_ERR_INVALID_ARG
        h = ctypes.c_void_p()
        assert _lib.lib().sa_cache_create(ctypes.byref(c), None, ctypes.byref(h)) == \
            _lib.SA_ERR_INVALID_ARG
        assert h.value is None
    S.sa_plan_chunk(base, 0, 0)


def test_state_errors():
    c = S.config_for(ALL[1])  # C = 2
    with pytest.raises(S.SAError) as e:
        S.sa_plan_chunk(c, 3, 0)
    assert e.value.status == _lib.SA_ERR_STATE
    with pytest.raises(S.SAError):
        S.sa_refresh_delta(c, 5, 0)
    assert _lib.lib().sa_append_attend(None, None, None, None, None, None, None) == \
        _lib.SA_ERR_INVALID_ARG
    assert b"NULL" in _lib.lib().sa_last_error_string()


def test_wait_probe_validates_its_limit():
    for bad in (0, 99_999, 10_000_000_001):
        st, _ = S.sa_wait_probe(bad) if torch.cuda.is_available() else \
            (_lib.lib().sa_wait_probe(ctypes.c_uint64(bad), None, None), None)
        assert st == _lib.SA_ERR_INVALID_ARG
    assert b"limit_ns" in _lib.lib().sa_last_error_string()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device refusal")
def test_wait_probe_without_device_is_refused():
    assert _lib.lib().sa_wait_probe(ctypes.c_uint64(2_000_000), None, None) == \
        _lib.SA_ERR_UNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device refusal")
def test_create_without_device_is_refused():
    h = ctypes.c_void_p()
    c = S.config_for(ALL[1])
    assert _lib.lib().sa_cache_create(ctypes.byref(c), None, ctypes.byref(h)) == \
        _lib.SA_ERR_UNSUPPORTED
    assert h.value is None


@pytest.mark.parametrize("C,Sn,W", [(1, 1, 2), (2, 1, 4), (1, 1, 6), (1, 1, 3), (2, 1, 8),
                                    (2, 0, 0), (3, 2, 3), (1, 3, 2), (2, 2, 2)])
def test_planner_matches_oracle(C, Sn, W):
    w = Workload("p", B=1, H=2, D=64, fh=3, fw=5, C=C, S=Sn, W=W, n_chunks=1, dtype="bf16",
                 refresh_period=7)
    cfg = S.config_for(w)
    ocfg = O.cfg_for(w)
    base = 0
    for c in range(0, 120):
        if c > 0 and c % 7 == 0:
            d = S.sa_refresh_delta(cfg, c * C, base)
            assert d == O.refresh_delta(ocfg, c, base)
            base += d
        assert base == O.base_at(ocfg, c)
        pl = S.sa_plan_chunk(cfg, c * C, base)
        assert pl.chunk == c and pl.n_frames == C
        assert pl.n_keys == O.n_keys(ocfg, c)
        assert pl.sink_len + pl.ring_len == pl.n_keys
        for i in range(C):
            f = c * C + i
            assert pl.dest_row[i] == O.frame_slot(ocfg, f) * w.F
            assert pl.t_pos[i] == f - base
            assert pl.is_sink[i] == (f < Sn)
        # keys are the row prefix [0, n_keys): the occupied slots are exactly
        # the first n_keys / F slots after this chunk's append
        sf = O.slot_frames(ocfg, c)
        occupied = [s for s, f in enumerate(sf) if f >= 0]
        assert occupied == list(range(pl.n_keys // w.F))


def _gdn_cfg(**kw):
    c = _lib.sa_gdn_config()
    c.batch, c.heads, c.head_dim, c.dtype, c.tokens, c.scale = 2, 3, 128, _lib.SA_BF16, 64, 0.0
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value", [("batch", 0), ("batch", 65), ("heads", 0),
                                         ("head_dim", 96), ("dtype", 2), ("tokens", -1),
                                         ("scale", -1.0), ("scale", float("inf"))])
def test_gdn_chunk_validates_config(field, value):
    """Argument checks run before any device call (no GPU needed)."""
    c = _gdn_cfg(**{field: value})
    buf = ctypes.create_string_buffer(1 << 12)
    p = ctypes.cast(ctypes.addressof(buf) + (16 - ctypes.addressof(buf) % 16) % 16, ctypes.c_void_p)
    st = _lib.lib().sa_gdn_chunk(ctypes.byref(c), p, p, p, p, p, p, p, p, 1 << 30, None, None)
    assert st == _lib.SA_ERR_INVALID_ARG
    assert _lib.lib().sa_last_error_string()
    n = ctypes.c_size_t()
    assert _lib.lib().sa_gdn_workspace_size(ctypes.byref(c), ctypes.byref(n)) == \
        _lib.SA_ERR_INVALID_ARG


def test_gdn_chunk_validates_pointers():
    L = _lib.lib()
    c = _gdn_cfg()
    assert L.sa_gdn_chunk(None, None, None, None, None, None, None, None, None, 0, None,
                          None) == _lib.SA_ERR_INVALID_ARG
    buf = ctypes.create_string_buffer(1 << 12)
    base = ctypes.addressof(buf) + (16 - ctypes.addressof(buf) % 16) % 16
    p = ctypes.c_void_p(base)
    big = 1 << 30
    assert L.sa_gdn_chunk(ctypes.byref(c), None, p, p, p, p, p, p, p, big, None, None) == \
        _lib.SA_ERR_INVALID_ARG                      # state NULL
    assert L.sa_gdn_chunk(ctypes.byref(c), ctypes.c_void_p(base + 4), p, p, p, p, p, p, p, big,
                          None, None) == _lib.SA_ERR_INVALID_ARG   # state not 16-byte aligned
    assert L.sa_gdn_chunk(ctypes.byref(c), p, p, None, p, p, p, p, p, big, None, None) == \
        _lib.SA_ERR_INVALID_ARG                      # k NULL with tokens > 0
    assert L.sa_gdn_chunk(ctypes.byref(c), p, ctypes.c_void_p(base + 1), p, p, p, p, p, p, big,
                          None, None) == _lib.SA_ERR_INVALID_ARG   # q misaligned for bf16
    assert b"aligned" in L.sa_last_error_string()
    assert L.sa_gdn_chunk(ctypes.byref(c), p, p, p, p, p, p, p, None, big, None, None) == \
        _lib.SA_ERR_INVALID_ARG                      # workspace NULL
    n = ctypes.c_size_t()
    assert L.sa_gdn_workspace_size(ctypes.byref(c), ctypes.byref(n)) == _lib.SA_OK
    # header + B * H * ceil(T / 64) blocks of 96 KiB of operand images (the
    # images are 128 key dims wide for D = 64 too)
    per = 98304
    assert n.value == 1024 + 2 * 3 * 1 * per
    c.tokens = 65
    assert L.sa_gdn_workspace_size(ctypes.byref(c), ctypes.byref(n)) == _lib.SA_OK
    assert n.value == 1024 + 2 * 3 * 2 * per
    c.head_dim = 64
    assert L.sa_gdn_workspace_size(ctypes.byref(c), ctypes.byref(n)) == _lib.SA_OK
    assert n.value == 1024 + 2 * 3 * 2 * per
    c.head_dim = 128
    assert L.sa_gdn_workspace_size(ctypes.byref(c), ctypes.byref(n)) == _lib.SA_OK
    assert L.sa_gdn_chunk(ctypes.byref(c), p, p, p, p, p, p, p, p, n.value - 16, None,
                          None) == _lib.SA_ERR_INVALID_ARG   # workspace too small
    assert b"workspace" in L.sa_last_error_string()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device refusal")
def test_gdn_chunk_without_device_is_refused():
    buf = ctypes.create_string_buffer(1 << 12)
    p = ctypes.c_void_p(ctypes.addressof(buf) + (16 - ctypes.addressof(buf) % 16) % 16)
    c = _gdn_cfg()
    assert _lib.lib().sa_gdn_chunk(ctypes.byref(c), p, p, p, p, p, p, p, p, 1 << 30, None,
                                   None) == _lib.SA_ERR_UNSUPPORTED


def test_gdn_binding_checks_shapes_before_the_call():
    """The Python binding refuses mismatched tensors before reaching the library."""
    from rolling_kv_cache_sa_b200 import sa_gdn_chunk
    B, T, H, D = 2, 5, 3, 64
    q = torch.zeros(B, T, H, D)
    ok = dict(state=torch.zeros(B, H, D, D), k=torch.zeros_like(q), v=torch.zeros_like(q),
              g=torch.zeros(B, T, H), beta=torch.zeros(B, T, H), out=torch.zeros_like(q))
    bad = [("state", torch.zeros(B, H, D, D + 1)), ("k", torch.zeros(B, T, H, D + 1)),
           ("v", torch.zeros(B, T, H, D, dtype=torch.bfloat16)), ("g", torch.zeros(B, T, H + 1)),
           ("beta", torch.zeros(B, T, H, dtype=torch.float64)),
           ("out", torch.zeros(B, T, H, D).transpose(0, 1).contiguous().transpose(0, 1))]
    for name, t in bad:
        args = dict(ok, **{name: t})
        with pytest.raises(ValueError, match=name):
            sa_gdn_chunk(args["state"], q, args["k"], args["v"], args["g"], args["beta"],
                         args["out"])
