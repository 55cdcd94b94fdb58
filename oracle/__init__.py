"""ctypes wrapper of the fp64 C oracle (oracle.c): the rolling-cache attention
path and the GDN block's gated delta rule.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg; never by the product path. It shares no code
with the CUDA path (only the seeded input generator).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from inputgen import Spec, spec_for
from inputgen.workloads import Workload

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

EXACT, STORE_F32, STORE_BF16, STORE_E4M3 = 0, 1, 2, 3


class Cfg(ctypes.Structure):
    _fields_ = [
        ("H", ctypes.c_int32), ("D", ctypes.c_int32), ("fh", ctypes.c_int32),
        ("fw", ctypes.c_int32), ("C", ctypes.c_int32), ("S", ctypes.c_int32),
        ("W", ctypes.c_int32), ("rope_dims", ctypes.c_int32 * 3),
        ("rope_base", ctypes.c_double), ("scale", ctypes.c_double),
        ("refresh_period", ctypes.c_int64), ("store", ctypes.c_int32),
        ("in_dtype", ctypes.c_int32), ("sink_repin", ctypes.c_int32), ("pad_", ctypes.c_int32),
        ("sink_update_period", ctypes.c_int64), ("sink_alpha", ctypes.c_double),
        ("fp8_scale", ctypes.c_void_p),
    ]


_P = ctypes.POINTER
_D = ctypes.c_void_p


def lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(_HERE, "liboracle.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        L = ctypes.CDLL(path)
        C, S = _P(Cfg), _P(Spec)
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        sig = {
            "orc_round_store": ([i32, ctypes.c_double], ctypes.c_double),
            "orc_theta": ([C, i32, i32], ctypes.c_double),
            "orc_rope_vec": ([C, _D, ctypes.c_double, ctypes.c_double, ctypes.c_double, _D], None),
            "orc_rope_tband": ([C, _D, ctypes.c_double, _D], None),
            "orc_refresh_due": ([C, i64], i32),
            "orc_refresh_delta": ([C, i64, i64], i64),
            "orc_base_at": ([C, i64], i64),
            "orc_visible": ([C, i64, i64], i32),
            "orc_frame_slot": ([C, i64], i64),
            "orc_slot_frames": ([C, i64, _D], None),
            "orc_n_keys": ([C, i64], i64),
            "orc_input_block": ([C, S, i64, i64, i32, _D], i32),
            "orc_stored_key_frame": ([C, S, i64, i64, i64, _D], i32),
            "orc_query_rot": ([C, S, i64, i64, _D], i32),
            "orc_cache_contents": ([C, S, i64, i64, _D, _D, _D], i32),
            "orc_attend_rows": ([C, S, i64, i64, i32, _D, _D, _D], i32),
            "orc_bruteforce_rows": ([C, S, i64, i64, i32, _D, _D, _D], i32),
            "orc_attend_rows_uncommitted": ([C, S, S, i64, i64, i32, _D, _D, _D], i32),
            "orc_sink_pos": ([C, i64, i64], ctypes.c_double),
            "orc_sink_raw": ([C, S, i64, i64, i64, i32, _D], i32),
            "orc_gdn_chunk": ([i32, i32, i64, ctypes.c_double, _D, _D, _D, _D, _D, _D, _D], i32),
            "orc_num_threads": ([], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = L
    return _LIB


def cfg_for(w: Workload, store: int | None = None, refresh_period: int | None = None) -> Cfg:
    """Oracle configuration of a workload. store defaults to the workload's
    storage dtype (bf16 or fp32 rounding); pass EXACT for the exact mode."""
    c = Cfg()
    c.H, c.D, c.fh, c.fw, c.C, c.S, c.W = w.H, w.D, w.fh, w.fw, w.C, w.S, w.W
    for i in range(3):
        c.rope_dims[i] = w.dims[i]
    c.rope_base = w.rope_base
    c.scale = 0.0
    c.refresh_period = w.refresh_period if refresh_period is None else refresh_period
    if store is None:
        store = STORE_E4M3 if w.cache == "e4m3" else (STORE_BF16 if w.dtype == "bf16" else STORE_F32)
    c.store = store
    c.in_dtype = 1 if w.dtype == "bf16" else 0
    if w.fp8_scales:
        arr = np.ascontiguousarray(np.asarray(w.fp8_scales, dtype=np.float64).reshape(3, w.H))
        c._scales = arr  # keeps the array alive with the struct
        c.fp8_scale = arr.ctypes.data
    else:
        c.fp8_scale = None
    c.sink_repin = 1 if w.sink_repin else 0
    c.sink_update_period = w.sink_update_period
    c.sink_alpha = w.sink_alpha
    return c


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed ({rc})")


def round_store(store: int, x: float) -> float:
    return lib().orc_round_store(store, x)


def theta(cfg: Cfg, band: int, j: int) -> float:
    return lib().orc_theta(ctypes.byref(cfg), band, j)


def rope_vec(cfg: Cfg, x: np.ndarray, t: float, y: float, w: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    lib().orc_rope_vec(ctypes.byref(cfg), _ptr(x), t, y, w, _ptr(out))
    return out


def rope_tband(cfg: Cfg, x: np.ndarray, t: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    lib().orc_rope_tband(ctypes.byref(cfg), _ptr(x), t, _ptr(out))
    return out


def refresh_due(cfg: Cfg, c: int) -> bool:
    return bool(lib().orc_refresh_due(ctypes.byref(cfg), c))


def refresh_delta(cfg: Cfg, c: int, base: int) -> int:
    return lib().orc_refresh_delta(ctypes.byref(cfg), c, base)


def base_at(cfg: Cfg, c: int) -> int:
    return lib().orc_base_at(ctypes.byref(cfg), c)


def visible(cfg: Cfg, c: int, f: int) -> bool:
    return bool(lib().orc_visible(ctypes.byref(cfg), c, f))


def frame_slot(cfg: Cfg, f: int) -> int:
    return lib().orc_frame_slot(ctypes.byref(cfg), f)


def slot_frames(cfg: Cfg, c: int) -> np.ndarray:
    out = np.empty(cfg.S + cfg.W + cfg.C, dtype=np.int64)
    lib().orc_slot_frames(ctypes.byref(cfg), c, _ptr(out))
    return out


def n_keys(cfg: Cfg, c: int) -> int:
    return lib().orc_n_keys(ctypes.byref(cfg), c)


def input_block(cfg: Cfg, spec: Spec, stream: int, chunk: int, tensor: int) -> np.ndarray:
    out = np.empty((cfg.C * cfg.fh * cfg.fw, cfg.H, cfg.D), dtype=np.float64)
    _check(lib().orc_input_block(ctypes.byref(cfg), ctypes.byref(spec), stream, chunk, tensor,
                                 _ptr(out)), "orc_input_block")
    return out


def stored_key_frame(cfg: Cfg, spec: Spec, stream: int, f: int, c: int) -> np.ndarray:
    out = np.empty((cfg.fh * cfg.fw, cfg.H, cfg.D), dtype=np.float64)
    _check(lib().orc_stored_key_frame(ctypes.byref(cfg), ctypes.byref(spec), stream, f, c,
                                      _ptr(out)), "orc_stored_key_frame")
    return out


def query_rot(cfg: Cfg, spec: Spec, stream: int, c: int) -> np.ndarray:
    out = np.empty((cfg.C * cfg.fh * cfg.fw, cfg.H, cfg.D), dtype=np.float64)
    _check(lib().orc_query_rot(ctypes.byref(cfg), ctypes.byref(spec), stream, c, _ptr(out)),
           "orc_query_rot")
    return out


def cache_contents(cfg: Cfg, spec: Spec, stream: int, c: int):
    """(K' [H, (S+R)F, D], V [H, (S+R)F, D], slot_frame [S+R]) after chunk c."""
    rows = (cfg.S + cfg.W + cfg.C) * cfg.fh * cfg.fw
    k = np.empty((cfg.H, rows, cfg.D), dtype=np.float64)
    v = np.empty_like(k)
    sf = np.empty(cfg.S + cfg.W + cfg.C, dtype=np.int64)
    _check(lib().orc_cache_contents(ctypes.byref(cfg), ctypes.byref(spec), stream, c, _ptr(k),
                                    _ptr(v), _ptr(sf)), "orc_cache_contents")
    return k, v, sf


def _rows(fn, cfg, spec, stream, c, toks, heads):
    toks = np.ascontiguousarray(toks, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    assert toks.shape == heads.shape and toks.ndim == 1
    out = np.empty((len(toks), cfg.D), dtype=np.float64)
    _check(fn(ctypes.byref(cfg), ctypes.byref(spec), stream, c, len(toks), _ptr(toks),
              _ptr(heads), _ptr(out)), fn.__name__)
    return out


def attend_rows(cfg: Cfg, spec: Spec, stream: int, c: int, toks, heads) -> np.ndarray:
    """Cache-path attention output rows (tok, head) of chunk c: [n, D] fp64."""
    return _rows(lib().orc_attend_rows, cfg, spec, stream, c, toks, heads)


def sink_pos(cfg: Cfg, f: int, c: int) -> float:
    """Temporal position of sink frame f while chunk c is processed."""
    return lib().orc_sink_pos(ctypes.byref(cfg), f, c)


def sink_raw(cfg: Cfg, spec: Spec, stream: int, f: int, c: int, tensor: int) -> np.ndarray:
    """Raw key (tensor K) or value (V) of sink frame f at chunk c, [F, H, D]."""
    out = np.empty((cfg.fh * cfg.fw, cfg.H, cfg.D), dtype=np.float64)
    _check(lib().orc_sink_raw(ctypes.byref(cfg), ctypes.byref(spec), stream, f, c, tensor,
                              _ptr(out)), "orc_sink_raw")
    return out


def attend_rows_uncommitted(cfg: Cfg, spec_cache: Spec, spec_chunk: Spec, stream: int, c: int,
                            toks, heads) -> np.ndarray:
    """Rows of chunk c attended with uncommitted inputs: frames before the
    chunk from spec_cache, the chunk's queries, keys and values from
    spec_chunk. [n, D] fp64."""
    toks = np.ascontiguousarray(toks, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    assert toks.shape == heads.shape and toks.ndim == 1
    out = np.empty((len(toks), cfg.D), dtype=np.float64)
    _check(lib().orc_attend_rows_uncommitted(
        ctypes.byref(cfg), ctypes.byref(spec_cache), ctypes.byref(spec_chunk), stream, c,
        len(toks), _ptr(toks), _ptr(heads), _ptr(out)), "orc_attend_rows_uncommitted")
    return out


def bruteforce_rows(cfg: Cfg, spec: Spec, stream: int, c: int, toks, heads) -> np.ndarray:
    """Brute-force masked full-sequence attention rows (exact, absolute positions)."""
    return _rows(lib().orc_bruteforce_rows, cfg, spec, stream, c, toks, heads)


def gdn_chunk(scale: float, state: np.ndarray, q, k, v, g, beta) -> np.ndarray:
    """One call of the Gated DeltaNet recurrence (orc_gdn_chunk) over T tokens:
    state [H, D, D] float64 (value dim, key dim) is updated in place; q, k, v
    [T, H, D]; g (log decay) and beta [T, H]. Returns out [T, H, D] float64."""
    assert state.dtype == np.float64 and state.flags["C_CONTIGUOUS"]
    H, D, D2 = state.shape
    assert D == D2
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    g, beta = (np.ascontiguousarray(x, dtype=np.float64) for x in (g, beta))
    T = q.shape[0]
    assert q.shape == k.shape == v.shape == (T, H, D) and g.shape == beta.shape == (T, H)
    out = np.empty((T, H, D), dtype=np.float64)
    _check(lib().orc_gdn_chunk(H, D, T, scale, _ptr(state), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                               _ptr(beta), _ptr(out)), "orc_gdn_chunk")
    return out


def gdn_inputs(w: Workload, stream: int, c: int, g_scale: float):
    """Generated inputs of chunk c of a stream for the GDN block, as stored:
    q, k, v [Lc, H, D] and g, beta [Lc, H], float64."""
    from inputgen import fill_gates_host
    cfg = cfg_for(w)
    spec = spec_for(w)
    q = input_block(cfg, spec, stream, c, 0)
    k = input_block(cfg, spec, stream, c, 1)
    v = input_block(cfg, spec, stream, c, 2)
    g, beta = fill_gates_host(w, stream, c, g_scale)
    return q, k, v, g.astype(np.float64), beta.astype(np.float64)


def gdn_stream(w: Workload, stream: int, c: int, g_scale: float, scale: float, heads=None,
               state: np.ndarray | None = None, c0: int = 0):
    """Runs the GDN block over chunks c0..c of a stream from `state` (zero when
    None) with the generated inputs; returns (out of chunk c [Lc, H', D],
    state after chunk c [H', D, D]) for the heads `heads` (all when None)."""
    hs = np.arange(w.H) if heads is None else np.asarray(heads)
    if state is None:
        state = np.zeros((len(hs), w.D, w.D), dtype=np.float64)
    out = None
    for ch in range(c0, c + 1):
        q, k, v, g, beta = gdn_inputs(w, stream, ch, g_scale)
        out = gdn_chunk(scale, state, q[:, hs], k[:, hs], v[:, hs], g[:, hs], beta[:, hs])
    return out, state


def num_threads() -> int:
    return lib().orc_num_threads()
