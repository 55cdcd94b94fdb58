"""Seeded synthetic inputs shared by the oracle side and the GPU side.

Loads ``libsa_inputgen.so`` (built from ``inputgen.cu``). Holds none of the
attention method's arithmetic: values are pure functions of
(seed, stream, chunk, tensor, element index).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .workloads import Workload  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

Q, K, V = 0, 1, 2
GATE, BETA = 4, 5
SINK_UPDATE_CHUNK0 = 1 << 40  # chunk coordinate base of sink-update blocks (sa_inputgen.h)
F32, BF16 = 0, 1


class Spec(ctypes.Structure):
    _fields_ = [
        ("seed", ctypes.c_uint64),
        ("dist", ctypes.c_int32 * 3),
        ("outlier_frac", ctypes.c_double),
        ("outlier_scale", ctypes.c_float),
        ("pad_", ctypes.c_int32),
    ]


def lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(_HERE, "libsa_inputgen.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        L = ctypes.CDLL(path)
        L.ig_fill_host.argtypes = [ctypes.POINTER(Spec), ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                   ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]
        L.ig_fill_host.restype = ctypes.c_int
        L.ig_fill_device.argtypes = [ctypes.POINTER(Spec), ctypes.c_int32,
                                     ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                                     ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
        L.ig_fill_device.restype = ctypes.c_int
        L.ig_fill_gates_host.argtypes = [ctypes.POINTER(Spec), ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                         ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
        L.ig_fill_gates_host.restype = ctypes.c_int
        _LIB = L
    return _LIB


def spec_for(w: Workload) -> Spec:
    s = Spec()
    s.seed = w.seed
    for i in range(3):
        s.dist[i] = w.dist[i]
    s.outlier_frac = w.outlier_frac
    s.outlier_scale = w.outlier_scale
    return s


def dtype_code(w: Workload) -> int:
    return BF16 if w.dtype == "bf16" else F32


def fill_host(w: Workload, stream: int, chunk: int, tensor: int, tok0: int = 0,
              n_tok: int | None = None) -> np.ndarray:
    """Block [n_tok, H, D] of one tensor; float32, or uint16 bf16 bits."""
    n_tok = w.Lc - tok0 if n_tok is None else n_tok
    dt = dtype_code(w)
    out = np.empty((n_tok, w.H, w.D), dtype=np.uint16 if dt == BF16 else np.float32)
    sp = spec_for(w)
    rc = lib().ig_fill_host(ctypes.byref(sp), stream, chunk, tensor, tok0, n_tok, w.H, w.D, dt,
                            out.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"ig_fill_host failed ({rc})")
    return out


def fill_gates_host(w: Workload, stream: int, chunk: int, g_scale: float, tok0: int = 0,
                    n_tok: int | None = None):
    """Gated DeltaNet gate inputs of one chunk: (g, beta), float32 [n_tok, H]
    each; g = log decay in (-g_scale, 0), beta in (0, 1)."""
    n_tok = w.Lc - tok0 if n_tok is None else n_tok
    g = np.empty((n_tok, w.H), dtype=np.float32)
    beta = np.empty((n_tok, w.H), dtype=np.float32)
    sp = spec_for(w)
    rc = lib().ig_fill_gates_host(ctypes.byref(sp), stream, chunk, tok0, n_tok, w.H,
                                  ctypes.c_float(g_scale), g.ctypes.data, beta.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"ig_fill_gates_host failed ({rc})")
    return g, beta


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def fill_host_f32(w: Workload, stream: int, chunk: int, tensor: int, **kw) -> np.ndarray:
    """Same block as fill_host, converted to float32 values."""
    a = fill_host(w, stream, chunk, tensor, **kw)
    return bf16_bits_to_f32(a) if a.dtype == np.uint16 else a


def sink_update_chunk(u: int) -> int:
    """Chunk coordinate of the sink-update block applied before chunk u."""
    return SINK_UPDATE_CHUNK0 + u


def fill_device(w: Workload, stream_ids, chunks, tensor: int, out_ptr: int, cuda_stream: int,
                n_tok: int | None = None):
    """Fill a device buffer [len(chunks), n_tok, H, D] (n_tok defaults to Lc);
    chunks[i] < 0 skips slot i."""
    n = len(chunks)
    sids = (ctypes.c_int64 * n)(*stream_ids)
    chs = (ctypes.c_int64 * n)(*chunks)
    sp = spec_for(w)
    rc = lib().ig_fill_device(ctypes.byref(sp), n, sids, chs, tensor,
                              w.Lc if n_tok is None else n_tok, w.H, w.D,
                              dtype_code(w), ctypes.c_void_p(out_ptr), ctypes.c_void_p(cuda_stream))
    if rc != 0:
        raise RuntimeError(f"ig_fill_device failed ({rc})")
