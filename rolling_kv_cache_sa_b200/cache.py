"""Python binding of libsa.so: the C-ABI calls under the same names, plus a
small handle class. Argument marshalling only -- every step of the path runs
in the library's CUDA kernels; PyTorch supplies device memory and streams."""
from __future__ import annotations

import ctypes
import math
from typing import Optional, Sequence

import numpy as np
import torch

from ._lib import SA_BF16, SA_BF16_E4M3, SA_F32, check, lib, sa_chunk_plan, sa_config


def make_config(batch: int, heads: int, head_dim: int, frame_h: int, frame_w: int,
                chunk_frames: int, sink_frames: int, window_frames: int,
                rope_dims: Sequence[int], rope_base: float = 10000.0,
                softmax_scale: float = 0.0, dtype: str = "bf16") -> sa_config:
    c = sa_config()
    c.batch, c.heads, c.head_dim = batch, heads, head_dim
    c.frame_h, c.frame_w = frame_h, frame_w
    c.chunk_frames, c.sink_frames, c.window_frames = chunk_frames, sink_frames, window_frames
    for i in range(3):
        c.rope_dims[i] = int(rope_dims[i])
    c.rope_base = rope_base
    c.softmax_scale = softmax_scale
    c.dtype = {"bf16": SA_BF16, "f32": SA_F32, "bf16_e4m3": SA_BF16_E4M3}[dtype]
    return c


def config_for(w) -> sa_config:
    """sa_config of a workload description (inputgen.workloads.Workload)."""
    dtype = "bf16_e4m3" if getattr(w, "cache", "") == "e4m3" else w.dtype
    return make_config(w.B, w.H, w.D, w.fh, w.fw, w.C, w.S, w.W, w.dims, w.rope_base, 0.0, dtype)


def _mask(active, n: int):
    if active is None:
        return None
    a = (ctypes.c_uint8 * n)(*[1 if x else 0 for x in active])
    return a


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


# ---- the C-ABI calls, same names -------------------------------------------------
def sa_cache_create(cfg: sa_config, stream: Optional[torch.cuda.Stream] = None) -> int:
    h = ctypes.c_void_p()
    check(lib().sa_cache_create(ctypes.byref(cfg), ctypes.c_void_p(_stream_ptr(stream)),
                                ctypes.byref(h)), "sa_cache_create")
    return h.value


def sa_append_attend(h: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                     active=None, stream: Optional[torch.cuda.Stream] = None, batch: int = 0):
    check(lib().sa_append_attend(h, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 _mask(active, batch or q.shape[0]), _stream_ptr(stream)),
          "sa_append_attend")


def sa_attend(h: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
              active=None, stream: Optional[torch.cuda.Stream] = None, batch: int = 0):
    check(lib().sa_attend(h, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                          _mask(active, batch or q.shape[0]), _stream_ptr(stream)), "sa_attend")


def sa_cache_set_sink_mode(h: int, mode: int):
    check(lib().sa_cache_set_sink_mode(h, mode), "sa_cache_set_sink_mode")


def sa_cache_set_fp8_scales(h: int, q_scale=None, k_scale=None, v_scale=None):
    arrs = [None if x is None else (ctypes.c_float * len(x))(*[float(v) for v in x])
            for x in (q_scale, k_scale, v_scale)]
    check(lib().sa_cache_set_fp8_scales(h, *arrs), "sa_cache_set_fp8_scales")


def sa_cache_get_fp8_scales(h: int, heads: int) -> np.ndarray:
    """The handle's e4m3 scales as a [3, H] array (q, k, v)."""
    arrs = [(ctypes.c_float * heads)() for _ in range(3)]
    check(lib().sa_cache_get_fp8_scales(h, *arrs), "sa_cache_get_fp8_scales")
    return np.array([list(a) for a in arrs], dtype=np.float64)


def sa_sink_update(h: int, k_new: torch.Tensor, v_new: torch.Tensor, alpha: float, active=None,
                   stream: Optional[torch.cuda.Stream] = None, batch: int = 0):
    check(lib().sa_sink_update(h, k_new.data_ptr(), v_new.data_ptr(), ctypes.c_float(alpha),
                               _mask(active, batch or k_new.shape[0]), _stream_ptr(stream)),
          "sa_sink_update")


def sa_rope_refresh(h: int, active=None, batch: int = 0,
                    stream: Optional[torch.cuda.Stream] = None):
    check(lib().sa_rope_refresh(h, _mask(active, batch), _stream_ptr(stream)), "sa_rope_refresh")


def sa_cache_reset(h: int, streams=None, batch: int = 0):
    check(lib().sa_cache_reset(h, _mask(streams, batch)), "sa_cache_reset")


def sa_cache_destroy(h: int):
    check(lib().sa_cache_destroy(h), "sa_cache_destroy")


def sa_append_attend_host(h: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                          out: torch.Tensor, active=None,
                          stream: Optional[torch.cuda.Stream] = None):
    for t in (q, k, v, out):
        assert t.device.type == "cpu" and t.is_contiguous()
    check(lib().sa_append_attend_host(h, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      _mask(active, q.shape[0]), _stream_ptr(stream)),
          "sa_append_attend_host")


def sa_append_attend_host_async(h: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                out: torch.Tensor, active=None,
                                stream: Optional[torch.cuda.Stream] = None):
    for t in (q, k, v, out):
        assert t.device.type == "cpu" and t.is_contiguous()
    check(lib().sa_append_attend_host_async(h, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            out.data_ptr(), _mask(active, q.shape[0]),
                                            _stream_ptr(stream)), "sa_append_attend_host_async")


def sa_host_wait(h: int):
    check(lib().sa_host_wait(h), "sa_host_wait")


def sa_cache_export(h: int, stream: Optional[torch.cuda.Stream] = None) -> np.ndarray:
    """The handle's checkpoint as a uint8 host array."""
    n = ctypes.c_size_t()
    check(lib().sa_cache_export_size(h, ctypes.byref(n)), "sa_cache_export_size")
    buf = np.empty(n.value, dtype=np.uint8)
    check(lib().sa_cache_export(h, buf.ctypes.data, n.value, _stream_ptr(stream)),
          "sa_cache_export")
    return buf


def sa_cache_import(h: int, blob: np.ndarray, stream: Optional[torch.cuda.Stream] = None):
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    check(lib().sa_cache_import(h, blob.ctypes.data, blob.size, _stream_ptr(stream)),
          "sa_cache_import")


def sa_stream_state(h: int, b: int):
    fw, base = ctypes.c_int64(), ctypes.c_int64()
    check(lib().sa_stream_state(h, b, ctypes.byref(fw), ctypes.byref(base)), "sa_stream_state")
    return fw.value, base.value


def sa_cache_copy_out(h: int, b: int, k_host: np.ndarray, v_host: np.ndarray,
                      stream: Optional[torch.cuda.Stream] = None):
    check(lib().sa_cache_copy_out(h, b, k_host.ctypes.data, v_host.ctypes.data,
                                  _stream_ptr(stream)), "sa_cache_copy_out")


def sa_get_device_status(h: int, stream: Optional[torch.cuda.Stream] = None) -> int:
    return lib().sa_get_device_status(h, _stream_ptr(stream))


def sa_plan_chunk(cfg: sa_config, frames_written: int, pos_base: int) -> sa_chunk_plan:
    plan = sa_chunk_plan()
    check(lib().sa_plan_chunk(ctypes.byref(cfg), frames_written, pos_base, ctypes.byref(plan)),
          "sa_plan_chunk")
    return plan


def sa_refresh_delta(cfg: sa_config, frames_written: int, pos_base: int) -> int:
    d = ctypes.c_int64()
    check(lib().sa_refresh_delta(ctypes.byref(cfg), frames_written, pos_base, ctypes.byref(d)),
          "sa_refresh_delta")
    return d.value


def sa_profile_begin(h: int):
    check(lib().sa_profile_begin(h), "sa_profile_begin")


def sa_profile_end(h: int):
    ms = [ctypes.c_double() for _ in range(3)]
    n = [ctypes.c_int32() for _ in range(3)]
    check(lib().sa_profile_end(h, ctypes.byref(ms[0]), ctypes.byref(n[0]), ctypes.byref(ms[1]),
                               ctypes.byref(n[1]), ctypes.byref(ms[2]), ctypes.byref(n[2])),
          "sa_profile_end")
    return {"append": (ms[0].value, n[0].value), "attend": (ms[1].value, n[1].value),
            "refresh": (ms[2].value, n[2].value)}


def sa_profile_launches(h: int) -> int:
    n = ctypes.c_int64()
    check(lib().sa_profile_launches(h, ctypes.byref(n)), "sa_profile_launches")
    return n.value


def _need(t, name: str, shape, dtype, device):
    if not isinstance(t, torch.Tensor) or t.device != device or t.dtype != dtype or \
            not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        got = (f"{tuple(t.shape)} {t.dtype} on {t.device}"
               f"{'' if t.is_contiguous() else ', not contiguous'}"
               if isinstance(t, torch.Tensor) else type(t).__name__)
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on "
                         f"{device}; got {got}")


def sa_append_attend_noalloc(cfg: sa_config, k_cache: torch.Tensor, v_cache: torch.Tensor,
                             k_raw: Optional[torch.Tensor], frames_written, pos_base,
                             q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                             active=None, stream: Optional[torch.cuda.Stream] = None):
    """Allocation-free append + attention over caller-owned cache buffers.
    frames_written / pos_base: ctypes int64 arrays of length B (host);
    frames_written is advanced in place; pos_base must stay at each stream's
    first value (there is no allocation-free refresh).

    The library cannot check the sizes of the buffers it is given, so they
    are checked here before the call: k_cache and v_cache [B, H, (S+W+C)*F, D],
    k_raw [B, H, S*F, D] (when S > 0), q, k, v and out [B, C*F, H, D], all
    contiguous, of the configuration's dtype and on the current device."""
    if cfg.dtype == SA_BF16_E4M3:
        raise ValueError("the allocation-free entry runs SA_F32 and SA_BF16 caches")
    B, H, D = cfg.batch, cfg.heads, cfg.head_dim
    F = cfg.frame_h * cfg.frame_w
    Lc = cfg.chunk_frames * F
    ntok = (cfg.sink_frames + cfg.window_frames + cfg.chunk_frames) * F
    dt = torch.float32 if cfg.dtype == SA_F32 else torch.bfloat16
    dev = torch.device("cuda", torch.cuda.current_device())
    _need(k_cache, "k_cache", (B, H, ntok, D), dt, dev)
    _need(v_cache, "v_cache", (B, H, ntok, D), dt, dev)
    if cfg.sink_frames > 0:
        _need(k_raw, "k_raw", (B, H, cfg.sink_frames * F, D), dt, dev)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _need(t, n, (B, Lc, H, D), dt, dev)
    if len(frames_written) != B or len(pos_base) != B:
        raise ValueError(f"frames_written and pos_base must hold {B} entries")
    if active is not None and len(active) != B:
        raise ValueError(f"active must hold {B} entries")
    check(lib().sa_append_attend_noalloc(
        ctypes.byref(cfg), k_cache.data_ptr(), v_cache.data_ptr(),
        k_raw.data_ptr() if (k_raw is not None and cfg.sink_frames > 0) else None,
        frames_written, pos_base, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
        _mask(active, cfg.batch), _stream_ptr(stream)), "sa_append_attend_noalloc")


def sa_noalloc_device_status(stream: Optional[torch.cuda.Stream] = None):
    """Raises SAError(SA_ERR_DEVICE_TIMEOUT) if a bounded wait of an
    allocation-free call on the current device gave up since the last read;
    synchronises the stream and clears the word."""
    check(lib().sa_noalloc_device_status(_stream_ptr(stream)), "sa_noalloc_device_status")


def sa_wait_probe(limit_ns: int, stream: Optional[torch.cuda.Stream] = None):
    """Runs the bounded-wait check; returns (status, [waited_ns warp0, warp1])
    without raising (SA_ERR_DEVICE_TIMEOUT is the designed outcome)."""
    w = (ctypes.c_int64 * 2)()
    st = lib().sa_wait_probe(ctypes.c_uint64(limit_ns), w, ctypes.c_void_p(_stream_ptr(stream)))
    return st, [w[0], w[1]]


def sa_abi_version() -> int:
    return lib().sa_abi_version()


# ---- handle class -----------------------------------------------------------------
class SACache:
    """Owns one libsa cache handle on the current CUDA device."""

    def __init__(self, cfg: sa_config, stream: Optional[torch.cuda.Stream] = None):
        self.cfg = cfg
        self.B, self.H, self.D = cfg.batch, cfg.heads, cfg.head_dim
        self.F = cfg.frame_h * cfg.frame_w
        self.Lc = cfg.chunk_frames * self.F
        self.R = cfg.window_frames + cfg.chunk_frames
        self.ntok = (cfg.sink_frames + self.R) * self.F
        self.dtype = torch.float32 if cfg.dtype == SA_F32 else torch.bfloat16
        self.fp8 = cfg.dtype == SA_BF16_E4M3
        self.scales = np.ones((3, cfg.heads))
        self.device = torch.device("cuda", torch.cuda.current_device())
        self.h = sa_cache_create(cfg, stream)

    def _check_tensor(self, t: torch.Tensor, name: str):
        if t.device != self.device or t.dtype != self.dtype or not t.is_contiguous() or \
                tuple(t.shape) != (self.B, self.Lc, self.H, self.D):
            raise ValueError(f"{name} must be a contiguous {self.dtype} tensor of shape "
                             f"{(self.B, self.Lc, self.H, self.D)} on {self.device}")

    def append_attend(self, q, k, v, out, active=None, stream=None):
        for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
            self._check_tensor(t, n)
        sa_append_attend(self.h, q, k, v, out, active, stream, self.B)

    def attend(self, q, k, v, out, active=None, stream=None):
        """Attention of the next chunk without committing it (a denoising step
        that is not the chunk's last)."""
        for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
            self._check_tensor(t, n)
        sa_attend(self.h, q, k, v, out, active, stream, self.B)

    def append_attend_host_async(self, q, k, v, out, active=None, stream=None):
        """Queues the host-buffer step and returns; host_wait() before reading
        out or reusing the inputs."""
        sa_append_attend_host_async(self.h, q, k, v, out, active, stream)

    def host_wait(self):
        sa_host_wait(self.h)

    def export(self, stream=None) -> np.ndarray:
        """Checkpoint (cache contents and stream state) as a host byte array."""
        return sa_cache_export(self.h, stream)

    def import_(self, blob, stream=None):
        """Restores a checkpoint of a handle with the same configuration."""
        sa_cache_import(self.h, blob, stream)
        if self.fp8:  # the scales travel with the checkpoint
            self.scales = sa_cache_get_fp8_scales(self.h, self.H)

    def set_fp8_scales(self, q_scale=None, k_scale=None, v_scale=None):
        """Per-head scales of an e4m3 cache (before the first chunk)."""
        sa_cache_set_fp8_scales(self.h, q_scale, k_scale, v_scale)
        for i, x in enumerate((q_scale, k_scale, v_scale)):
            self.scales[i] = 1.0 if x is None else np.asarray(x, dtype=np.float64)

    def set_sink_mode(self, mode: int):
        sa_cache_set_sink_mode(self.h, mode)

    def sink_update(self, k_new, v_new, alpha: float = 1.0, active=None, stream=None):
        """Blends new data into the sink (k_new, v_new: [B, S*F, H, D])."""
        shape = (self.B, self.cfg.sink_frames * self.F, self.H, self.D)
        for t, n in ((k_new, "k_new"), (v_new, "v_new")):
            if t.device != self.device or t.dtype != self.dtype or not t.is_contiguous() or \
                    tuple(t.shape) != shape:
                raise ValueError(f"{n} must be a contiguous {self.dtype} tensor of shape {shape}")
        sa_sink_update(self.h, k_new, v_new, alpha, active, stream, self.B)

    def append_attend_host(self, q, k, v, out, active=None, stream=None):
        sa_append_attend_host(self.h, q, k, v, out, active, stream)

    def rope_refresh(self, active=None, stream=None):
        sa_rope_refresh(self.h, active, self.B, stream)

    def reset(self, streams=None):
        sa_cache_reset(self.h, streams, self.B)

    def state(self, b: int):
        return sa_stream_state(self.h, b)

    def copy_out(self, b: int):
        """(K', V) of stream b as float32 numpy arrays [H, (S+R)F, D]."""
        shape = (self.H, self.ntok, self.D)
        if self.fp8:  # e4m3 bytes, scaled by the head's k or v scale
            kb = np.empty(shape, np.uint8)
            vb = np.empty(shape, np.uint8)
            sa_cache_copy_out(self.h, b, kb, vb)
            dec = lambda x: torch.from_numpy(x).view(torch.float8_e4m3fn).float().numpy()  # noqa: E731
            return (dec(kb) / self.scales[1][:, None, None]).astype(np.float64), \
                (dec(vb) / self.scales[2][:, None, None]).astype(np.float64)
        if self.cfg.dtype == SA_BF16:
            kb = np.empty(shape, np.uint16)
            vb = np.empty(shape, np.uint16)
            sa_cache_copy_out(self.h, b, kb, vb)
            f = lambda x: (x.astype(np.uint32) << 16).view(np.float32)  # noqa: E731
            return f(kb), f(vb)
        kf = np.empty(shape, np.float32)
        vf = np.empty(shape, np.float32)
        sa_cache_copy_out(self.h, b, kf, vf)
        return kf, vf

    def device_status(self, stream=None) -> int:
        return sa_get_device_status(self.h, stream)

    def profile_begin(self):
        sa_profile_begin(self.h)

    def profile_end(self):
        return sa_profile_end(self.h)

    def profile_launches(self) -> int:
        return sa_profile_launches(self.h)

    def close(self):
        if self.h:
            sa_cache_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def attention_flops(cfg: sa_config, n_keys: int) -> float:
    """Algorithmic FLOPs of one (stream, chunk): 4 * Lc * n_keys * D * H (QK^T and PV)."""
    Lc = cfg.chunk_frames * cfg.frame_h * cfg.frame_w
    return 4.0 * Lc * n_keys * cfg.head_dim * cfg.heads


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
