"""Binding of sa_gdn_chunk, the Gated DeltaNet block (argument marshalling only;
the recurrence runs in the library's CUDA kernel).

Per stream b and head h, over the call's tokens in order (k and q divided by
their norms):  S <- exp(g_t) S (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
o_t = scale S q_t, with S [D (value), D (key)] fp32 kept by the caller.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from ._lib import SA_BF16, SA_F32, check, lib, sa_gdn_config

_DT = {torch.float32: SA_F32, torch.bfloat16: SA_BF16}


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def sa_gdn_chunk(state: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 g: torch.Tensor, beta: torch.Tensor, out: torch.Tensor, scale: float = 0.0,
                 active=None, stream: Optional[torch.cuda.Stream] = None) -> None:
    """q, k, v, out [B, T, H, D] (fp32 or bf16, contiguous, on the GPU); g, beta
    [B, T, H] fp32; state [B, H, D, D] fp32, updated in place."""
    B, T, H, D = q.shape
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, q.shape, q.dtype),
                               ("out", out, q.shape, q.dtype), ("g", g, (B, T, H), torch.float32),
                               ("beta", beta, (B, T, H), torch.float32),
                               ("state", state, (B, H, D, D), torch.float32)):
        if tuple(t.shape) != tuple(shape) or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name}: expected contiguous {dt} {tuple(shape)}, got "
                             f"{t.dtype} {tuple(t.shape)}")
    if q.dtype not in _DT or not q.is_contiguous():
        raise ValueError("q must be contiguous fp32 or bf16")
    c = sa_gdn_config()
    c.batch, c.heads, c.head_dim, c.dtype = B, H, D, _DT[q.dtype]
    c.tokens, c.scale = T, scale
    mask = None if active is None else (ctypes.c_uint8 * B)(*[1 if a else 0 for a in active])
    check(lib().sa_gdn_chunk(ctypes.byref(c), state.data_ptr(), q.data_ptr(), k.data_ptr(),
                             v.data_ptr(), g.data_ptr(), beta.data_ptr(), out.data_ptr(), mask,
                             ctypes.c_void_p(_stream_ptr(stream))), "sa_gdn_chunk")


class GDNState:
    """The recurrent state of one GDN block for B streams ([B, H, D, D] fp32,
    zero at the start of each stream)."""

    def __init__(self, batch: int, heads: int, head_dim: int, device=None):
        self.state = torch.zeros(batch, heads, head_dim, head_dim, dtype=torch.float32,
                                 device=device or "cuda")

    def reset(self, streams=None) -> None:
        if streams is None:
            self.state.zero_()
        else:
            for b in streams:
                self.state[b].zero_()

    def step(self, q, k, v, g, beta, out, scale: float = 0.0, active=None, stream=None) -> None:
        sa_gdn_chunk(self.state, q, k, v, g, beta, out, scale, active, stream)
