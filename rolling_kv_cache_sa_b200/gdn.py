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


_WORKSPACES: dict = {}


def _config(B: int, T: int, H: int, D: int, dtype, scale: float) -> sa_gdn_config:
    c = sa_gdn_config()
    c.batch, c.heads, c.head_dim, c.dtype = B, H, D, _DT[dtype]
    c.tokens, c.scale = T, scale
    return c


def sa_gdn_workspace_size(batch: int, tokens: int, heads: int, head_dim: int,
                          dtype=torch.bfloat16) -> int:
    """Bytes of device workspace sa_gdn_chunk needs for these sizes."""
    n = ctypes.c_size_t()
    check(lib().sa_gdn_workspace_size(ctypes.byref(_config(batch, tokens, heads, head_dim, dtype,
                                                            0.0)), ctypes.byref(n)),
          "sa_gdn_workspace_size")
    return n.value


def gdn_workspace(batch: int, tokens: int, heads: int, head_dim: int, device=None) -> torch.Tensor:
    """A device buffer large enough for sa_gdn_chunk with these sizes."""
    n = sa_gdn_workspace_size(batch, tokens, heads, head_dim)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device or "cuda")


def sa_gdn_chunk(state: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 g: torch.Tensor, beta: torch.Tensor, out: torch.Tensor, scale: float = 0.0,
                 active=None, stream: Optional[torch.cuda.Stream] = None,
                 workspace: Optional[torch.Tensor] = None) -> None:
    """q, k, v, out [B, T, H, D] (fp32 or bf16, contiguous, on the GPU); g, beta
    [B, T, H] fp32; state [B, H, D, D] fp32, updated in place. workspace: a
    device buffer of at least sa_gdn_workspace_size bytes; when omitted, a
    buffer kept per device and grown as needed is used (do not omit it inside
    a CUDA-graph capture that must not allocate)."""
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
    c = _config(B, T, H, D, q.dtype, scale)
    need = sa_gdn_workspace_size(B, T, H, D)
    if workspace is None:
        key = q.device
        ws = _WORKSPACES.get(key)
        if ws is None or ws.numel() < need:
            ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
            _WORKSPACES[key] = ws
        workspace = ws
    mask = None if active is None else (ctypes.c_uint8 * B)(*[1 if a else 0 for a in active])
    check(lib().sa_gdn_chunk(ctypes.byref(c), state.data_ptr(), q.data_ptr(), k.data_ptr(),
                             v.data_ptr(), g.data_ptr(), beta.data_ptr(), out.data_ptr(),
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             mask, ctypes.c_void_p(_stream_ptr(stream))), "sa_gdn_chunk")


def sa_gdn_device_status(workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None):
    """Raises SAError(SA_ERR_DEVICE_TIMEOUT) if a bounded wait of the last call
    that used this workspace gave up (synchronises the stream)."""
    check(lib().sa_gdn_device_status(workspace.data_ptr(), ctypes.c_void_p(_stream_ptr(stream))),
          "sa_gdn_device_status")


class GDNState:
    """The recurrent state of one GDN block for B streams ([B, H, D, D] fp32,
    zero at the start of each stream) and a workspace for calls of up to
    max_tokens tokens."""

    def __init__(self, batch: int, heads: int, head_dim: int, device=None,
                 max_tokens: int = 4096):
        self.state = torch.zeros(batch, heads, head_dim, head_dim, dtype=torch.float32,
                                 device=device or "cuda")
        self.workspace = gdn_workspace(batch, max_tokens, heads, head_dim, device)

    def reset(self, streams=None) -> None:
        if streams is None:
            self.state.zero_()
        else:
            for b in streams:
                self.state[b].zero_()

    def step(self, q, k, v, g, beta, out, scale: float = 0.0, active=None, stream=None) -> None:
        need = sa_gdn_workspace_size(q.shape[0], q.shape[1], q.shape[2], q.shape[3])
        if self.workspace.numel() < need:
            self.workspace = torch.empty(need, dtype=torch.uint8, device=self.state.device)
        sa_gdn_chunk(self.state, q, k, v, g, beta, out, scale, active, stream, self.workspace)
