"""Streaming session: applies the refresh policy before each append.

StreamDiffusionV2 (technical summary, section 2.A.2) resets RoPE offsets
periodically at block boundaries; here a stream is refreshed right before its
chunk c whenever c > 0 and c % refresh_period == 0. Host bookkeeping only.
"""
from __future__ import annotations

from typing import Optional, Sequence

from .cache import SACache, sa_refresh_delta


class StreamSession:
    def __init__(self, cache: SACache, refresh_period: int = 0):
        self.cache = cache
        self.period = refresh_period
        self.C = cache.cfg.chunk_frames

    def next_chunk(self, b: int) -> int:
        fw, _ = self.cache.state(b)
        return fw // self.C

    def refresh_mask(self, active: Optional[Sequence[bool]]):
        if self.period <= 0:
            return None
        mask = []
        for b in range(self.cache.B):
            on = active is None or bool(active[b])
            fw, base = self.cache.state(b)
            c = fw // self.C
            # a refresh whose offset is already 0 (the chunk's uncommitted
            # steps refreshed it) changes nothing and is skipped
            due = on and c > 0 and c % self.period == 0 and \
                sa_refresh_delta(self.cache.cfg, fw, base) != 0
            mask.append(due)
        return mask if any(mask) else None

    def step(self, q, k, v, out, active: Optional[Sequence[bool]] = None, stream=None):
        """One streamed chunk for every active stream: refresh if due, then
        the fused append + attention."""
        mask = self.refresh_mask(active)
        if mask is not None:
            self.cache.rope_refresh(mask, stream)
        self.cache.append_attend(q, k, v, out, active, stream)

    def step_uncommitted(self, q, k, v, out, active: Optional[Sequence[bool]] = None,
                         stream=None):
        """A denoising step of the next chunk that is not kept: refresh if due
        (the chunk's later steps then find nothing to rebase), then attention over the cached context and this
        step's keys and values without advancing the streams."""
        mask = self.refresh_mask(active)
        if mask is not None:
            self.cache.rope_refresh(mask, stream)
        self.cache.attend(q, k, v, out, active, stream)

    def step_host_async(self, q, k, v, out, active: Optional[Sequence[bool]] = None,
                        stream=None):
        """Same as step_host, queued without waiting (pipelined copies); call
        cache.host_wait() before reading out."""
        mask = self.refresh_mask(active)
        if mask is not None:
            self.cache.rope_refresh(mask, stream)
        self.cache.append_attend_host_async(q, k, v, out, active, stream)

    def step_host(self, q, k, v, out, active: Optional[Sequence[bool]] = None, stream=None):
        """Same as step with host tensors (copies inside the call)."""
        mask = self.refresh_mask(active)
        if mask is not None:
            self.cache.rope_refresh(mask, stream)
        self.cache.append_attend_host(q, k, v, out, active, stream)
