"""Synthetic streaming workloads for the rolling KV-cache attention path.

Pure data: shapes, value recipes and the streaming schedule. No arithmetic of
the attention method lives here.

Token grids follow the video resolutions the pages run at, divided by the
16x spatial compression of a latent video DiT: 512p -> 32x32 (StreamDiT,
abstract), 480x832 -> 30x52 (StreamDiffusionV2, results: 480p), 1280x704 ->
44x80 (SANA-Streaming, introduction).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Tuple

NORMAL, UNIFORM, ZERO, ONES = 0, 1, 2, 3


def rope_split(D: int) -> Tuple[int, int, int]:
    """3D RoPE band widths (t, h, w): d_h = d_w = 2*floor(D/6), d_t = rest.

    Gives 44/42/42 at D=128 and 24/20/20 at D=64 (every band even, so pairs
    never straddle a band)."""
    dh = 2 * (D // 6)
    return (D - 2 * dh, dh, dh)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    fh: int
    fw: int
    C: int  # frames per chunk
    S: int  # sink frames
    W: int  # window frames
    n_chunks: int  # chunks per stream
    dtype: str  # "f32" or "bf16"
    dist: Tuple[int, int, int] = (NORMAL, NORMAL, NORMAL)
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    seed: int = 0
    rope_dims: Tuple[int, int, int] | None = None
    rope_base: float = 10000.0
    refresh_period: int = 0  # chunks; 0 = never
    starts: Tuple[int, ...] = field(default_factory=tuple)  # global start step per stream
    sink_repin: bool = False  # after a refresh the sink sits right before the window
    sink_update_period: int = 0  # sink update before chunk u (u > 0, u % period == 0); 0 = never
    sink_alpha: float = 1.0  # weight of the new sink data (1 = replace)
    cache: str = ""  # "" = the cache keeps dtype; "e4m3" = bf16 in/out, e4m3 cache and MMAs
    fp8_scales: Tuple = ()  # e4m3 cache: ((q scales per head), (k ...), (v ...)); () = 1

    @property
    def F(self) -> int:
        return self.fh * self.fw

    @property
    def Lc(self) -> int:
        return self.C * self.F

    @property
    def R(self) -> int:
        return self.W + self.C

    @property
    def dims(self) -> Tuple[int, int, int]:
        return self.rope_dims if self.rope_dims is not None else rope_split(self.D)

    @property
    def start_steps(self) -> Tuple[int, ...]:
        return self.starts if self.starts else tuple(0 for _ in range(self.B))

    @property
    def n_steps(self) -> int:
        return max(self.start_steps) + self.n_chunks

    def local_chunks(self, g: int):
        """Local chunk index of each stream at global step g (-1 = inactive)."""
        out = []
        for s in self.start_steps:
            c = g - s
            out.append(c if 0 <= c < self.n_chunks else -1)
        return out

    def refresh_due(self, c: int) -> bool:
        return self.refresh_period > 0 and c > 0 and c % self.refresh_period == 0

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY_F32 = Workload("tiny_fp32_8x8", B=1, H=2, D=64, fh=8, fw=8, C=1, S=1, W=2, n_chunks=8,
                    dtype="f32", refresh_period=4)
P512 = Workload("512p_32x32_h24", B=1, H=24, D=128, fh=32, fw=32, C=2, S=1, W=4, n_chunks=64,
                dtype="bf16", refresh_period=32)
BATCHED_480 = Workload("480x832_30x52_b4_ragged", B=4, H=12, D=128, fh=30, fw=52, C=1, S=1, W=6,
                       n_chunks=128, dtype="bf16", starts=(0, 3, 7, 12))
SANA_1280 = Workload("1280x704_44x80_h16", B=1, H=16, D=128, fh=44, fw=80, C=1, S=1, W=3,
                     n_chunks=256, dtype="bf16", dist=(NORMAL, NORMAL, UNIFORM))
LONG_STRESS = Workload("long_stress_b8_10000", B=8, H=16, D=128, fh=32, fw=32, C=2, S=1, W=8,
                       n_chunks=10000, dtype="bf16", outlier_frac=0.01, outlier_scale=20.0,
                       refresh_period=256, starts=(0, 3, 7, 12, 18, 25, 33, 42))

ALL = (TINY_F32, P512, BATCHED_480, SANA_1280, LONG_STRESS)
BY_NAME = {w.name: w for w in ALL}
