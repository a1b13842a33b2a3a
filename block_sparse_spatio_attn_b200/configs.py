"""The five synthetic workloads of the block-sparse spatio-temporal attention study.

Each workload is a video token grid (frames x patch rows x patch cols), a list of
heads with their type (spatial or temporal), band width and token order, the head
dimension, the tile size of the block map and the seed of the inputs.

Where the numbers come from:
  * 75,600 tokens, 10 heads, head dim 128 and synthetic BF16 inputs are the
    measurement setup of "Accelerating Spatio-Temporal Attention for Video Diffusion
    on TPUs" as summarised on the aihirek.info page (section "A TPU-kernel
    kialakitasa dontonek bizonyult") and the oossa.com page ("Die Fakten").
  * Spatial heads look at nearby frames, temporal heads at a small in-frame region
    over many frames, both keep the first frame as an anchor (aihirek.info, section
    "A Sparse VideoGen a figyelmi fejeket osztalyozza").
  * 81-frame 720p video gives 50K-400K tokens; 2K is 4x the 720p length (aihirek.info,
    "A lenyeg roviden" and the bottleneck section) -- hence the 302,400-token case.
  * The pages give no band widths; the widths below are this library's fixed choice.

This module holds parameters only, no arithmetic of the method.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List

SPATIAL = 0
TEMPORAL = 1

ORDER_FRAME_MAJOR = 0
ORDER_TEMPORAL_MAJOR = 1          # anchor-first temporal-major (frame 0 first, then s-major)
ORDER_TEMPORAL_MAJOR_STRICT = 2   # literal s*F + f


@dataclass
class Workload:
    name: str
    frames: int
    grid_h: int
    grid_w: int
    head_dim: int
    head_type: List[int]
    band: List[int]
    order: List[int]
    seed: int
    tile_q: int = 128
    tile_k: int = 128
    anchor_frame0: int = 1
    structured: bool = False          # low-rank position bias (2K classification case)
    classify_fraction: float = 0.0    # fraction of query rows the head classifier samples
    cand_spatial: List[int] = field(default_factory=list)   # classifier candidate widths
    cand_temporal: List[int] = field(default_factory=list)

    @property
    def heads(self) -> int:
        return len(self.head_type)

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def tokens(self) -> int:
        return self.frames * self.grid_h * self.grid_w

    def with_orders(self, order: int) -> "Workload":
        """Same workload with every temporal head in `order` (spatial heads stay frame-major)."""
        o = [order if t == TEMPORAL else ORDER_FRAME_MAJOR for t in self.head_type]
        w = Workload(**{**self.__dict__})
        w.order = o
        return w

    def with_tile(self, tq: int, tk: int) -> "Workload":
        w = Workload(**{**self.__dict__})
        w.tile_q, w.tile_k = tq, tk
        return w


def tiny() -> Workload:
    """3 frames x 8x8 grid = 192 tokens, 2 heads, d=64, tile 64x64, frame-major."""
    return Workload("tiny_192tok_2h_d64", 3, 8, 8, 64,
                    [SPATIAL, TEMPORAL], [1, 8],
                    [ORDER_FRAME_MAJOR, ORDER_FRAME_MAJOR], seed=0, tile_q=64, tile_k=64)


def mid() -> Workload:
    """13 frames x 24x40 = 12,480 tokens, 2 spatial (|df|<=2) + 2 temporal (|ds|<=160) heads."""
    return Workload("mid_12480tok_4h_d128", 13, 24, 40, 128,
                    [SPATIAL, SPATIAL, TEMPORAL, TEMPORAL], [2, 2, 160, 160],
                    [ORDER_FRAME_MAJOR, ORDER_FRAME_MAJOR,
                     ORDER_TEMPORAL_MAJOR, ORDER_TEMPORAL_MAJOR], seed=1)


def headline() -> Workload:
    """21 frames x 45x80 = 75,600 tokens, 5 spatial (|df|<=3) + 5 temporal (|ds|<=600) heads."""
    return Workload("headline_75600tok_10h_d128", 21, 45, 80, 128,
                    [SPATIAL] * 5 + [TEMPORAL] * 5, [3] * 5 + [600] * 5,
                    [ORDER_FRAME_MAJOR] * 5 + [ORDER_TEMPORAL_MAJOR] * 5, seed=2)


def permutation_study(order: int = ORDER_TEMPORAL_MAJOR) -> Workload:
    """75,600 tokens, all 10 heads temporal (|ds|<=600), in the given token order."""
    return Workload("permstudy_75600tok_10T_d128", 21, 45, 80, 128,
                    [TEMPORAL] * 10, [600] * 10, [order] * 10, seed=3)


def twok() -> Workload:
    """21 frames x 90x160 = 302,400 tokens, 10 heads with structured inputs; the head
    types come from the online classifier (1% of query rows per head)."""
    return Workload("2k_302400tok_10h_d128", 21, 90, 160, 128,
                    [SPATIAL] * 5 + [TEMPORAL] * 5, [3] * 5 + [2400] * 5,
                    [ORDER_FRAME_MAJOR] * 5 + [ORDER_TEMPORAL_MAJOR] * 5, seed=4,
                    structured=True, classify_fraction=0.01,
                    cand_spatial=[3] * 10, cand_temporal=[2400] * 10)


ALL = {"tiny": tiny, "mid": mid, "headline": headline,
       "permstudy": permutation_study, "2k": twok}
