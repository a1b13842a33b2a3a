"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

Recipe (the same for the CUDA path and the oracle; nothing here computes attention):
  * one CPU ``torch.Generator`` seeded with the workload's seed;
  * Q, then K, then V; for each tensor, head by head, a ``[tokens, d]`` fp32 draw
    from N(0, 1), rounded to bf16;
  * tokens are in frame-major order (token t is frame t // S, in-frame index t % S);
  * structured workloads add a low-rank position bias to Q and K before rounding:
    heads of the first half get beta * U_h @ phi(f), heads of the second half get
    beta * U_h @ phi(s / sigma), with U_h a random orthonormal d x 8 basis (QR of a
    Gaussian draw from the same generator, taken before Q), phi(x) =
    [cos(w_j x), sin(w_j x)]_{j=1..4}, w_j = j * pi / 8 and sigma = temporal band / 4.
    This gives heads that favour frame-local keys and heads that favour same-position
    keys, so the head classifier has a right answer to find.

The pages measure on synthetic BF16 inputs ("Accelerating Spatio-Temporal Attention for
Video Diffusion on TPUs", aihirek.info summary, "A lenyeg roviden"); no public data set
is involved.
"""
from __future__ import annotations

import math
from typing import Tuple

import torch

from .configs import Workload

STRUCT_BETA = 3.0
STRUCT_RANK = 8


def _position_features(x: torch.Tensor) -> torch.Tensor:
    """phi(x) = [cos(w_j x), sin(w_j x)] for w_j = j*pi/8, j = 1..4  -> [len(x), 8]."""
    w = torch.arange(1, 5, dtype=torch.float64) * (math.pi / 8.0)
    ang = x.to(torch.float64)[:, None] * w[None, :]
    return torch.cat([torch.cos(ang), torch.sin(ang)], dim=1)


def make_qkv(wl: Workload, device: str | torch.device = "cpu",
             heads: int | None = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q, K, V as bf16 ``[heads, tokens, d]`` in frame-major order on `device`."""
    H = wl.heads if heads is None else heads
    N, d, S = wl.tokens, wl.head_dim, wl.tokens_per_frame
    g = torch.Generator(device="cpu").manual_seed(wl.seed)
    bases = None
    if wl.structured:
        bases = []
        for _ in range(wl.heads):
            a = torch.randn(d, STRUCT_RANK, generator=g, dtype=torch.float32).double()
            qmat, _ = torch.linalg.qr(a)
            bases.append(qmat)
        t = torch.arange(N, dtype=torch.int64)
        feat_f = _position_features((t // S).double())
        half = wl.heads // 2
    out = []
    for ti in range(3):
        x = torch.empty(H, N, d, dtype=torch.bfloat16, device=device)
        for h in range(H):
            r = torch.randn(N, d, generator=g, dtype=torch.float32)
            if bases is not None and ti < 2:
                if h < half:
                    feat = feat_f
                else:
                    sigma = wl.band[h] / 4.0 if wl.band[h] > 0 else 1.0
                    feat = _position_features((t % S).double() / sigma)
                r = (r.double() + STRUCT_BETA * feat @ bases[h].T).float()
            x[h].copy_(r.to(torch.bfloat16))
        out.append(x)
    return out[0], out[1], out[2]


def default_sample_rows(tokens: int, n: int) -> torch.Tensor:
    """Evenly spread query rows r_i = floor((2i+1) * N / (2n)), i = 0..n-1 (int32)."""
    i = torch.arange(n, dtype=torch.int64)
    return ((2 * i + 1) * tokens // (2 * n)).to(torch.int32)
