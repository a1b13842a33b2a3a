"""Shared helpers of the test suite: running the CUDA path through the C ABI and
comparing it with the oracle.  Tolerances: bf16 inputs with fp32 accumulation must come
within max-abs 2e-2 and relative Frobenius 1e-2 of the fp64 oracle; LSE within 1e-3."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from block_sparse_spatio_attn_b200 import configs as C

MAX_ABS = 2e-2
REL_FRO = 1e-2
LSE_ABS = 1e-3


def problem_of(wl, order=None, tile_q=None, tile_k=None):
    from block_sparse_spatio_attn_b200 import svga
    return svga.ProblemSpec.from_workload(wl, order=order, tile_q=tile_q, tile_k=tile_k)


def run_sparse_path(wl, q, k, v, naive=False, order=None, tile_q=None, tile_k=None,
                    with_lse=True, flags=None):
    """Frame-major Q/K/V on the GPU -> permute -> block-sparse attention -> unpermute.
    flags overrides `naive` when given.
    Returns (O frame-major bf16 [H,N,d], LSE in each head's order [H,N] or None, map)."""
    from block_sparse_spatio_attn_b200 import svga
    prob = problem_of(wl, order, tile_q, tile_k)
    bmap = svga.build_block_map(prob)
    qp, kp, vp = (torch.empty_like(x) for x in (q, k, v))
    for s, d in ((q, qp), (k, kp), (v, vp)):
        svga.svga_permute_tokens(s, d, prob)
    op = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device) \
        if with_lse else None
    if flags is None:
        flags = svga.FLAG_NAIVE_B1 if naive else 0
    svga.svga_sparse_attention_fwd(qp, kp, vp, op, lse, prob, bmap,
                                   1.0 / math.sqrt(wl.head_dim), flags)
    o = torch.empty_like(q)
    svga.svga_unpermute_tokens(op, o, prob)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0, f"device status {bmap.device_status()}"
    return o, lse, bmap


def lse_to_frame_major(lse: np.ndarray, wl, order) -> np.ndarray:
    """Reorder per-head LSE [H, N] from each head's token order to frame-major."""
    F, S = wl.frames, wl.tokens_per_frame
    out = np.empty_like(lse)
    for h in range(lse.shape[0]):
        perm = oracle.permutation(order[h], F, S)   # position -> frame-major token
        out[h, perm] = lse[h]
    return out


def oracle_rows(wl, q, k, v, h, rows, type_=None, band=None):
    """Oracle O, LSE of head h for frame-major rows (inputs are CPU bf16 tensors)."""
    F, S = wl.frames, wl.tokens_per_frame
    t = wl.head_type[h] if type_ is None else type_
    w = wl.band[h] if band is None else band
    return oracle.attention_rows(q[h].float().numpy(), k[h].float().numpy(),
                                 v[h].float().numpy(), F, S, 1.0 / math.sqrt(wl.head_dim),
                                 t, w, wl.anchor_frame0, np.asarray(rows, np.int32))


def oracle_rows_tile_aligned(wl, q, k, v, h, rows, order, tq, tk):
    """Oracle O, LSE of head h under the tile-aligned (snapped) mask, for frame-major
    rows; the kept-element counts are taken for each group of rows sharing a q-tile."""
    F, S = wl.frames, wl.tokens_per_frame
    rows = np.asarray(rows, np.int32)
    qt = oracle.q_tiles_of_rows(order, F, S, tq, rows)
    o = np.empty((rows.size, wl.head_dim))
    lse = np.empty(rows.size)
    args = [x[h].float().numpy() for x in (q, k, v)]
    for i in np.unique(qt):
        sel = np.nonzero(qt == i)[0]
        counts = oracle.tile_counts_range(wl.head_type[h], wl.band[h], wl.anchor_frame0, order,
                                          F, S, tq, tk, int(i), int(i) + 1)
        o[sel], lse[sel] = oracle.attention_rows_tile_aligned(
            *args, F, S, 1.0 / math.sqrt(wl.head_dim), order, tq, tk, counts, int(i),
            rows[sel])
    return o, lse


def assert_attn_close(o_gpu: np.ndarray, o_ref: np.ndarray, lse_gpu=None, lse_ref=None,
                      what=""):
    o_gpu = np.asarray(o_gpu, np.float64)
    diff = o_gpu - o_ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(o_ref), 1e-30))
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {MAX_ABS}"
    assert rel <= REL_FRO, f"{what}: rel-Frobenius {rel:.3e} > {REL_FRO}"
    if lse_gpu is not None:
        lerr = float(np.abs(np.asarray(lse_gpu, np.float64) - lse_ref).max())
        assert lerr <= LSE_ABS, f"{what}: LSE max-abs {lerr:.3e} > {LSE_ABS}"
    return max_abs, rel


def kernel_blocks(N: int) -> list:
    """Indices of the 128-row query blocks a row sample covers whole: the first work item
    (blocks 0 and 1: one block per softmax warpgroup), a middle pair (an even and the odd
    block after it), and the last two blocks (the ragged last block and its neighbour)."""
    nb = -(-N // 128)
    mid = (nb // 2) // 2 * 2
    return sorted({b for b in (0, 1, mid, mid + 1, nb - 2, nb - 1) if 0 <= b < nb})


def block_rows(wl, orders=None) -> np.ndarray:
    """Frame-major tokens of every row of kernel_blocks(N), for each token order in
    `orders` (default: the orders of the workload's heads).  A query block is a run of
    128 consecutive positions of the head's order, so for a temporal-major head its rows
    are scattered over the frame-major tokens."""
    N, F, S = wl.tokens, wl.frames, wl.tokens_per_frame
    orders = sorted(set(wl.order if orders is None else orders))
    rows = set()
    for od in orders:
        perm = oracle.permutation(od, F, S)   # position -> frame-major token
        for b in kernel_blocks(N):
            rows.update(perm[b * 128: min(N, b * 128 + 128)].tolist())
    return np.array(sorted(rows), np.int32)


def sample_rows(wl, per_head: int = 160, seed: int = 0, orders=None) -> np.ndarray:
    """Deterministic row sample (frame-major tokens): every row of the whole 128-row
    query blocks of kernel_blocks(N) in each head's token order (block_rows: all 128 TMEM
    lanes of both softmax warpgroups, and the ragged last block), the last 16 tokens,
    plus `per_head` spread rows."""
    N = wl.tokens
    rng = np.random.default_rng(seed)
    rows = set(block_rows(wl, orders).tolist())
    rows.update(range(max(0, N - 16), N))
    rows.update(rng.choice(N, size=min(N, per_head), replace=False).tolist())
    return np.array(sorted(rows), np.int32)
