"""fp64 CPU oracle for block-sparse spatio-temporal attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` are the only code that may import this package.  It shares nothing with
the CUDA library and never imports it.

Everything heavy is plain C in ``svga_oracle.c`` (built here with gcc + OpenMP); the
Python side only marshals numpy arrays and applies the classifier's argmin.  Sources of
each definition are given in the C file's header and in the docstrings below.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svga_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

FRAME_MAJOR, TEMPORAL_ANCHOR_FIRST, TEMPORAL_STRICT = 0, 1, 2
SPATIAL, TEMPORAL, DENSE = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, IEEE arithmetic: no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I = ctypes.c_int
            LL = ctypes.c_longlong
            lib.orc_position.restype = LL
            lib.orc_position.argtypes = [I, I, I, I, I]
            lib.orc_order_coords.restype = I
            lib.orc_order_coords.argtypes = [I, I, I, P, P]
            lib.orc_keep.restype = I
            lib.orc_keep.argtypes = [I, I, I, I, I, I, I]
            lib.orc_kept_count.restype = LL
            lib.orc_kept_count.argtypes = [I, I, I, I, I]
            lib.orc_mask.restype = None
            lib.orc_mask.argtypes = [I, I, I, I, I, P]
            lib.orc_tile_counts.restype = I
            lib.orc_tile_counts.argtypes = [I, I, I, I, I, I, I, I, P]
            lib.orc_classes_and_lists.restype = None
            lib.orc_classes_and_lists.argtypes = [P, LL, LL, I, I, P, P, P, P, P]
            lib.orc_attention_rows.restype = None
            lib.orc_attention_rows.argtypes = [P, P, P, I, I, I, ctypes.c_double,
                                               I, I, I, P, I, P, P]
            lib.orc_tile_counts_range.restype = I
            lib.orc_tile_counts_range.argtypes = [I, I, I, I, I, I, I, I, LL, LL, P]
            lib.orc_attention_rows_tile_aligned.restype = I
            lib.orc_attention_rows_tile_aligned.argtypes = [P, P, P, I, I, I, ctypes.c_double,
                                                            I, I, I, P, LL, LL, P, I, P, P]
            lib.orc_position_padded.restype = LL
            lib.orc_position_padded.argtypes = [I, I, I, I, I, I]
            lib.orc_order_coords_padded.restype = I
            lib.orc_order_coords_padded.argtypes = [I, I, I, I, P, P]
            lib.orc_tile_counts_padded.restype = I
            lib.orc_tile_counts_padded.argtypes = [I, I, I, I, I, I, I, I, I, P]
            lib.orc_num_threads.restype = I
            lib.orc_num_threads.argtypes = []
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().orc_num_threads()


def position(order: int, F: int, S: int, f: int, s: int) -> int:
    """Position of token (f, s) in `order` (see the C header for the three orders)."""
    return _load().orc_position(order, F, S, f, s)


def order_coords(order: int, F: int, S: int):
    """(f_of_pos, s_of_pos) int32 arrays: the coordinates held at each position."""
    N = F * S
    fp = np.empty(N, np.int32)
    sp = np.empty(N, np.int32)
    rc = _load().orc_order_coords(order, F, S, _ptr(fp), _ptr(sp))
    if rc != 0:
        raise ValueError("order is not a bijection")
    return fp, sp


def permutation(order: int, F: int, S: int) -> np.ndarray:
    """perm[pos] = frame-major token index held at position `pos` of `order`."""
    fp, sp = order_coords(order, F, S)
    return fp.astype(np.int64) * S + sp


def frame_stride(S: int, frame_pad: int) -> int:
    """Sp: S rounded up to a multiple of frame_pad (S itself when frame_pad is 0)."""
    return S if frame_pad == 0 else -(-S // frame_pad) * frame_pad


def position_padded(order: int, F: int, S: int, Sp: int, f: int, s: int) -> int:
    """Position of token (f, s) in the padded layout (frame-major frames at stride Sp)."""
    return _load().orc_position_padded(order, F, S, Sp, f, s)


def permutation_padded(order: int, F: int, S: int, Sp: int) -> np.ndarray:
    """perm[pos] = frame-major token at position `pos` of the padded layout
    (F * Sp positions), -1 where the position holds no token."""
    NP = F * Sp
    fp = np.empty(NP, np.int32)
    sp = np.empty(NP, np.int32)
    rc = _load().orc_order_coords_padded(order, F, S, Sp, _ptr(fp), _ptr(sp))
    if rc != 0:
        raise ValueError(f"padded layout invalid ({rc})")
    perm = fp.astype(np.int64) * S + sp
    perm[fp < 0] = -1
    return perm


def tile_map_padded(type_: int, band: int, anchor: int, order: int, F: int, S: int, Sp: int,
                    tq: int, tk: int) -> dict:
    """tile_map of one head in the padded layout: classes and lists over the F * Sp
    positions, by counting kept elements (positions without a token keep nothing, so a
    tile holding one is never full)."""
    NP = F * Sp
    nq, nk = -(-NP // tq), -(-NP // tk)
    counts = np.empty(nq * nk, np.int64)
    rc = _load().orc_tile_counts_padded(type_, band, anchor, order, F, S, Sp, tq, tk,
                                        _ptr(counts))
    if rc != 0:
        raise RuntimeError(f"orc_tile_counts_padded failed ({rc})")
    cls = np.empty(nq * nk, np.uint8)
    fptr = np.empty(nq + 1, np.int32)
    bptr = np.empty(nq + 1, np.int32)
    fidx = np.empty(nq * nk, np.int32)
    bidx = np.empty(nq * nk, np.int32)
    _load().orc_classes_and_lists(_ptr(counts), nq, nk, tq, tk, _ptr(cls), _ptr(fptr),
                                  _ptr(fidx), _ptr(bptr), _ptr(bidx))
    return {"counts": counts.reshape(nq, nk), "cls": cls.reshape(nq, nk),
            "full_ptr": fptr, "full_idx": fidx[: fptr[-1]].copy(),
            "bnd_ptr": bptr, "bnd_idx": bidx[: bptr[-1]].copy(), "n_q": nq, "n_k": nk}


def keep(type_: int, band: int, anchor: int, fq: int, sq: int, fk: int, sk: int) -> bool:
    return bool(_load().orc_keep(type_, band, anchor, fq, sq, fk, sk))


def kept_count(type_: int, band: int, anchor: int, F: int, S: int) -> int:
    """Kept (q, k) pairs of one head, counted pair by pair."""
    return int(_load().orc_kept_count(type_, band, anchor, F, S))


def mask(type_: int, band: int, anchor: int, F: int, S: int) -> np.ndarray:
    """Element mask [N, N] (uint8) in frame-major order.  Small N only."""
    N = F * S
    m = np.empty((N, N), np.uint8)
    _load().orc_mask(type_, band, anchor, F, S, _ptr(m))
    return m


def tile_map(type_: int, band: int, anchor: int, order: int, F: int, S: int,
             tq: int, tk: int) -> dict:
    """Tile classes and per-q-tile CSR lists of one head, by counting kept elements."""
    N = F * S
    nq, nk = -(-N // tq), -(-N // tk)
    counts = np.empty(nq * nk, np.int64)
    rc = _load().orc_tile_counts(type_, band, anchor, order, F, S, tq, tk, _ptr(counts))
    if rc != 0:
        raise RuntimeError(f"orc_tile_counts failed ({rc})")
    cls = np.empty(nq * nk, np.uint8)
    fptr = np.empty(nq + 1, np.int32)
    bptr = np.empty(nq + 1, np.int32)
    fidx = np.empty(nq * nk, np.int32)
    bidx = np.empty(nq * nk, np.int32)
    _load().orc_classes_and_lists(_ptr(counts), nq, nk, tq, tk, _ptr(cls), _ptr(fptr),
                                  _ptr(fidx), _ptr(bptr), _ptr(bidx))
    return {"counts": counts.reshape(nq, nk), "cls": cls.reshape(nq, nk),
            "full_ptr": fptr, "full_idx": fidx[: fptr[-1]].copy(),
            "bnd_ptr": bptr, "bnd_idx": bidx[: bptr[-1]].copy(), "n_q": nq, "n_k": nk}


def tile_counts_range(type_: int, band: int, anchor: int, order: int, F: int, S: int,
                      tq: int, tk: int, i0: int, i1: int) -> np.ndarray:
    """Kept-element counts [i1 - i0, n_k] of the q-tiles i0 <= i < i1 of one head."""
    N = F * S
    nk = -(-N // tk)
    counts = np.empty((i1 - i0) * nk, np.int64)
    rc = _load().orc_tile_counts_range(type_, band, anchor, order, F, S, tq, tk, i0, i1,
                                       _ptr(counts))
    if rc != 0:
        raise RuntimeError(f"orc_tile_counts_range failed ({rc})")
    return counts.reshape(i1 - i0, nk)


def q_tiles_of_rows(order: int, F: int, S: int, tq: int, rows) -> np.ndarray:
    """q-tile index (position in `order` // tq) of each frame-major token in rows."""
    return np.array([position(order, F, S, int(t) // S, int(t) % S) // tq for t in rows],
                    np.int64)


def attention_rows_tile_aligned(q: np.ndarray, k: np.ndarray, v: np.ndarray, F: int, S: int,
                                scale: float, order: int, tq: int, tk: int,
                                counts: np.ndarray, i0: int, rows: np.ndarray):
    """Tile-aligned (B3) attention of one head: the mask snapped to tiles, i.e. a query
    keeps every key of each tile (in the head's token order) that holds a kept pair.
    counts: [n, n_k] kept-element counts of q-tiles i0 .. i0 + n - 1, covering the rows'
    q-tiles (tile_counts_range / tile_map).  Returns (O [n, d], LSE [n]) in float64."""
    q = np.ascontiguousarray(q, dtype=np.float32)
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int64)
    n, d = rows.shape[0], q.shape[1]
    o = np.empty((n, d), np.float64)
    lse = np.empty(n, np.float64)
    rc = _load().orc_attention_rows_tile_aligned(
        _ptr(q), _ptr(k), _ptr(v), F, S, d, float(scale), order, tq, tk, _ptr(counts), i0,
        counts.shape[0], _ptr(rows), n, _ptr(o), _ptr(lse))
    if rc != 0:
        raise RuntimeError(f"orc_attention_rows_tile_aligned failed ({rc})")
    return o, lse


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, F: int, S: int,
                   scale: float, type_: int, band: int, anchor: int,
                   rows: np.ndarray):
    """Masked softmax(scale q k^T) v for the given frame-major query rows of one head.

    q, k, v: [N, d] arrays of bf16 values (any float dtype; converted to float32, which
    holds bf16 exactly).  Returns (O [n, d] float64, LSE [n] float64)."""
    q = np.ascontiguousarray(q, dtype=np.float32)
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    n, d = rows.shape[0], q.shape[1]
    o = np.empty((n, d), np.float64)
    lse = np.empty(n, np.float64)
    _load().orc_attention_rows(_ptr(q), _ptr(k), _ptr(v), F, S, d, float(scale), type_,
                               band, anchor, _ptr(rows), n, _ptr(o), _ptr(lse))
    return o, lse


def classify(q: np.ndarray, k: np.ndarray, v: np.ndarray, F: int, S: int, scale: float,
             w_spatial: int, w_temporal: int, anchor: int, rows: np.ndarray):
    """Online head profiling of one head, as the aihirek.info summary describes it
    (section "A Sparse VideoGen a figyelmi fejeket osztalyozza"): on a few query rows
    compute the dense, the spatial and the temporal outputs and pick the sparse mask
    whose output deviates least from the dense one.  Deviation = mean squared error
    over the sampled rows x d; a tie goes to spatial.

    Returns (type, mse_spatial, mse_temporal)."""
    od, _ = attention_rows(q, k, v, F, S, scale, DENSE, 0, anchor, rows)
    os_, _ = attention_rows(q, k, v, F, S, scale, SPATIAL, w_spatial, anchor, rows)
    ot, _ = attention_rows(q, k, v, F, S, scale, TEMPORAL, w_temporal, anchor, rows)
    ms = float(np.mean((os_ - od) ** 2))
    mt = float(np.mean((ot - od) ** 2))
    return (SPATIAL if ms <= mt else TEMPORAL), ms, mt


def select_band(q: np.ndarray, k: np.ndarray, v: np.ndarray, F: int, S: int, scale: float,
                candidates, anchor: int, rows: np.ndarray, max_kept_fraction: float):
    """Per-head choice among candidate masks (type, band), extending the online profiling
    the aihirek.info summary describes (section "A Sparse VideoGen a figyelmi fejeket
    osztalyozza": keep the mask whose output deviates least from dense on a few query
    rows) to several bands.  The pages give no cost rule, so a candidate is eligible when
    its kept-pair fraction (counted pair by pair) is at most max_kept_fraction; among the
    eligible ones the least mean squared deviation wins, the earlier on a tie.

    Returns (index of the chosen candidate or -1, [mse per candidate],
    [kept fraction per candidate])."""
    N = F * S
    od, _ = attention_rows(q, k, v, F, S, scale, DENSE, 0, anchor, rows)
    mses, fracs = [], []
    best = -1
    for i, (t, w) in enumerate(candidates):
        ox, _ = attention_rows(q, k, v, F, S, scale, t, w, anchor, rows)
        mses.append(float(np.mean((ox - od) ** 2)))
        fracs.append(kept_count(t, w, anchor, F, S) / float(N * N))
        if fracs[-1] <= max_kept_fraction and (best < 0 or mses[-1] < mses[best]):
            best = i
    return best, mses, fracs

