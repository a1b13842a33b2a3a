"""Pins of the oracle's padded layout, the exact reading of the tile-aligned traversal
(B3: ainews.tenesys.com, "Co sie zmienilo?" item 4; oossa.com, opening paragraph: the
mask is aligned with the tiles the kernel computes).  Frame-major frames are laid out
with a stride Sp (S rounded up to whole tiles); temporal-major heads keep their order.
The layout changes which pairs share a tile, never which pairs are kept.  CPU only.

What pins it, independently of the C loops under test:
  * the layout's defining properties: each frame is one run starting at a multiple of
    Sp, every token appears once, and removing the empty positions gives the unpadded
    order (itself pinned in test_oracle.py);
  * tile counts against a block sum of the element mask (oracle.mask, pinned pair by
    pair) scattered to the padded positions, and their total against the kept count;
  * the reading's purpose: with Sp a multiple of both tiles, no tile of a frame-major
    spatial head is cut by a frame boundary: every tile keeps all of its token pairs or
    none;
  * a hand-derived class matrix (docstring of test_class_matrix_by_hand).
"""
import numpy as np
import pytest

import oracle

FM, AF, ST = oracle.FRAME_MAJOR, oracle.TEMPORAL_ANCHOR_FIRST, oracle.TEMPORAL_STRICT
SP, TP = oracle.SPATIAL, oracle.TEMPORAL

SHAPES = [(3, 5, 8), (4, 6, 8), (5, 7, 16), (2, 9, 16), (3, 16, 16), (6, 10, 12)]


@pytest.mark.parametrize("F,S,Sp", SHAPES)
@pytest.mark.parametrize("order", [FM, AF, ST])
def test_layout_properties(F, S, Sp, order):
    perm = oracle.permutation_padded(order, F, S, Sp)
    assert perm.shape == (F * Sp,)
    tokens = perm[perm >= 0]
    assert sorted(tokens.tolist()) == list(range(F * S))           # each token once
    np.testing.assert_array_equal(tokens, oracle.permutation(order, F, S))
    if order == FM:
        for f in range(F):
            run = np.nonzero((perm >= f * S) & (perm < (f + 1) * S))[0]
            assert run[0] == f * Sp and run[0] % Sp == 0               # starts on the stride
            assert np.array_equal(run, np.arange(f * Sp, f * Sp + S))  # one contiguous run
    else:
        assert (perm[: F * S] >= 0).all() and (perm[F * S:] == -1).all()
    for f in range(F):
        for s in range(S):
            assert perm[oracle.position_padded(order, F, S, Sp, f, s)] == f * S + s


def _block_counts(type_, band, anchor, order, F, S, Sp, tq, tk):
    """Kept-pair counts per (q-tile, k-tile) of the padded layout, from the frame-major
    element mask: scatter rows and columns to their positions, then sum blocks."""
    N, NP = F * S, F * Sp
    m = oracle.mask(type_, band, anchor, F, S).astype(np.int64)
    perm = oracle.permutation_padded(order, F, S, Sp)
    big = np.zeros((NP, NP), np.int64)
    pos = np.nonzero(perm >= 0)[0]
    big[np.ix_(pos, pos)] = m[np.ix_(perm[pos], perm[pos])]
    nq, nk = -(-NP // tq), -(-NP // tk)
    pad = np.zeros((nq * tq, nk * tk), np.int64)
    pad[:NP, :NP] = big
    return pad.reshape(nq, tq, nk, tk).sum(axis=(1, 3)), N


@pytest.mark.parametrize("F,S,Sp", SHAPES)
@pytest.mark.parametrize("type_,band,order", [(SP, 0, FM), (SP, 1, FM), (TP, 2, AF),
                                              (TP, 1, ST), (TP, 3, FM), (SP, 2, AF)])
@pytest.mark.parametrize("anchor", [0, 1])
def test_tile_counts_against_block_sums(F, S, Sp, type_, band, order, anchor):
    for tq, tk in ((4, 4), (8, 4), (4, 8)):
        want, _ = _block_counts(type_, band, anchor, order, F, S, Sp, tq, tk)
        m = oracle.tile_map_padded(type_, band, anchor, order, F, S, Sp, tq, tk)
        np.testing.assert_array_equal(m["counts"], want)
        assert int(m["counts"].sum()) == oracle.kept_count(type_, band, anchor, F, S)
        # a tile holding a position without a token is never full
        perm = oracle.permutation_padded(order, F, S, Sp)
        nq, nk = m["n_q"], m["n_k"]
        for i in range(nq):
            for j in range(nk):
                qt = perm[i * tq: (i + 1) * tq]
                kt = perm[j * tk: (j + 1) * tk]
                holes = len(qt) < tq or len(kt) < tk or (qt < 0).any() or (kt < 0).any()
                if holes:
                    assert m["cls"][i, j] != 1


@pytest.mark.parametrize("F,S,T,band,anchor", [(5, 7, 4, 1, 1), (4, 10, 4, 0, 0),
                                               (6, 12, 8, 2, 1), (3, 20, 8, 1, 0)])
def test_frames_never_cut_a_tile(F, S, T, band, anchor):
    """Sp a multiple of both tiles: every tile of a frame-major spatial head keeps all of
    its token pairs or none (no tile is a boundary tile because of a frame edge)."""
    Sp = -(-S // T) * T
    perm = oracle.permutation_padded(FM, F, S, Sp)
    m = oracle.tile_map_padded(SP, band, anchor, FM, F, S, Sp, T, T)
    for i in range(m["n_q"]):
        nq_tok = int((perm[i * T: (i + 1) * T] >= 0).sum())
        for j in range(m["n_k"]):
            nk_tok = int((perm[j * T: (j + 1) * T] >= 0).sum())
            c = int(m["counts"][i, j])
            assert c in (0, nq_tok * nk_tok), (i, j, c, nq_tok, nk_tok)
    # whereas the unpadded layout cuts tiles at frame edges when S is not a multiple of T
    if S % T:
        u = oracle.tile_map(SP, band, anchor, FM, F, S, T, T)
        assert (u["cls"] == 2).any()


def test_class_matrix_by_hand():
    """F = 3, S = 5, Sp = 8, 4 x 4 tiles, spatial band 0 with the anchor.  Each frame
    fills positions f*8 .. f*8+4: its first tile holds 4 tokens, its second 1 token and
    3 empty positions.  A query of frame f keeps the keys of frames f and 0.  So tile
    (i, j) (frames i // 2 and j // 2) is kept iff j // 2 in {i // 2, 0}, and full iff
    kept and both tiles are the token-only first tiles (i, j even)."""
    want = np.array([[1, 2, 0, 0, 0, 0],
                     [2, 2, 0, 0, 0, 0],
                     [1, 2, 1, 2, 0, 0],
                     [2, 2, 2, 2, 0, 0],
                     [1, 2, 0, 0, 1, 2],
                     [2, 2, 0, 0, 2, 2]], np.uint8)
    m = oracle.tile_map_padded(SP, 0, 1, FM, 3, 5, 8, 4, 4)
    np.testing.assert_array_equal(m["cls"], want)


def test_stride_equal_to_frame_is_the_plain_layout():
    for order in (FM, AF, ST):
        np.testing.assert_array_equal(oracle.permutation_padded(order, 4, 6, 6),
                                      oracle.permutation(order, 4, 6))
        a = oracle.tile_map_padded(TP, 2, 1, order, 4, 6, 6, 4, 8)
        b = oracle.tile_map(TP, 2, 1, order, 4, 6, 4, 8)
        np.testing.assert_array_equal(a["counts"], b["counts"])


def test_frame_stride():
    assert oracle.frame_stride(3600, 0) == 3600
    assert oracle.frame_stride(3600, 128) == 3712
    assert oracle.frame_stride(14400, 128) == 14464
    assert oracle.frame_stride(256, 128) == 256
