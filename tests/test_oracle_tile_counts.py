"""Pins of the oracle's tile classification at realistic sizes (CPU only).

The pages build their kernel on a per-tile classification: tiles with no kept pair are
skipped, fully kept tiles take the unmasked fast path, the rest are masked ("Accelerating
Spatio-Temporal Attention for Video Diffusion on TPUs", aihirek.info, section "A
TPU-kernel kialakitasa dontonek bizonyult"; ainews.tenesys.com, "Co sie zmienilo?"
items 1-2).  The oracle classifies a tile by counting its kept elements on the grid
padded to whole tiles, where padded pairs count as not kept.

The integers below were counted independently of this oracle, by a separate numpy script
that materialised the element mask per q-tile when the method was first studied; they
are literals here, not outputs of the oracle.  A wrong padding rule, an off-by-one in a
band edge, a mistake in the anchor-first temporal-major order or a swapped query/key
side changes at least one of them.  Each row: (full, boundary, empty) tiles of one head.

A second group checks the row sampler of the GPU parity tests: the rows it returns cover
every row of the chosen 128-row query blocks in each head's token order.
"""
import numpy as np
import pytest

import oracle
from block_sparse_spatio_attn_b200 import configs as C

SP, TP = oracle.SPATIAL, oracle.TEMPORAL
FM, AF, ST = oracle.FRAME_MAJOR, oracle.TEMPORAL_ANCHOR_FIRST, oracle.TEMPORAL_STRICT

# (name, type, band, order, frames, tokens per frame, tile, full, boundary, empty)
SMALL = [
    ("tiny spatial FM", SP, 1, FM, 3, 64, 64, 8, 0, 1),
    ("tiny temporal FM", TP, 8, FM, 3, 64, 64, 3, 6, 0),
    ("tiny temporal strict", TP, 8, ST, 3, 64, 64, 0, 9, 0),
    ("tiny temporal anchor-first", TP, 8, AF, 3, 64, 64, 3, 6, 0),
    ("mid spatial FM 64", SP, 2, FM, 13, 960, 64, 15525, 0, 22500),
    ("mid spatial FM 128", SP, 2, FM, 13, 960, 128, 3752, 255, 5597),
    ("mid temporal FM 128", TP, 160, FM, 13, 960, 128, 1232, 4326, 4046),
    ("mid temporal strict 128", TP, 160, ST, 13, 960, 128, 2767, 6837, 0),
    ("mid temporal anchor-first 128", TP, 160, AF, 13, 960, 128, 3181, 561, 5862),
    ("mid temporal anchor-first 64", TP, 160, AF, 13, 960, 64, 13347, 800, 23878),
]

HEADLINE = [
    ("headline spatial FM 64", SP, 3, FM, 21, 3600, 64, 479197, 4159, 913768),
    ("headline spatial FM 128", SP, 3, FM, 21, 3600, 128, 119194, 2335, 227752),
    ("headline spatial FM 256", SP, 3, FM, 21, 3600, 256, 29567, 1224, 56825),
    ("headline temporal FM 64", TP, 600, FM, 21, 3600, 64, 427390, 91093, 878641),
    ("headline temporal FM 128", TP, 600, FM, 21, 3600, 128, 95128, 46460, 207693),
    ("headline temporal FM 256", TP, 600, FM, 21, 3600, 256, 18282, 23233, 46101),
    ("headline temporal strict 64", TP, 600, ST, 21, 3600, 64, 424914, 971226, 984),
    ("headline temporal strict 128", TP, 600, ST, 21, 3600, 128, 105544, 243737, 0),
    ("headline temporal strict 256", TP, 600, ST, 21, 3600, 256, 26263, 61353, 0),
    ("headline temporal anchor-first 64", TP, 600, AF, 21, 3600, 64, 469143, 7472, 920509),
    ("headline temporal anchor-first 128", TP, 600, AF, 21, 3600, 128, 116178, 3734, 229369),
    ("headline temporal anchor-first 256", TP, 600, AF, 21, 3600, 256, 28544, 1868, 57204),
]

TWOK = [
    ("2k spatial FM 128", SP, 3, FM, 21, 14400, 128, 1920492, 6525, 3656752),
    ("2k temporal anchor-first 128", TP, 2400, AF, 21, 14400, 128, 1884355, 14287, 3685127),
]


def _check(case):
    name, t, w, order, F, S, T, nf, nb, ne = case
    m = oracle.tile_map(t, w, 1, order, F, S, T, T)
    cls = m["cls"]
    got = (int((cls == 1).sum()), int((cls == 2).sum()), int((cls == 0).sum()))
    assert got == (nf, nb, ne), f"{name}: oracle {got}, independent count {(nf, nb, ne)}"
    # the CSR lists hold exactly the full and boundary tiles
    assert int(m["full_ptr"][-1]) == nf and int(m["bnd_ptr"][-1]) == nb


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c[0])
def test_tile_counts_small(case):
    _check(case)


@pytest.mark.slow
@pytest.mark.parametrize("case", HEADLINE, ids=lambda c: c[0])
def test_tile_counts_headline(case):
    _check(case)


@pytest.mark.slow
@pytest.mark.parametrize("case", TWOK, ids=lambda c: c[0])
def test_tile_counts_2k(case):
    _check(case)


# ------------------------------------------------------------- the GPU tests' row sample
@pytest.mark.parametrize("wl", [C.tiny(), C.mid(), C.headline(), C.twok(),
                                C.permutation_study(C.ORDER_TEMPORAL_MAJOR_STRICT)],
                         ids=lambda w: w.name)
def test_sample_rows_cover_whole_kernel_blocks(wl):
    from tests.helpers import kernel_blocks, sample_rows
    N, F, S = wl.tokens, wl.frames, wl.tokens_per_frame
    rows = set(sample_rows(wl, 64).tolist())
    blocks = kernel_blocks(N)
    nb = -(-N // 128)
    # the first work item, an odd block (the second warpgroup's) and the ragged last block
    assert 0 in blocks and 1 in blocks and (nb - 1) in blocks
    if nb >= 6:
        assert any(b % 2 == 1 and 1 < b < nb - 2 for b in blocks)
    for od in set(wl.order):
        perm = oracle.permutation(od, F, S)
        for b in blocks:
            want = perm[b * 128: min(N, b * 128 + 128)]
            assert len(want) == min(128, N - b * 128)
            missing = [int(t) for t in want if int(t) not in rows]
            assert not missing, f"order {od} block {b}: rows {missing[:4]} not sampled"
    assert all(0 <= r < N for r in rows)
    assert len(rows) == len(np.unique(sample_rows(wl, 64)))
