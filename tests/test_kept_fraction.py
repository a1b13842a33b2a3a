"""The library's closed-form kept fraction (svga_kept_fraction, the eligibility test of
the band selection) against the oracle's pair-by-pair count, and the oracle's band
selection on a constructed case (CPU only)."""
import numpy as np
import pytest

import oracle
from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200 import svga

SHAPES = [(1, 1, 5), (3, 2, 4), (5, 3, 3), (7, 4, 5), (4, 1, 17)]


@pytest.mark.parametrize("F,gh,gw", SHAPES)
@pytest.mark.parametrize("anchor", [0, 1])
def test_kept_fraction_matches_pair_count(F, gh, gw, anchor):
    S = gh * gw
    prob = svga.ProblemSpec(1, F, gh, gw, 64, [0], [0], [0], anchor, 64, 64)
    for t in (oracle.SPATIAL, oracle.TEMPORAL):
        for w in (0, 1, 2, 5, 40, 65535):
            want = oracle.kept_count(t, w, anchor, F, S) / float((F * S) ** 2)
            got = svga.svga_kept_fraction(prob, t, w)
            assert got == pytest.approx(want, rel=0, abs=1e-15), (t, w)


def test_headline_kept_fractions():
    """The headline heads keep 34.47 % (spatial, |df| <= 3) and 33.88 % (temporal,
    |ds| <= 600) of the pairs; together 34.18 %, the bench's kept fraction."""
    prob = svga.ProblemSpec.from_workload(C.headline())
    fs = svga.svga_kept_fraction(prob, 0, 3)
    ft = svga.svga_kept_fraction(prob, 1, 600)
    # spatial: S^2 x (kept frame pairs 152 + anchored frames) / N^2, by hand: frames
    # 0..20, |df| <= 3, frame 0 added where it is outside the band
    frames = sum(min(20, f + 3) - max(0, f - 3) + 1 + (1 if f - 3 > 0 else 0) for f in range(21))
    assert fs == pytest.approx(frames / 21 ** 2, abs=1e-15)
    assert round(fs, 5) == 0.34467 and round(ft, 5) == 0.33884
    assert round((fs + ft) / 2, 6) == 0.341758


def test_select_band_oracle_on_a_constructed_case():
    """Q and K equal and constant within a frame, different across frames: a query's
    scores peak on its own frame, so the narrowest spatial band that keeps the own frame
    (band 0) already matches dense up to the other frames' weight; a temporal band keeps
    other frames' keys too.  With a budget that admits the temporal band and spatial
    bands 0 and 1, the least deviation is spatial; a budget below every candidate's
    fraction leaves nothing eligible."""
    F, S, d = 4, 6, 8
    rng = np.random.default_rng(0)
    basis = rng.standard_normal((F, d)) * 3.0
    q = np.repeat(basis, S, axis=0).astype(np.float32)
    k = q.copy()
    v = rng.standard_normal((F * S, d)).astype(np.float32)
    rows = np.arange(F * S, dtype=np.int32)
    cands = [(oracle.TEMPORAL, 1), (oracle.SPATIAL, 0), (oracle.SPATIAL, 1),
             (oracle.SPATIAL, 3)]
    best, mses, fracs = oracle.select_band(q, k, v, F, S, 1.0, cands, 0, rows, 0.6)
    assert fracs[3] == 1.0 and fracs[3] > 0.6              # every pair: not eligible
    assert fracs[1] == pytest.approx(0.25)                  # own frame of 4
    assert cands[best][0] == oracle.SPATIAL
    assert mses[best] == min(m for m, f in zip(mses, fracs) if f <= 0.6)
    best, _, _ = oracle.select_band(q, k, v, F, S, 1.0, cands, 0, rows, 0.01)
    assert best == -1
