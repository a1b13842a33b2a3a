"""Randomised pins of the oracle's mask, kept count, tile counts, tile classes and CSR
lists (CPU only).  For small random problems (frames, grid, head type, band, anchor, token
order, tile sizes with ragged tails), everything on the reference side is recomputed here
by brute force: the mask from its definition with numpy broadcasting, the token orders
from their position formulas, tile counts by summing the reordered, zero-padded mask,
classes and lists from the counts.  The reference side calls nothing in the oracle."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle


def tokens_of_positions(order, F, S):
    """Frame-major token at each position of `order`, from the orders' definitions:
    frame-major t = f*S + s; strict temporal-major position s*F + f; anchor-first:
    frame 0 at positions 0..S-1, then frame f >= 1 at S + s*(F-1) + (f-1)."""
    tok = np.empty(F * S, np.int64)
    for f in range(F):
        for s in range(S):
            if order == oracle.FRAME_MAJOR:
                p = f * S + s
            elif order == oracle.TEMPORAL_STRICT:
                p = s * F + f
            else:
                p = s if f == 0 else S + s * (F - 1) + (f - 1)
            tok[p] = f * S + s
    return tok


def brute_mask(type_, band, anchor, F, S):
    t = np.arange(F * S)
    f, s = t // S, t % S
    if type_ == oracle.SPATIAL:
        near = np.abs(f[:, None] - f[None, :]) <= band
    else:
        near = np.abs(s[:, None] - s[None, :]) <= band
    return near | (bool(anchor) & (f[None, :] == 0))


@settings(max_examples=150, deadline=None)
@given(F=st.integers(1, 6), gh=st.integers(1, 6), gw=st.integers(1, 8),
       type_=st.sampled_from([oracle.SPATIAL, oracle.TEMPORAL]), band=st.integers(0, 9),
       anchor=st.integers(0, 1),
       order=st.sampled_from([oracle.FRAME_MAJOR, oracle.TEMPORAL_ANCHOR_FIRST,
                              oracle.TEMPORAL_STRICT]),
       tq=st.sampled_from([8, 16, 24, 32, 48, 64]), tk=st.sampled_from([8, 16, 20, 32, 64]))
def test_oracle_tiles_match_brute_force(F, gh, gw, type_, band, anchor, order, tq, tk):
    S = gh * gw
    N = F * S
    m = brute_mask(type_, band, anchor, F, S)
    assert oracle.kept_count(type_, band, anchor, F, S) == int(m.sum())
    np.testing.assert_array_equal(oracle.mask(type_, band, anchor, F, S), m.astype(np.uint8))

    tok = tokens_of_positions(order, F, S)
    mp = m[np.ix_(tok, tok)]                       # the mask in position order
    nq, nk = -(-N // tq), -(-N // tk)
    pad = np.zeros((nq * tq, nk * tk), np.int64)
    pad[:N, :N] = mp
    counts = pad.reshape(nq, tq, nk, tk).sum(axis=(1, 3))
    cls = np.where(counts == 0, 0, np.where(counts == tq * tk, 1, 2)).astype(np.uint8)

    got = oracle.tile_map(type_, band, anchor, order, F, S, tq, tk)
    np.testing.assert_array_equal(got["counts"], counts)
    np.testing.assert_array_equal(got["cls"], cls)
    for c, ptr, idx in ((1, "full_ptr", "full_idx"), (2, "bnd_ptr", "bnd_idx")):
        rows = [np.nonzero(cls[i] == c)[0] for i in range(nq)]
        np.testing.assert_array_equal(got[ptr], np.cumsum([0] + [len(r) for r in rows]))
        np.testing.assert_array_equal(got[idx], np.concatenate(rows).astype(np.int32)
                                      if rows else np.zeros(0, np.int32))


@settings(max_examples=60, deadline=None)
@given(F=st.integers(1, 5), gh=st.integers(1, 5), gw=st.integers(1, 6),
       d=st.sampled_from([4, 8, 16]),
       type_=st.sampled_from([oracle.SPATIAL, oracle.TEMPORAL]), band=st.integers(0, 6),
       anchor=st.integers(0, 1), seed=st.integers(0, 2 ** 16),
       scale=st.floats(0.05, 2.0))
def test_oracle_attention_matches_library_sdpa(F, gh, gw, d, type_, band, anchor, seed,
                                               scale):
    """O against torch's fp64 scaled_dot_product_attention under the brute-force mask, LSE
    against torch.logsumexp; rows with no kept key (possible without the anchor only if
    the band excludes the query itself, which it never does) are not produced here."""
    import torch
    S = gh * gw
    N = F * S
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(N, d, generator=g, dtype=torch.float64).float() for _ in range(3))
    m = torch.from_numpy(brute_mask(type_, band, anchor, F, S))
    rows = np.arange(N, dtype=np.int32)
    o, lse = oracle.attention_rows(q.numpy(), k.numpy(), v.numpy(), F, S, scale, type_, band,
                                   anchor, rows)
    qd, kd, vd = q.double(), k.double(), v.double()
    ref = torch.nn.functional.scaled_dot_product_attention(
        qd[None], kd[None], vd[None], attn_mask=m[None], scale=scale)[0]
    logits = (qd @ kd.T) * scale
    ref_lse = torch.logsumexp(logits.masked_fill(~m, float("-inf")), dim=1)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


@settings(max_examples=60, deadline=None)
@given(F=st.integers(1, 5), gh=st.integers(1, 5), gw=st.integers(1, 6),
       type_=st.sampled_from([oracle.SPATIAL, oracle.TEMPORAL]), band=st.integers(0, 6),
       anchor=st.integers(0, 1),
       order=st.sampled_from([oracle.FRAME_MAJOR, oracle.TEMPORAL_ANCHOR_FIRST,
                              oracle.TEMPORAL_STRICT]),
       tq=st.sampled_from([4, 8, 12, 16]), tk=st.sampled_from([4, 8, 10, 16]),
       seed=st.integers(0, 2 ** 16))
def test_oracle_tile_aligned_matches_library_sdpa(F, gh, gw, type_, band, anchor, order, tq,
                                                  tk, seed):
    """The tile-aligned traversal keeps every key of each (q-tile, k-tile) of the head's
    token order that holds an exactly kept pair.  That snapped mask is built here from
    brute-force tile counts and mapped back to frame-major tokens; the oracle gets the
    same counts and must match torch's fp64 SDPA under it."""
    import torch
    S = gh * gw
    N = F * S
    d, scale = 8, 0.3
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(N, d, generator=g, dtype=torch.float64).float() for _ in range(3))
    tok = tokens_of_positions(order, F, S)
    mp = brute_mask(type_, band, anchor, F, S)[np.ix_(tok, tok)]
    nq, nk = -(-N // tq), -(-N // tk)
    pad = np.zeros((nq * tq, nk * tk), np.int64)
    pad[:N, :N] = mp
    counts = pad.reshape(nq, tq, nk, tk).sum(axis=(1, 3))
    snapped_pos = (counts[np.arange(N)[:, None] // tq, np.arange(N)[None, :] // tk] > 0)
    snapped = np.zeros((N, N), bool)
    snapped[np.ix_(tok, tok)] = snapped_pos          # back to frame-major tokens
    rows = np.arange(N, dtype=np.int32)
    o, lse = oracle.attention_rows_tile_aligned(q.numpy(), k.numpy(), v.numpy(), F, S, scale,
                                                order, tq, tk, counts, 0, rows)
    m = torch.from_numpy(snapped)
    qd, kd, vd = q.double(), k.double(), v.double()
    ref = torch.nn.functional.scaled_dot_product_attention(
        qd[None], kd[None], vd[None], attn_mask=m[None], scale=scale)[0]
    ref_lse = torch.logsumexp(((qd @ kd.T) * scale).masked_fill(~m, float("-inf")), dim=1)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


@settings(max_examples=40, deadline=None)
@given(F=st.integers(2, 5), gh=st.integers(1, 5), gw=st.integers(2, 6),
       w_s=st.integers(0, 3), w_t=st.integers(0, 8), anchor=st.integers(0, 1),
       n_rows=st.integers(1, 12), seed=st.integers(0, 2 ** 16))
def test_oracle_classifier_matches_library_sdpa(F, gh, gw, w_s, w_t, anchor, n_rows, seed):
    """Deviations of the spatial and temporal outputs from the dense one (mean square over
    the sampled rows x d) and the choice (the smaller, a tie to spatial), with the three
    outputs from torch's fp64 SDPA under the brute-force masks."""
    import torch
    S = gh * gw
    N = F * S
    d, scale = 8, 0.4
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(N, d, generator=g, dtype=torch.float64).float() for _ in range(3))
    rows = np.sort(np.random.default_rng(seed).choice(N, size=min(n_rows, N),
                                                      replace=False)).astype(np.int32)
    qd, kd, vd = q.double(), k.double(), v.double()

    def sdpa(mask):
        m = torch.from_numpy(mask)
        return torch.nn.functional.scaled_dot_product_attention(
            qd[None], kd[None], vd[None], attn_mask=m[None], scale=scale)[0].numpy()[rows]

    od = sdpa(np.ones((N, N), bool))
    ms = float(np.mean((sdpa(brute_mask(oracle.SPATIAL, w_s, anchor, F, S)) - od) ** 2))
    mt = float(np.mean((sdpa(brute_mask(oracle.TEMPORAL, w_t, anchor, F, S)) - od) ** 2))
    t, ms_o, mt_o = oracle.classify(q.numpy(), k.numpy(), v.numpy(), F, S, scale, w_s, w_t,
                                    anchor, rows)
    assert abs(ms_o - ms) <= 1e-12 and abs(mt_o - mt) <= 1e-12
    if abs(ms - mt) > 1e-12:
        assert t == (oracle.SPATIAL if ms < mt else oracle.TEMPORAL)


@settings(max_examples=80, deadline=None)
@given(F=st.integers(1, 9), S=st.integers(1, 40),
       order=st.sampled_from([oracle.FRAME_MAJOR, oracle.TEMPORAL_ANCHOR_FIRST,
                              oracle.TEMPORAL_STRICT]))
def test_oracle_permutation_matches_the_order_formulas(F, S, order):
    """oracle.permutation (position -> frame-major token) equals the order written out
    from its position formula, and is a permutation of 0..N-1."""
    perm = oracle.permutation(order, F, S)
    np.testing.assert_array_equal(perm, tokens_of_positions(order, F, S))
    np.testing.assert_array_equal(np.sort(perm), np.arange(F * S))
