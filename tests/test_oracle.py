"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test names what it pins and where the fact comes from: a closed form, a library
routine, a hand-derived value or a brute force written here from the definition.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200.inputs import make_qkv


# ----------------------------------------------------------------------------- masks
def closed_form_kept(type_, band, anchor, F, S):
    """Kept pairs of one head in closed form.
    spatial : S^2 * sum_fq |{fk : |fq-fk| <= w} U {0}|
    temporal: every query keeps all S frame-0 keys (F*S*S pairs); the other F-1 key
              frames keep, for each query frame, c = sum_sq |[sq-w, sq+w] n [0, S-1]|
              pairs; total F*S^2 + F*(F-1)*c."""
    if type_ == oracle.SPATIAL:
        tot = 0
        for fq in range(F):
            ks = {fk for fk in range(F) if abs(fq - fk) <= band}
            if anchor:
                ks.add(0)
            tot += len(ks)
        return S * S * tot
    c = sum(min(S - 1, sq + band) - max(0, sq - band) + 1 for sq in range(S))
    if anchor:
        return F * S * S + F * (F - 1) * c
    return F * F * c


@pytest.mark.parametrize("wl", [C.tiny(), C.mid()], ids=lambda w: w.name)
def test_kept_count_closed_form(wl):
    F, S = wl.frames, wl.tokens_per_frame
    for t, w in sorted(set(zip(wl.head_type, wl.band))):
        assert oracle.kept_count(t, w, 1, F, S) == closed_form_kept(t, w, 1, F, S)


@pytest.mark.slow
def test_kept_count_closed_form_headline():
    wl = C.headline()
    F, S = wl.frames, wl.tokens_per_frame
    for t, w in [(oracle.SPATIAL, 3), (oracle.TEMPORAL, 600)]:
        assert oracle.kept_count(t, w, 1, F, S) == closed_form_kept(t, w, 1, F, S)


def test_kept_count_without_anchor_and_edges():
    # no anchor: spatial band 0 keeps exactly the query's own frame: F * S^2 pairs
    assert oracle.kept_count(oracle.SPATIAL, 0, 0, 4, 6) == 4 * 36
    # band >= F-1 keeps everything
    assert oracle.kept_count(oracle.SPATIAL, 3, 1, 4, 6) == (24 * 24)
    # temporal band 0 without anchor: same in-frame index only: S * F^2 pairs
    assert oracle.kept_count(oracle.TEMPORAL, 0, 0, 4, 6) == 6 * 16
    for t in (oracle.SPATIAL, oracle.TEMPORAL):
        for w in (0, 1, 2, 5):
            for a in (0, 1):
                assert oracle.kept_count(t, w, a, 5, 7) == closed_form_kept(t, w, a, 5, 7)


def test_tiny_spatial_fraction_is_eight_ninths():
    # 3 frames, |df| <= 1 plus the frame-0 anchor: frame pairs kept are
    # (0,0) (0,1) | (1,0) (1,1) (1,2) | (2,0) (2,1) (2,2) -> 8 of 9
    wl = C.tiny()
    F, S = wl.frames, wl.tokens_per_frame
    assert oracle.kept_count(oracle.SPATIAL, 1, 1, F, S) * 9 == 8 * (F * S) ** 2


def test_mask_matches_python_predicate_tiny():
    """The element mask against a predicate written here from the definitions."""
    F, S = 3, 64
    for t, w in [(oracle.SPATIAL, 1), (oracle.TEMPORAL, 8)]:
        m = oracle.mask(t, w, 1, F, S)
        N = F * S
        ref = np.zeros((N, N), np.uint8)
        for qi in range(N):
            fq, sq = divmod(qi, S)
            for ki in range(N):
                fk, sk = divmod(ki, S)
                near = abs(fq - fk) <= w if t == oracle.SPATIAL else abs(sq - sk) <= w
                ref[qi, ki] = 1 if (near or fk == 0) else 0
        np.testing.assert_array_equal(m, ref)


# ---------------------------------------------------------------------- permutation
def test_orders_against_numpy_transpose():
    """Strict temporal-major is the transpose of the [F, S] grid; anchor-first keeps
    frame 0 in front and transposes frames 1..F-1."""
    for F, S in [(3, 64), (13, 960), (21, 12), (1, 5), (2, 3)]:
        fm = np.arange(F * S).reshape(F, S)
        strict = fm.T.reshape(-1)
        np.testing.assert_array_equal(oracle.permutation(oracle.TEMPORAL_STRICT, F, S), strict)
        af = np.concatenate([fm[0], fm[1:].T.reshape(-1)])
        np.testing.assert_array_equal(oracle.permutation(oracle.TEMPORAL_ANCHOR_FIRST, F, S), af)
        np.testing.assert_array_equal(oracle.permutation(oracle.FRAME_MAJOR, F, S),
                                      np.arange(F * S))


# -------------------------------------------------------------------- tile classes
def brute_tile_counts(t, w, anchor, perm, F, S, tq, tk):
    N = F * S
    nq, nk = -(-N // tq), -(-N // tk)
    cnt = np.zeros((nq, nk), np.int64)
    for p in range(N):
        fq, sq = divmod(int(perm[p]), S)
        for r in range(N):
            fk, sk = divmod(int(perm[r]), S)
            near = abs(fq - fk) <= w if t == oracle.SPATIAL else abs(sq - sk) <= w
            if near or (anchor and fk == 0):
                cnt[p // tq, r // tk] += 1
    return cnt


@pytest.mark.parametrize("order", [oracle.FRAME_MAJOR, oracle.TEMPORAL_ANCHOR_FIRST,
                                   oracle.TEMPORAL_STRICT])
@pytest.mark.parametrize("tq,tk", [(64, 64), (64, 32), (48, 80)])
def test_tile_counts_brute_force(order, tq, tk):
    F, S = 3, 40   # 120 tokens: ragged tails for every tile size here
    perm = oracle.permutation(order, F, S)
    for t, w in [(oracle.SPATIAL, 1), (oracle.TEMPORAL, 5)]:
        got = oracle.tile_map(t, w, 1, order, F, S, tq, tk)
        ref = brute_tile_counts(t, w, 1, perm, F, S, tq, tk)
        np.testing.assert_array_equal(got["counts"], ref)


def test_tiny_spatial_tile_classes_by_hand():
    # tiny, tile 64 = one frame: row f_q=0 keeps frames {0,1}, f_q=1 keeps all,
    # f_q=2 keeps {0,1,2}: 8 full tiles, tile (0, 2) empty
    m = oracle.tile_map(oracle.SPATIAL, 1, 1, oracle.FRAME_MAJOR, 3, 64, 64, 64)
    expect = np.array([[1, 1, 0], [1, 1, 1], [1, 1, 1]], np.uint8)
    np.testing.assert_array_equal(m["cls"], expect)
    assert m["full_idx"].tolist() == [0, 1, 0, 1, 2, 0, 1, 2]
    assert m["bnd_idx"].size == 0


@pytest.mark.parametrize("wl", [C.mid()], ids=lambda w: w.name)
def test_tile_map_invariants(wl):
    F, S = wl.frames, wl.tokens_per_frame
    N = F * S
    for t, w, o in set(zip(wl.head_type, wl.band, wl.order)):
        for tq, tk in [(128, 128), (64, 128), (256, 64)]:
            m = oracle.tile_map(t, w, 1, o, F, S, tq, tk)
            cnt, cls = m["counts"], m["cls"]
            # counts sum to the kept count of the head (order does not change it)
            assert cnt.sum() == closed_form_kept(t, w, 1, F, S)
            assert ((cls == 1) == (cnt == tq * tk)).all()
            assert ((cls == 0) == (cnt == 0)).all()
            # padded tiles are never full
            if N % tk:
                assert (cls[:, -1] != 1).all()
            if N % tq:
                assert (cls[-1, :] != 1).all()
            # lists: ascending per q-tile and equal to the classes
            for i in range(m["n_q"]):
                fl = m["full_idx"][m["full_ptr"][i]:m["full_ptr"][i + 1]]
                bl = m["bnd_idx"][m["bnd_ptr"][i]:m["bnd_ptr"][i + 1]]
                assert (np.diff(fl) > 0).all() and (np.diff(bl) > 0).all()
                np.testing.assert_array_equal(fl, np.nonzero(cls[i] == 1)[0])
                np.testing.assert_array_equal(bl, np.nonzero(cls[i] == 2)[0])


# ----------------------------------------------------------------------- attention
def brute_attention_row(q, k, v, qi, S, scale, keep):
    """Direct double loops with math.exp for one query row."""
    N, d = k.shape
    xs = []
    for j in range(N):
        if keep(qi, j):
            xs.append((j, scale * sum(float(q[qi, c]) * float(k[j, c]) for c in range(d))))
    m = max(x for _, x in xs)
    den = sum(math.exp(x - m) for _, x in xs)
    out = [sum(math.exp(x - m) * float(v[j, c]) for j, x in xs) / den for c in range(d)]
    return out, m + math.log(den)


def test_tiny_brute_force():
    wl = C.tiny()
    q, k, v = make_qkv(wl)
    F, S, d = wl.frames, wl.tokens_per_frame, wl.head_dim
    scale = 1.0 / math.sqrt(d)
    rows = np.array([0, 5, 63, 64, 100, 130, 191], np.int32)
    for h, (t, w) in enumerate(zip(wl.head_type, wl.band)):
        qh, kh, vh = (x[h].float().numpy() for x in (q, k, v))

        def keep(qi, kj):
            fq, sq = divmod(qi, S)
            fk, sk = divmod(kj, S)
            near = abs(fq - fk) <= w if t == C.SPATIAL else abs(sq - sk) <= w
            return near or fk == 0

        o, lse = oracle.attention_rows(qh, kh, vh, F, S, scale, t, w, 1, rows)
        for r, qi in enumerate(rows):
            ob, lb = brute_attention_row(qh, kh, vh, int(qi), S, scale, keep)
            np.testing.assert_allclose(o[r], ob, rtol=0, atol=1e-12)
            assert abs(lse[r] - lb) <= 1e-12


def _sdpa64(q, k, v, scale, mask=None):
    qt, kt, vt = (torch.from_numpy(np.asarray(x, np.float64))[None] for x in (q, k, v))
    am = None if mask is None else torch.from_numpy(mask.astype(bool))[None]
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=am, scale=scale)[0].numpy()


def test_dense_equals_library_sdpa():
    """All-ones mask: the oracle equals torch's fp64 scaled-dot-product attention."""
    wl = C.tiny()
    q, k, v = make_qkv(wl)
    F, S, d = wl.frames, wl.tokens_per_frame, wl.head_dim
    scale = 1.0 / math.sqrt(d)
    rows = np.arange(F * S, dtype=np.int32)
    qh, kh, vh = (x[0].float().numpy() for x in (q, k, v))
    o, lse = oracle.attention_rows(qh, kh, vh, F, S, scale, oracle.DENSE, 0, 1, rows)
    np.testing.assert_allclose(o, _sdpa64(qh, kh, vh, scale), rtol=0, atol=1e-12)
    x = scale * qh.astype(np.float64) @ kh.astype(np.float64).T
    mx = x.max(1)
    np.testing.assert_allclose(lse, mx + np.log(np.exp(x - mx[:, None]).sum(1)), atol=1e-12)


def test_masked_equals_library_sdpa():
    """Masked softmax arithmetic pinned by torch's fp64 SDPA with a boolean mask."""
    F, S, d = 4, 30, 32
    N = F * S
    g = torch.Generator().manual_seed(11)
    q, k, v = (torch.randn(N, d, generator=g).to(torch.bfloat16).float().numpy()
               for _ in range(3))
    scale = 0.3
    rows = np.arange(N, dtype=np.int32)
    for t, w in [(oracle.SPATIAL, 1), (oracle.TEMPORAL, 4), (oracle.TEMPORAL, 0)]:
        m = oracle.mask(t, w, 1, F, S)
        o, _ = oracle.attention_rows(q, k, v, F, S, scale, t, w, 1, rows)
        np.testing.assert_allclose(o, _sdpa64(q, k, v, scale, m), rtol=0, atol=1e-12)


# ---------------------------------------------------- tile-aligned traversal (B3)
def brute_snapped_mask(t, w, anchor, order, F, S, tq, tk):
    """Frame-major [N, N] mask of the tile-aligned traversal, built here with numpy: the
    exact predicate on the coordinates of each position of `order` (the order written
    as a grid transpose), any-kept per (q-tile, k-tile) through a padded reshape, then
    every pair of a visited tile kept, mapped back to frame-major tokens."""
    N = F * S
    fm = np.arange(N).reshape(F, S)
    if order == oracle.FRAME_MAJOR:
        perm = fm.reshape(-1)
    elif order == oracle.TEMPORAL_ANCHOR_FIRST:
        perm = np.concatenate([fm[0], fm[1:].T.reshape(-1)])
    else:
        perm = fm.T.reshape(-1)
    f, s = np.divmod(perm, S)
    c = f if t == oracle.SPATIAL else s
    keep = np.abs(c[:, None] - c[None, :]) <= w
    if anchor:
        keep |= (f == 0)[None, :]
    nq, nk = -(-N // tq), -(-N // tk)
    pad = np.zeros((nq * tq, nk * tk), bool)
    pad[:N, :N] = keep
    visited = pad.reshape(nq, tq, nk, tk).any(axis=(1, 3))
    snapped = visited[np.arange(N) // tq][:, np.arange(N) // tk]
    assert (snapped >= keep).all()      # a superset of the exact kept set
    out = np.zeros((N, N), bool)
    out[np.ix_(perm, perm)] = snapped
    return out


@pytest.mark.parametrize("order", [oracle.FRAME_MAJOR, oracle.TEMPORAL_ANCHOR_FIRST,
                                   oracle.TEMPORAL_STRICT])
@pytest.mark.parametrize("tq,tk", [(32, 32), (32, 16), (36, 52)])
def test_tile_aligned_equals_library_sdpa_on_snapped_mask(order, tq, tk):
    """The tile-aligned oracle equals torch's fp64 SDPA under the snapped mask built
    independently above (6 frames x 40 tokens; ragged tiles at 32 and 36 x 52).  The
    snapped mask must differ from both the exact and the all-ones mask here, so that
    the tile indexing is really exercised."""
    F, S, d = 6, 40, 16
    N = F * S
    g = torch.Generator().manual_seed(21)
    q, k, v = (torch.randn(N, d, generator=g).to(torch.bfloat16).float().numpy()
               for _ in range(3))
    scale = 0.35
    rows = np.arange(N, dtype=np.int32)
    nontrivial = 0
    # without the anchor too: under the strict order every key tile holds frame-0 keys
    for t, w, a in [(oracle.SPATIAL, 1, 1), (oracle.TEMPORAL, 3, 1), (oracle.TEMPORAL, 3, 0)]:
        counts = oracle.tile_map(t, w, a, order, F, S, tq, tk)["counts"]
        o, lse = oracle.attention_rows_tile_aligned(q, k, v, F, S, scale, order, tq, tk,
                                                    counts, 0, rows)
        m = brute_snapped_mask(t, w, a, order, F, S, tq, tk)
        nontrivial += (not m.all()) and (m != oracle.mask(t, w, a, F, S).astype(bool)).any()
        np.testing.assert_allclose(o, _sdpa64(q, k, v, scale, m), rtol=0, atol=1e-12)
        x = scale * q.astype(np.float64) @ k.astype(np.float64).T
        x = np.where(m, x, -np.inf)
        mx = x.max(1)
        np.testing.assert_allclose(lse, mx + np.log(np.exp(x - mx[:, None]).sum(1)),
                                   atol=1e-12)
    assert nontrivial >= 1


def test_tile_aligned_reduces_to_exact_when_frames_fill_tiles():
    """Frame-major spatial heads whose frames are whole tiles have no boundary tile, so
    snapping changes nothing: the tile-aligned result is the exact one."""
    wl = C.tiny()                        # 3 frames of 64 tokens
    q, k, v = make_qkv(wl)
    F, S = wl.frames, wl.tokens_per_frame
    rows = np.arange(F * S, dtype=np.int32)
    qh, kh, vh = (x[0].float().numpy() for x in (q, k, v))
    m = oracle.tile_map(oracle.SPATIAL, 1, 1, oracle.FRAME_MAJOR, F, S, 64, 64)
    assert m["bnd_idx"].size == 0
    o, lse = oracle.attention_rows_tile_aligned(qh, kh, vh, F, S, 0.125, oracle.FRAME_MAJOR,
                                                64, 64, m["counts"], 0, rows)
    oe, le = oracle.attention_rows(qh, kh, vh, F, S, 0.125, oracle.SPATIAL, 1, 1, rows)
    np.testing.assert_allclose(o, oe, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, le, rtol=0, atol=1e-12)


def test_tile_counts_range_is_a_slice_of_the_full_counts():
    F, S = 3, 40
    for order in (oracle.FRAME_MAJOR, oracle.TEMPORAL_ANCHOR_FIRST):
        full = oracle.tile_map(oracle.TEMPORAL, 5, 1, order, F, S, 48, 80)["counts"]
        np.testing.assert_array_equal(
            oracle.tile_counts_range(oracle.TEMPORAL, 5, 1, order, F, S, 48, 80, 1, 3),
            full[1:3])
    with pytest.raises(RuntimeError):
        oracle.tile_counts_range(oracle.TEMPORAL, 5, 1, 0, F, S, 48, 80, 2, 9)


def test_special_cases():
    F, S, d = 3, 20, 16
    N = F * S
    rows = np.arange(N, dtype=np.int32)
    g = torch.Generator().manual_seed(5)
    q = torch.randn(N, d, generator=g).float().numpy()
    k = torch.randn(N, d, generator=g).float().numpy()
    v = torch.randn(N, d, generator=g).float().numpy()
    for t, w in [(oracle.SPATIAL, 1), (oracle.TEMPORAL, 3)]:
        msk = oracle.mask(t, w, 1, F, S).astype(bool)
        # V constant -> O equals that vector for every row, whatever the mask
        c = np.linspace(-2, 3, d).astype(np.float32)
        o, _ = oracle.attention_rows(q, k, np.tile(c, (N, 1)), F, S, 0.25, t, w, 1, rows)
        np.testing.assert_allclose(o, np.tile(c, (N, 1)), atol=1e-12)
        # Q = 0 -> O is the plain mean of V over the kept keys; LSE = ln |K(q)|
        o, lse = oracle.attention_rows(np.zeros_like(q), k, v, F, S, 0.25, t, w, 1, rows)
        mean = np.stack([v[msk[i]].astype(np.float64).mean(0) for i in range(N)])
        np.testing.assert_allclose(o, mean, atol=1e-12)
        np.testing.assert_allclose(lse, np.log(msk.sum(1)), atol=1e-12)
    # a single kept key (one frame, temporal band 0, no anchor) -> O = that V row
    o, lse = oracle.attention_rows(q[:S], k[:S], v[:S], 1, S, 0.25, oracle.TEMPORAL, 0, 0,
                                   np.arange(S, dtype=np.int32))
    np.testing.assert_allclose(o, v[:S].astype(np.float64), atol=1e-15)
    np.testing.assert_allclose(lse, 0.25 * np.einsum("ij,ij->i", q[:S].astype(np.float64),
                                                     k[:S].astype(np.float64)), atol=1e-12)


def test_permute_attend_unpermute_equals_original_order():
    """Check (e): attention computed in a permuted layout, with the mask carried by the
    tokens' own coordinates, comes back equal after the inverse permutation."""
    F, S, d = 5, 12, 16
    N = F * S
    g = torch.Generator().manual_seed(3)
    q, k, v = (torch.randn(N, d, generator=g).float().numpy() for _ in range(3))
    rows = np.arange(N, dtype=np.int32)
    for order in (oracle.TEMPORAL_ANCHOR_FIRST, oracle.TEMPORAL_STRICT):
        perm = oracle.permutation(order, F, S)
        m = oracle.mask(oracle.TEMPORAL, 2, 1, F, S)
        o_ref, _ = oracle.attention_rows(q, k, v, F, S, 0.5, oracle.TEMPORAL, 2, 1, rows)
        # permuted layout: row p holds token perm[p]; the mask follows the tokens
        o_perm = _sdpa64(q[perm], k[perm], v[perm], 0.5, m[np.ix_(perm, perm)])
        back = np.empty_like(o_perm)
        back[perm] = o_perm
        np.testing.assert_allclose(back, o_ref, atol=1e-12)


def test_empty_row_definition():
    # no anchor, spatial band 0, but the query asks for frames that hold no keys is
    # impossible with these masks; an explicit all-masked row only arises without the
    # anchor and with a negative band, which the library rejects.  The oracle's
    # definition for it is O = 0, LSE = -inf.
    F, S, d = 2, 4, 8
    z = np.ones((F * S, d), np.float32)
    o, lse = oracle.attention_rows(z, z, z, F, S, 1.0, oracle.SPATIAL, -1, 0,
                                   np.arange(F * S, dtype=np.int32))
    assert (o == 0).all() and np.isneginf(lse).all()


# ---------------------------------------------------------------------- classifier
def test_classifier_exact_cases():
    F, S, d = 4, 16, 32
    N = F * S
    g = torch.Generator().manual_seed(9)
    q, k, v = (torch.randn(N, d, generator=g).float().numpy() for _ in range(3))
    rows = np.arange(0, N, 3, dtype=np.int32)
    # a spatial band covering all frames equals dense: its deviation is exactly zero
    t, ms, mt = oracle.classify(q, k, v, F, S, 0.2, F - 1, 1, 1, rows)
    assert ms == 0.0 and mt > 0.0 and t == oracle.SPATIAL
    # a temporal band covering the whole frame equals dense
    t, ms, mt = oracle.classify(q, k, v, F, S, 0.2, 0, S - 1, 1, rows)
    assert mt == 0.0 and ms > 0.0 and t == oracle.TEMPORAL


def test_classifier_finds_structured_heads():
    """Structured inputs (frame bias for the first half of the heads, same-position bias
    for the second half) on a reduced grid: the classifier must recover the split."""
    wl = C.Workload("struct_small", 7, 6, 10, 64, [0, 0, 1, 1], [1, 1, 10, 10],
                    [0] * 4, seed=4, structured=True)
    wl.band = [1, 1, 40, 40]
    q, k, v = make_qkv(wl)
    F, S = wl.frames, wl.tokens_per_frame
    rows = np.arange(0, F * S, 7, dtype=np.int32)
    types = []
    for h in range(wl.heads):
        qh, kh, vh = (x[h].float().numpy() for x in (q, k, v))
        t, ms, mt = oracle.classify(qh, kh, vh, F, S, 1.0 / math.sqrt(wl.head_dim),
                                    1, 10, 1, rows)
        types.append(t)
    assert types == [oracle.SPATIAL, oracle.SPATIAL, oracle.TEMPORAL, oracle.TEMPORAL]
