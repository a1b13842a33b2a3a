"""Block-sparse and dense attention on the GPU (through the C ABI) against the fp64 oracle.

Tolerance (bf16 inputs, fp32 accumulation): max-abs 2e-2, relative Frobenius 1e-2,
LSE max-abs 1e-3.  Full-size workloads are checked on sampled rows, including whole
128-row query blocks in each head's token order (first, middle and last work items,
both blocks of each, so every TMEM lane of both softmax warpgroups) and the ragged last
block."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_spatio_attn_b200 import svga  # noqa: E402
from tests.helpers import (assert_attn_close, lse_to_frame_major, oracle_rows,  # noqa: E402
                           oracle_rows_tile_aligned, run_sparse_path, sample_rows)

_cache = {}


def inputs(wl):
    key = (wl.name, wl.seed, wl.heads, wl.frames, wl.grid_h, wl.grid_w, wl.head_dim)
    if key not in _cache:
        q, k, v = make_qkv(wl)
        _cache.clear()
        _cache[key] = (q, k, v, q.cuda(), k.cuda(), v.cuda())
    return _cache[key]


def check_sparse(wl, rows=None, naive=False, order=None, tile_q=None, tile_k=None):
    q, k, v, qd, kd, vd = inputs(wl)
    order = wl.order if order is None else order
    o, lse, _ = run_sparse_path(wl, qd, kd, vd, naive=naive, order=order, tile_q=tile_q,
                                tile_k=tile_k)
    o = o.float().cpu().numpy()
    lse = lse_to_frame_major(lse.cpu().numpy(), wl, order)
    rows = np.arange(wl.tokens, dtype=np.int32) if rows is None else rows
    for h in range(wl.heads):
        ro, rl = oracle_rows(wl, q, k, v, h, rows)
        assert_attn_close(o[h, rows], ro, lse[h, rows], rl, what=f"{wl.name} head {h}")


def test_tiny_sparse_all_rows():
    check_sparse(C.tiny())


def test_tiny_sparse_naive_b1():
    check_sparse(C.tiny(), naive=True)


def test_tiny_temporal_major_orders():
    check_sparse(C.tiny(), order=[C.ORDER_TEMPORAL_MAJOR, C.ORDER_TEMPORAL_MAJOR])
    check_sparse(C.tiny(), order=[C.ORDER_TEMPORAL_MAJOR_STRICT] * 2)


def test_mid_sparse():
    wl = C.mid()
    check_sparse(wl, rows=sample_rows(wl, 600))


def test_mid_sparse_naive_b1_equals_b2():
    wl = C.mid()
    q, k, v, qd, kd, vd = inputs(wl)
    o1, l1, _ = run_sparse_path(wl, qd, kd, vd, naive=False)
    o2, l2, _ = run_sparse_path(wl, qd, kd, vd, naive=True)
    # the same arithmetic in the same order: masking only removes pairs that are kept
    # anyway on full tiles, so the results agree to the last bit
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)


@pytest.mark.parametrize("tq,tk", [(64, 64), (256, 128), (128, 256), (256, 256), (64, 128)])
def test_mid_tile_sizes(tq, tk):
    wl = C.mid()
    check_sparse(wl, rows=sample_rows(wl, 200, seed=tq + tk), tile_q=tq, tile_k=tk)


def test_mid_frame_major_temporal():
    wl = C.mid()
    check_sparse(wl, rows=sample_rows(wl, 200, seed=3, orders=[C.ORDER_FRAME_MAJOR]),
                 order=[C.ORDER_FRAME_MAJOR] * 4)


def test_headline_sparse_sampled():
    wl = C.headline()
    check_sparse(wl, rows=sample_rows(wl, 160))


def test_permstudy_strict_order_sampled():
    wl = C.permutation_study(C.ORDER_TEMPORAL_MAJOR_STRICT)
    check_sparse(wl.__class__(**{**wl.__dict__, "head_type": wl.head_type[:2],
                                 "band": wl.band[:2], "order": wl.order[:2]}),
                 rows=sample_rows(wl, 120))


def dense_check(wl, rows):
    q, k, v, qd, kd, vd = inputs(wl)
    o = torch.empty_like(qd)
    lse = torch.empty(wl.heads, wl.tokens, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    svga.svga_dense_attention_fwd(qd, kd, vd, o, lse, 1.0 / math.sqrt(wl.head_dim), st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    for h in range(wl.heads):
        ro, rl = oracle_rows(wl, q, k, v, h, rows, type_=oracle.DENSE, band=0)
        assert_attn_close(o[h, rows], ro, lse[h, rows], rl, what=f"dense {wl.name} head {h}")


def test_tiny_dense_all_rows():
    wl = C.tiny()
    dense_check(wl, np.arange(wl.tokens, dtype=np.int32))


def test_mid_dense_sampled():
    wl = C.mid()
    dense_check(wl, sample_rows(wl, 300))


def test_headline_dense_sampled():
    wl = C.headline()
    wl2 = wl.__class__(**{**wl.__dict__, "head_type": wl.head_type[:3], "band": wl.band[:3],
                          "order": wl.order[:3]})
    dense_check(wl2, sample_rows(wl2, 96))


@pytest.mark.parametrize("N_frames,gh,gw,d", [(2, 5, 10, 128), (1, 7, 9, 64), (3, 1, 43, 128)])
def test_small_and_ragged_shapes(N_frames, gh, gw, d):
    """One block, an odd number of blocks, single frame, N < 128."""
    wl = C.Workload("odd", N_frames, gh, gw, d, [C.SPATIAL, C.TEMPORAL], [0, 3],
                    [C.ORDER_FRAME_MAJOR, C.ORDER_TEMPORAL_MAJOR], seed=9)
    check_sparse(wl)
    dense_check(wl, np.arange(wl.tokens, dtype=np.int32))


def test_special_values():
    """V constant -> O equals it; Q = 0 -> plain masked mean of V (via the oracle)."""
    wl = C.mid()
    q, k, v, qd, kd, vd = inputs(wl)
    c = torch.linspace(-1, 1, wl.head_dim).to(torch.bfloat16)
    vc = c.expand(wl.heads, wl.tokens, wl.head_dim).contiguous().cuda()
    o, _, _ = run_sparse_path(wl, qd, kd, vc)
    err = (o.float().cpu() - c.float()).abs().max().item()
    assert err <= 1e-2
    qz = torch.zeros_like(qd)
    o, lse, _ = run_sparse_path(wl, qz, kd, vd)
    rows = sample_rows(wl, 100, seed=5)
    o = o.float().cpu().numpy()
    lse = lse_to_frame_major(lse.cpu().numpy(), wl, wl.order)
    zq = torch.zeros_like(q)
    for h in range(wl.heads):
        ro, rl = oracle_rows(wl, zq, k, v, h, rows)
        assert_attn_close(o[h, rows], ro, lse[h, rows], rl, what=f"Q=0 head {h}")


@pytest.mark.parametrize("direction", [1, -1])
def test_scores_rising_along_the_keys(direction):
    """Q and K share one direction whose weight in K grows with the token index (down
    to about -150, up to about +150 in units of the scaled score): with direction 1
    each new tile lies far above the reference maximum the kernels take from the
    first tile of a row, so the rescaling of O and of the running sums runs many times
    per row (with -1 it never does).  Both kernels (one CTA, and a CTA pair) still
    equal the oracle."""
    wl = C.mid()
    q, k, v, _, _, _ = inputs(wl)
    q2, k2 = q.clone(), k.clone()
    q2[..., 0] = 16.0
    ramp = torch.linspace(-106.0, 106.0, wl.tokens) * direction
    k2[..., 0] = ramp.to(torch.bfloat16)
    o, lse, _ = run_sparse_path(wl, q2.cuda(), k2.cuda(), v.cuda())
    rows = sample_rows(wl, 120, seed=11)
    o = o.float().cpu().numpy()
    lse = lse_to_frame_major(lse.cpu().numpy(), wl, wl.order)
    for h in range(wl.heads):
        ro, rl = oracle_rows(wl, q2, k2, v, h, rows)
        assert_attn_close(o[h, rows], ro, lse[h, rows], rl, what=f"rising scores head {h}")
    # the same through the one-CTA kernel (keys gathered from frame-major memory)
    prob = svga.ProblemSpec.from_workload(wl)
    bmap = svga.build_block_map(prob)
    qd = q2.cuda()
    qp = torch.empty_like(qd)
    svga.svga_permute_tokens(qd, qp, prob)
    op = torch.empty_like(qd)
    lsep = torch.empty(wl.heads, wl.tokens, dtype=torch.float32, device="cuda")
    svga.svga_sparse_attention_fwd(qp, k2.cuda(), v.cuda(), op, lsep, prob, bmap,
                                   1.0 / math.sqrt(wl.head_dim), svga.FLAG_KV_FRAME_MAJOR)
    o1 = torch.empty_like(qd)
    svga.svga_unpermute_tokens(op, o1, prob)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    o1 = o1.float().cpu().numpy()
    l1 = lse_to_frame_major(lsep.cpu().numpy(), wl, wl.order)
    for h in range(wl.heads):
        ro, rl = oracle_rows(wl, q2, k2, v, h, rows)
        assert_attn_close(o1[h, rows], ro, l1[h, rows], rl, what=f"rising scores, one CTA, head {h}")


def test_repeatable_bitwise():
    wl = C.mid()
    q, k, v, qd, kd, vd = inputs(wl)
    o1, l1, _ = run_sparse_path(wl, qd, kd, vd)
    o2, l2, _ = run_sparse_path(wl, qd, kd, vd)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ------------------------------------------------- tile-aligned traversal (B3, opt-in)
def check_tile_aligned(wl, rows=None, order=None, tile_q=None, tile_k=None):
    q, k, v, qd, kd, vd = inputs(wl)
    order = wl.order if order is None else order
    tq = wl.tile_q if tile_q is None else tile_q
    tk = wl.tile_k if tile_k is None else tile_k
    o, lse, _ = run_sparse_path(wl, qd, kd, vd, order=order, tile_q=tq, tile_k=tk,
                                flags=svga.FLAG_TILE_ALIGNED)
    o = o.float().cpu().numpy()
    lse = lse_to_frame_major(lse.cpu().numpy(), wl, order)
    rows = np.arange(wl.tokens, dtype=np.int32) if rows is None else rows
    for h in range(wl.heads):
        ro, rl = oracle_rows_tile_aligned(wl, q, k, v, h, rows, order[h], tq, tk)
        assert_attn_close(o[h, rows], ro, lse[h, rows], rl, what=f"{wl.name} B3 head {h}")


def test_tiny_tile_aligned_all_rows():
    check_tile_aligned(C.tiny(), tile_q=128, tile_k=64)


@pytest.mark.parametrize("tq,tk", [(128, 128), (256, 128), (128, 64), (256, 256)])
def test_mid_tile_aligned_sampled(tq, tk):
    wl = C.mid()
    check_tile_aligned(wl, rows=sample_rows(wl, 300), tile_q=tq, tile_k=tk)


def test_mid_tile_aligned_frame_major_temporal():
    """Temporal heads left frame-major: most visited tiles are boundary tiles there, so
    snapping keeps many more pairs than the exact mask."""
    wl = C.mid()
    check_tile_aligned(wl, rows=sample_rows(wl, 200, orders=[C.ORDER_FRAME_MAJOR]),
                       order=[C.ORDER_FRAME_MAJOR] * wl.heads)


def test_headline_tile_aligned():
    """Headline size: rows of three q-tiles per head against the oracle (the first, a
    middle one and the ragged last one)."""
    wl = C.headline()
    q, k, v, qd, kd, vd = inputs(wl)
    F, S = wl.frames, wl.tokens_per_frame
    o3, l3, _ = run_sparse_path(wl, qd, kd, vd, flags=svga.FLAG_TILE_ALIGNED)
    n_q = -(-wl.tokens // wl.tile_q)
    o3n = o3.float().cpu().numpy()
    for h in range(wl.heads):
        pos_of_row = np.empty(wl.tokens, np.int64)
        pos_of_row[oracle.permutation(wl.order[h], F, S)] = np.arange(wl.tokens)
        qt = pos_of_row // wl.tile_q
        rows = []
        for i in (0, n_q // 2, n_q - 1):
            rr = np.nonzero(qt == i)[0]
            rows.extend(rr[:: max(1, rr.size // 12)].tolist())
        rows = np.array(sorted(rows), np.int32)
        ro, rl = oracle_rows_tile_aligned(wl, q, k, v, h, rows, wl.order[h], wl.tile_q,
                                          wl.tile_k)
        lse = lse_to_frame_major(l3[h:h + 1].cpu().numpy(), wl, [wl.order[h]])[0]
        assert_attn_close(o3n[h, rows], ro, lse[rows], rl, what=f"headline B3 head {h}")


def test_tile_aligned_flag_validation():
    wl = C.tiny()
    q, k, v, qd, kd, vd = inputs(wl)
    with pytest.raises(svga.SvgaError) as e:
        run_sparse_path(wl, qd, kd, vd, tile_q=64, tile_k=128, flags=svga.FLAG_TILE_ALIGNED)
    assert e.value.status == 4
    for bad in (svga.FLAG_TILE_ALIGNED | svga.FLAG_NAIVE_B1, 1 << 8):   # unknown bit
        with pytest.raises(svga.SvgaError) as e:
            run_sparse_path(wl, qd, kd, vd, flags=bad)
        assert e.value.status == 1


# ----------------------------------------------------- one problem split into parts
def run_parts(wl, num_parts, flags=0):
    """Every part into its own NaN-filled buffers; returns (single-call O, LSE, per-part
    O list, per-part LSE list), all in each head's token order."""
    q, k, v, qd, kd, vd = inputs(wl)
    prob = svga.ProblemSpec.from_workload(wl)
    bmap = svga.build_block_map(prob)
    qp, kp, vp = (torch.empty_like(x) for x in (qd, kd, vd))
    for s, d in ((qd, qp), (kd, kp), (vd, vp)):
        svga.svga_permute_tokens(s, d, prob)
    scale = 1.0 / math.sqrt(wl.head_dim)
    o = torch.empty_like(qd)
    lse = torch.empty(wl.heads, wl.tokens, dtype=torch.float32, device="cuda")
    svga.svga_sparse_attention_fwd(qp, kp, vp, o, lse, prob, bmap, scale, flags)
    ops, lps = [], []
    for r in range(num_parts):
        op = torch.full_like(qd, float("nan"))
        lp = torch.full_like(lse, float("nan"))
        svga.svga_sparse_attention_fwd_part(qp, kp, vp, op, lp, prob, bmap, scale, flags, r,
                                            num_parts)
        ops.append(op)
        lps.append(lp)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    return o, lse, ops, lps


@pytest.mark.parametrize("num_parts", [1, 3, 8])
def test_mid_parts_write_every_row_once_and_match(num_parts):
    o, lse, ops, lps = run_parts(C.mid(), num_parts)
    written = torch.stack([~torch.isnan(op.float()).any(dim=-1) for op in ops])  # [P,H,N]
    assert (written.sum(0) == 1).all()
    for op, lp, w in zip(ops, lps, written):
        assert (torch.isnan(op.float()).all(dim=-1) == ~w).all()   # untouched rows stay NaN
        assert torch.equal(op[w], o[w])
        assert torch.equal(lp[w], lse[w])
        assert torch.isnan(lp[~w]).all()


def test_headline_eight_parts_match_single_call():
    o, lse, ops, lps = run_parts(C.headline(), 8, flags=0)
    comb = torch.zeros_like(o)
    count = torch.zeros(o.shape[:2], dtype=torch.int32, device=o.device)
    for op in ops:
        w = ~torch.isnan(op.float()).any(dim=-1)
        comb[w] = op[w]
        count += w.int()
    assert (count == 1).all()
    assert torch.equal(comb, o)


def test_part_argument_checks():
    wl = C.tiny()
    q, k, v, qd, kd, vd = inputs(wl)
    prob = svga.ProblemSpec.from_workload(wl)
    bmap = svga.build_block_map(prob)
    o = torch.empty_like(qd)
    for part, n in ((1, 1), (-1, 2), (0, 0), (0, 5000)):
        with pytest.raises(svga.SvgaError) as e:
            svga.svga_sparse_attention_fwd_part(qd, kd, vd, o, None, prob, bmap, 0.125, 0, part, n)
        assert e.value.status == 1


# ------------------------------- Q and O frame-major (only K and V permuted)
@pytest.mark.parametrize("name,flags,tiles", [
    ("tiny", 0, None), ("mid", 0, None), ("mid", svga.FLAG_NAIVE_B1, None),
    ("mid", svga.FLAG_TILE_ALIGNED, (256, 128)), ("mid", 0, (64, 64)), ("headline", 0, None)])
def test_qo_frame_major_equals_permuted_path(name, flags, tiles):
    """The kernel's own gather of Q rows and scatter of O rows gives the same bits as
    permute(Q) -> attention -> unpermute(O), and LSE lands at the frame-major token."""
    wl = C.ALL[name]()
    if tiles:
        wl = wl.with_tile(*tiles)
    q, k, v, qd, kd, vd = inputs(wl)
    o_ref, lse_ref, _ = run_sparse_path(wl, qd, kd, vd, flags=flags)
    lse_ref = lse_to_frame_major(lse_ref.cpu().numpy(), wl, wl.order)
    prob = svga.ProblemSpec.from_workload(wl)
    bmap = svga.build_block_map(prob)
    kp, vp = torch.empty_like(kd), torch.empty_like(vd)
    svga.svga_permute_tokens(kd, kp, prob)
    svga.svga_permute_tokens(vd, vp, prob)
    o = torch.full_like(qd, float("nan"))
    lse = torch.empty(wl.heads, wl.tokens, dtype=torch.float32, device="cuda")
    for part in range(2):   # two parts: each writes only its own rows, together all rows
        svga.svga_sparse_attention_fwd_part(qd, kp, vp, o, lse, prob, bmap,
                                            1.0 / math.sqrt(wl.head_dim),
                                            flags | svga.FLAG_QO_FRAME_MAJOR, part, 2)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    assert torch.equal(o, o_ref)
    np.testing.assert_array_equal(lse.cpu().numpy(), lse_ref)
    if name == "headline" and flags == 0:
        # the launch the bench times, checked against the oracle directly as well
        rows = sample_rows(wl, 96)
        on, ln = o.float().cpu().numpy(), lse.cpu().numpy()
        for h in (0, wl.heads - 1):          # one spatial and one temporal head
            ro, rl = oracle_rows(wl, q, k, v, h, rows)
            assert_attn_close(on[h, rows], ro, ln[h, rows], rl, what=f"headline QO-FM head {h}")


# ------------------------------- Q, K, V and O frame-major (nothing permuted)
@pytest.mark.parametrize("name,flags,tiles,order", [
    ("tiny", 0, None, C.ORDER_TEMPORAL_MAJOR), ("tiny", 0, (128, 64), C.ORDER_TEMPORAL_MAJOR_STRICT),
    ("mid", 0, None, None), ("mid", svga.FLAG_NAIVE_B1, None, None),
    ("mid", svga.FLAG_TILE_ALIGNED, (256, 128), None), ("mid", 0, (64, 64), None),
    ("mid", 0, (128, 256), C.ORDER_TEMPORAL_MAJOR_STRICT), ("odd", 0, None, None),
    ("headline", 0, None, None)])
def test_all_frame_major_equals_permuted_path(name, flags, tiles, order):
    """The kernel's gather of the key rows (K and V read from frame-major memory) fills
    the stages with the same bits the tile load of permuted K and V gives: O and LSE
    equal the permute -> attention -> unpermute path bit for bit, with K and V alone
    frame-major and with every tensor frame-major."""
    if name == "odd":   # one frame more than a power of two, rows not a multiple of 8
        wl = C.Workload("odd_fm", 9, 5, 7, 64, [0, 1, 1], [1, 2, 0],
                        [C.ORDER_FRAME_MAJOR, C.ORDER_TEMPORAL_MAJOR,
                         C.ORDER_TEMPORAL_MAJOR_STRICT], seed=21)
    else:
        wl = C.ALL[name]()
    if tiles:
        wl = wl.with_tile(*tiles)
    orders = wl.order if order is None else [order if t == C.TEMPORAL else o
                                             for t, o in zip(wl.head_type, wl.order)]
    q, k, v, qd, kd, vd = inputs(wl)
    o_ref, lse_ref, _ = run_sparse_path(wl, qd, kd, vd, order=orders, flags=flags)
    lse_fm = lse_to_frame_major(lse_ref.cpu().numpy(), wl, orders)
    prob = svga.ProblemSpec.from_workload(wl, order=orders)
    bmap = svga.build_block_map(prob)
    scale = 1.0 / math.sqrt(wl.head_dim)
    # K and V frame-major, Q and O in each head's order
    qp = torch.empty_like(qd)
    svga.svga_permute_tokens(qd, qp, prob)
    op = torch.full_like(qd, float("nan"))
    lse = torch.empty(wl.heads, wl.tokens, dtype=torch.float32, device="cuda")
    svga.svga_sparse_attention_fwd(qp, kd, vd, op, lse, prob, bmap, scale,
                                   flags | svga.FLAG_KV_FRAME_MAJOR)
    o = torch.empty_like(qd)
    svga.svga_unpermute_tokens(op, o, prob)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)
    # every tensor frame-major, in two parts
    o = torch.full_like(qd, float("nan"))
    for part in range(2):
        svga.svga_sparse_attention_fwd_part(
            qd, kd, vd, o, lse, prob, bmap, scale,
            flags | svga.FLAG_QO_FRAME_MAJOR | svga.FLAG_KV_FRAME_MAJOR, part, 2)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    assert torch.equal(o, o_ref)
    np.testing.assert_array_equal(lse.cpu().numpy(), lse_fm)
    if name in ("odd", "headline") and flags == 0:
        rows = sample_rows(wl, 96) if name == "headline" else np.arange(wl.tokens, dtype=np.int32)
        on, ln = o.float().cpu().numpy(), lse.cpu().numpy()
        for h in ((0, wl.heads - 1) if name == "headline" else range(wl.heads)):
            ro, rl = oracle_rows(wl, q, k, v, h, rows)
            assert_attn_close(on[h, rows], ro, ln[h, rows], rl, what=f"{name} all-FM head {h}")


def test_maximum_head_count():
    """4,096 heads (the largest count the library takes), 2 frames of 4x6 tokens, d = 64:
    the per-head parameters travel as kernel parameters sized for that many heads.
    Block map, permutation, attention and classification run for every head; a sample
    of heads is checked against the oracle."""
    H = 4096
    types = [C.SPATIAL if h % 2 == 0 else C.TEMPORAL for h in range(H)]
    wl = C.Workload("maxheads", 2, 4, 6, 64, types, [0 if t == C.SPATIAL else 5 for t in types],
                    [C.ORDER_FRAME_MAJOR if t == C.SPATIAL else C.ORDER_TEMPORAL_MAJOR
                     for t in types], seed=13)
    q, k, v, qd, kd, vd = inputs(wl)
    o, lse, bmap = run_sparse_path(wl, qd, kd, vd)
    svga.svga_validate_block_map(svga.ProblemSpec.from_workload(wl), bmap)
    o = o.float().cpu().numpy()
    lse = lse_to_frame_major(lse.cpu().numpy(), wl, wl.order)
    rows = np.arange(wl.tokens, dtype=np.int32)
    for h in (0, 1, 2047, 4094, 4095):
        ro, rl = oracle_rows(wl, q, k, v, h, rows)
        assert_attn_close(o[h], ro, lse[h], rl, what=f"maxheads head {h}")
    prob = svga.ProblemSpec.from_workload(wl)
    t, _ = svga.svga_classify_heads(qd, kd, vd, prob, [1] * H, [3] * H, None, 8,
                                    1.0 / math.sqrt(64))
    assert len(t) == H and set(t) <= {0, 1}
