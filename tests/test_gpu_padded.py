"""The padded layout (problem.frame_pad, the exact reading of the tile-aligned
traversal: ainews.tenesys.com, "Co sie zmienilo?" item 4; oossa.com, opening paragraph)
on the GPU, through the C ABI, against the oracle.

* permutation into and out of the padded layout: bit-exact against
  oracle.permutation_padded, positions without a token zero;
* block map: classes and lists bit-exact against oracle.tile_map_padded, and the
  library's own host validation passes;
* attention: the kept pairs are those of the unpadded problem, so O and LSE are checked
  against the exact oracle (tolerance as everywhere: max-abs 2e-2, relative Frobenius
  1e-2, LSE 1e-3); rows of the permuted output without a token read O = 0, lse = -inf.
"""
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
from tests.helpers import assert_attn_close, oracle_rows, sample_rows  # noqa: E402


def padded_problem(wl, frame_pad, order=None, tiles=None):
    tq, tk = tiles or (wl.tile_q, wl.tile_k)
    return svga.ProblemSpec.from_workload(wl, order=order, tile_q=tq, tile_k=tk,
                                          frame_pad=frame_pad)


CASES = [  # (workload, order override, tiles, frame_pad)
    ("tiny", None, (64, 64), 64),
    ("tiny", [C.ORDER_FRAME_MAJOR, C.ORDER_TEMPORAL_MAJOR_STRICT], (64, 64), 128),
    ("mid", None, (128, 128), 128),
    ("mid", None, (64, 128), 256),
    ("mid", [C.ORDER_FRAME_MAJOR] * 4, (128, 64), 128),
    ("odd", None, (64, 64), 64),
]


def workload(name):
    if name == "odd":   # 35 tokens per frame, head_dim 64, all three orders
        return C.Workload("odd_pad", 9, 5, 7, 64, [0, 1, 1], [1, 2, 0],
                          [C.ORDER_FRAME_MAJOR, C.ORDER_TEMPORAL_MAJOR,
                           C.ORDER_TEMPORAL_MAJOR_STRICT], seed=23)
    return C.ALL[name]()


def ids(c):
    return f"{c[0]}-{'orders' if c[1] else 'own'}-{c[2][0]}x{c[2][1]}-pad{c[3]}"


@pytest.mark.parametrize("case", CASES, ids=ids)
def test_permutation_bit_exact(case):
    name, order, tiles, fp = case
    wl = workload(name)
    order = wl.order if order is None else order
    prob = padded_problem(wl, fp, order, tiles)
    q, _, _ = make_qkv(wl)
    qd = q.cuda()
    dst = torch.full((wl.heads, prob.rows, wl.head_dim), float("nan"), dtype=torch.bfloat16,
                     device="cuda")
    svga.svga_permute_tokens(qd, dst, prob)
    back = torch.empty_like(qd)
    svga.svga_unpermute_tokens(dst, back, prob)
    torch.cuda.synchronize()
    Sp = oracle.frame_stride(wl.tokens_per_frame, fp)
    assert prob.rows == wl.frames * Sp
    got = dst.cpu()
    for h in range(wl.heads):
        perm = oracle.permutation_padded(order[h], wl.frames, wl.tokens_per_frame, Sp)
        has = perm >= 0
        assert torch.equal(got[h][torch.from_numpy(has)], q[h][torch.from_numpy(perm[has])])
        assert bool((got[h][torch.from_numpy(~has)] == 0).all())
    assert torch.equal(back.cpu(), q)
    # the map-driven permutation gives the same bits
    bmap = svga.build_block_map(prob)
    dst2 = torch.empty_like(dst)
    svga.svga_permute_tokens_mapped(qd, dst2, prob, bmap)
    back2 = torch.empty_like(qd)
    svga.svga_unpermute_tokens_mapped(dst2, back2, prob, bmap)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    assert torch.equal(dst2, dst) and torch.equal(back2, qd)


@pytest.mark.parametrize("case", CASES, ids=ids)
def test_map_bit_exact(case):
    name, order, tiles, fp = case
    wl = workload(name)
    order = wl.order if order is None else order
    tq, tk = tiles
    prob = padded_problem(wl, fp, order, tiles)
    bmap = svga.build_block_map(prob)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    svga.svga_validate_block_map(prob, bmap)
    F, S = wl.frames, wl.tokens_per_frame
    Sp = oracle.frame_stride(S, fp)
    NP = F * Sp
    nq, nk = -(-NP // tq), -(-NP // tk)
    cls = bmap.cls[: wl.heads * nq * nk].cpu().numpy().reshape(wl.heads, nq, nk)
    fptr = bmap.full_ptr.cpu().numpy()
    bptr = bmap.bnd_ptr.cpu().numpy()
    fidx = bmap.full_idx[: fptr[-1]].cpu().numpy()
    bidx = bmap.bnd_idx[: bptr[-1]].cpu().numpy()
    for h in range(wl.heads):
        m = oracle.tile_map_padded(wl.head_type[h], wl.band[h], wl.anchor_frame0, order[h],
                                   F, S, Sp, tq, tk)
        np.testing.assert_array_equal(cls[h], m["cls"], err_msg=f"head {h}")
        r0 = h * nq
        np.testing.assert_array_equal(fptr[r0: r0 + nq + 1] - fptr[r0], m["full_ptr"])
        np.testing.assert_array_equal(bptr[r0: r0 + nq + 1] - bptr[r0], m["bnd_ptr"])
        np.testing.assert_array_equal(fidx[fptr[r0]: fptr[r0 + nq]], m["full_idx"])
        np.testing.assert_array_equal(bidx[bptr[r0]: bptr[r0 + nq]], m["bnd_idx"])


def run_padded(wl, prob, q, k, v, flags=0):
    """Frame-major Q/K/V on the GPU -> padded permutation -> attention -> unpermute.
    Returns (O frame-major, O and lse in padded positions)."""
    bmap = svga.build_block_map(prob)
    shape = (wl.heads, prob.rows, wl.head_dim)
    qp, kp, vp = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    for s, d in ((q, qp), (k, kp), (v, vp)):
        svga.svga_permute_tokens(s, d, prob)
    op = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((wl.heads, prob.rows), float("nan"), device="cuda")
    svga.svga_sparse_attention_fwd(qp, kp, vp, op, lse, prob, bmap,
                                   1.0 / math.sqrt(wl.head_dim), flags)
    o = torch.empty_like(q)
    svga.svga_unpermute_tokens(op, o, prob)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    return o, op, lse


def check_against_oracle(wl, order, tiles, fp, rows=None, heads=None, flags=0):
    order = wl.order if order is None else order
    prob = padded_problem(wl, fp, order, tiles)
    q, k, v = make_qkv(wl)
    o, op, lse = run_padded(wl, prob, q.cuda(), k.cuda(), v.cuda(), flags)
    F, S = wl.frames, wl.tokens_per_frame
    Sp = oracle.frame_stride(S, fp)
    on, opn, ln = o.float().cpu().numpy(), op.float().cpu().numpy(), lse.cpu().numpy()
    rows = np.arange(wl.tokens, dtype=np.int32) if rows is None else rows
    for h in (range(wl.heads) if heads is None else heads):
        perm = oracle.permutation_padded(order[h], F, S, Sp)
        lse_fm = np.empty(wl.tokens)
        lse_fm[perm[perm >= 0]] = ln[h, perm >= 0]
        ro, rl = oracle_rows(wl, q, k, v, h, rows)
        assert_attn_close(on[h, rows], ro, lse_fm[rows], rl, what=f"{wl.name} pad head {h}")
        # positions without a token: O = 0, lse = -inf
        holes = perm < 0
        assert (opn[h, holes] == 0).all() and np.isneginf(ln[h, holes]).all()


@pytest.mark.parametrize("case", CASES, ids=ids)
def test_attention_all_rows_small(case):
    name, order, tiles, fp = case
    wl = workload(name)
    if wl.tokens > 1000:
        rows = sample_rows(wl, 96)
    else:
        rows = None
    check_against_oracle(wl, order, tiles, fp, rows=rows)


def test_attention_naive_traversal():
    """Every visited tile through the masked path (B1) on the padded layout."""
    check_against_oracle(C.mid(), None, (128, 128), 128, rows=sample_rows(C.mid(), 64),
                         flags=svga.FLAG_NAIVE_B1)


def test_attention_headline_sampled():
    """The headline workload with frames padded to 3,712 positions (29 tiles of 128):
    one spatial and one temporal head on whole sampled 128-row blocks."""
    wl = C.headline()
    check_against_oracle(wl, None, (128, 128), 128, rows=sample_rows(wl, 96),
                         heads=(0, wl.heads - 1))
