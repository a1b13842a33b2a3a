"""The CTA-pair attention kernel (SVGA_FLAG_CTA_PAIR) on the GPU, through the C ABI,
against the fp64 oracle, with the tolerance of the default kernel (max-abs 2e-2,
relative Frobenius 1e-2, LSE max-abs 1e-3).

The pair kernel takes the work items whose two 128-row blocks both exist and both visit
a key chunk; the others run in the one-CTA kernel within the same call.  The cases
cover items with a ragged second block (the 129-token shape: one valid row), ragged
last key chunks, both head types and orders, queries gathered from frame-major memory,
the split into parts, scores that force many reference raises, and the failure path."""
import math
import time

import numpy as np
import pytest
import torch

from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_spatio_attn_b200 import svga  # noqa: E402
from tests.helpers import (assert_attn_close, lse_to_frame_major, oracle_rows,  # noqa: E402
                           run_sparse_path, sample_rows)

PAIR = svga.FLAG_CTA_PAIR


def check(wl, q, k, v, rows, what):
    o, lse, _ = run_sparse_path(wl, q.cuda(), k.cuda(), v.cuda(), flags=PAIR)
    o = o.float().cpu().numpy()
    lse = lse_to_frame_major(lse.cpu().numpy(), wl, wl.order)
    for h in range(wl.heads):
        ro, rl = oracle_rows(wl, q, k, v, h, rows)
        assert_attn_close(o[h, rows], ro, lse[h, rows], rl, what=f"{what} head {h}")


@pytest.mark.parametrize("N_frames,gh,gw", [(3, 1, 43), (2, 5, 26), (4, 7, 9)])
def test_pair_small_and_ragged_all_rows(N_frames, gh, gw):
    """129, 260 and 252 tokens: pairs whose second block holds 1, 4 or 124 rows."""
    wl = C.Workload("odd_pair", N_frames, gh, gw, 128, [C.SPATIAL, C.TEMPORAL], [0, 3],
                    [C.ORDER_FRAME_MAJOR, C.ORDER_TEMPORAL_MAJOR], seed=9)
    q, k, v = make_qkv(wl)
    check(wl, q, k, v, np.arange(wl.tokens, dtype=np.int32), "ragged pair")


def test_pair_mid_sampled():
    wl = C.mid()
    q, k, v = make_qkv(wl)
    check(wl, q, k, v, sample_rows(wl, 300, seed=3), "mid pair")


def test_pair_headline_sampled():
    wl = C.headline()
    q, k, v = make_qkv(wl)
    check(wl, q, k, v, sample_rows(wl, 60, seed=4), "headline pair")


@pytest.mark.parametrize("direction", [1, -1])
def test_pair_scores_rising_along_the_keys(direction):
    """Scores that grow along the keys to about 150: the reference maximum is raised
    many times per row, passed between the two softmax groups, and O and both groups'
    sums are rescaled each time."""
    wl = C.mid()
    q, k, v = make_qkv(wl)
    q2, k2 = q.clone(), k.clone()
    q2[..., 0] = 16.0
    k2[..., 0] = (torch.linspace(-106.0, 106.0, wl.tokens) * direction).to(torch.bfloat16)
    check(wl, q2, k2, v, sample_rows(wl, 120, seed=11), "rising scores pair")


def test_pair_frame_major_queries_equal_permuted_path():
    """Q gathered from frame-major memory and O / LSE written back to it: the same bits
    as permute -> pair attention -> unpermute."""
    wl = C.mid()
    q, k, v = (x.cuda() for x in make_qkv(wl))
    o_ref, lse_ref, _ = run_sparse_path(wl, q, k, v, flags=PAIR)
    lse_fm = torch.from_numpy(lse_to_frame_major(lse_ref.cpu().numpy(), wl, wl.order))
    prob = svga.ProblemSpec.from_workload(wl)
    bmap = svga.build_block_map(prob)
    kp, vp = torch.empty_like(k), torch.empty_like(v)
    svga.svga_permute_tokens(k, kp, prob)
    svga.svga_permute_tokens(v, vp, prob)
    o = torch.full_like(q, float("nan"))
    lse = torch.empty(wl.heads, wl.tokens, dtype=torch.float32, device="cuda")
    svga.svga_sparse_attention_fwd(q, kp, vp, o, lse, prob, bmap, 1.0 / math.sqrt(wl.head_dim),
                                   PAIR | svga.FLAG_QO_FRAME_MAJOR)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    assert torch.equal(o, o_ref)
    assert torch.equal(lse.cpu(), lse_fm)


def test_pair_parts_equal_single_call():
    """Three parts, each launching the pair kernel over its share of the items, write
    every row once, with the bits of one call."""
    wl = C.mid()
    q, k, v = (x.cuda() for x in make_qkv(wl))
    prob = svga.ProblemSpec.from_workload(wl)
    bmap = svga.build_block_map(prob)
    qp, kp, vp = (torch.empty_like(x) for x in (q, k, v))
    for s, d in ((q, qp), (k, kp), (v, vp)):
        svga.svga_permute_tokens(s, d, prob)
    scale = 1.0 / math.sqrt(wl.head_dim)
    o1 = torch.empty_like(q)
    svga.svga_sparse_attention_fwd(qp, kp, vp, o1, None, prob, bmap, scale, PAIR)
    o3 = torch.full_like(q, float("nan"))
    for part in range(3):
        svga.svga_sparse_attention_fwd_part(qp, kp, vp, o3, None, prob, bmap, scale, PAIR, part, 3)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    assert torch.equal(o3, o1)


def test_pair_stalled_load_times_out_and_context_survives():
    """A K load that never arrives: both CTAs of every pair stop after their bounded
    waits, drain their copies and MMAs, meet at the cluster barrier and release TMEM;
    the status reads SVGA_ERR_TIMEOUT and the next call is exact."""
    wl = C.Workload("odd_pair", 3, 1, 43, 128, [C.SPATIAL, C.TEMPORAL], [0, 3],
                    [C.ORDER_FRAME_MAJOR, C.ORDER_TEMPORAL_MAJOR], seed=9)
    q, k, v = (x.cuda() for x in make_qkv(wl))
    prob = svga.ProblemSpec.from_workload(wl)
    bmap = svga.build_block_map(prob)
    qp, kp, vp = (torch.empty_like(x) for x in (q, k, v))
    for s, d in ((q, qp), (k, kp), (v, vp)):
        svga.svga_permute_tokens(s, d, prob)
    scale = 1.0 / math.sqrt(wl.head_dim)
    o_ref = torch.empty_like(q)
    svga.svga_sparse_attention_fwd(qp, kp, vp, o_ref, None, prob, bmap, scale, PAIR)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    o = torch.zeros_like(q)
    t0 = time.monotonic()
    svga.svga_sparse_attention_fwd(qp, kp, vp, o, None, prob, bmap, scale,
                                   PAIR | svga.FLAG_TEST_STALL)
    torch.cuda.synchronize()
    waited = time.monotonic() - t0
    assert bmap.device_status() == 7          # SVGA_ERR_TIMEOUT
    assert 0.5 < waited < 30.0, waited
    o2 = torch.empty_like(q)
    svga.svga_sparse_attention_fwd(qp, kp, vp, o2, None, prob, bmap, scale, PAIR)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    assert torch.equal(o2, o_ref)
