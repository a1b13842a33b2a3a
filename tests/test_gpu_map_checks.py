"""A block map handed to a call on another problem is refused on the device.

The attention kernel walks the plan of a map the caller built ("Accelerating
Spatio-Temporal Attention for Video Diffusion on TPUs", aihirek.info, section "A
TPU-kernel kialakitasa dontonek bizonyult": skip, full and boundary tiles come from the
map).  The host can only check that the plan is large enough; a map built for a larger
problem passes that check.  The kernels therefore compare the plan's header, work items
and head info with the call before using any offset: on a mismatch the status word reads
SVGA_ERR_INVALID_ARG, the outputs are untouched, and the next call with the right map
gives the same bits as before."""
import math

import pytest
import torch

from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_spatio_attn_b200 import svga  # noqa: E402


def _no_anchor(wl):
    w = C.Workload(**{**wl.__dict__})
    w.anchor_frame0 = 0
    return w


@pytest.mark.parametrize("small,big", [
    ("tiny", "mid"),            # other shape, head dim and tiles
    ("mid", "headline"),        # other shape
    ("mid", "mid_no_anchor"),   # same shape, the map built without the frame-0 anchor
], ids=["tiny<-mid", "mid<-headline", "mid<-mid-no-anchor"])
def test_map_of_another_problem_is_refused(small, big):
    wl = C.ALL[small]()
    wl_big = _no_anchor(C.mid()) if big == "mid_no_anchor" else C.ALL[big]()
    prob = svga.ProblemSpec.from_workload(wl)
    prob_big = svga.ProblemSpec.from_workload(wl_big)
    scale = 1.0 / math.sqrt(wl.head_dim)
    q, k, v = (x.cuda() for x in make_qkv(wl))
    qp, kp, vp = (torch.empty_like(x) for x in (q, k, v))
    for s, d in ((q, qp), (k, kp), (v, vp)):
        svga.svga_permute_tokens(s, d, prob)
    right = svga.build_block_map(prob)
    wrong = svga.build_block_map(prob_big)
    assert wrong.sizes["plan_bytes"] >= right.sizes["plan_bytes"]   # passes the host check

    o_ref = torch.empty_like(q)
    lse_ref = torch.empty(wl.heads, wl.tokens, dtype=torch.float32, device="cuda")
    svga.svga_sparse_attention_fwd(qp, kp, vp, o_ref, lse_ref, prob, right, scale)
    torch.cuda.synchronize()
    assert right.device_status() == 0

    for flags, part, parts in ((0, 0, 1), (svga.FLAG_QO_FRAME_MAJOR, 1, 2),
                               (svga.FLAG_KV_FRAME_MAJOR | svga.FLAG_TILE_ALIGNED, 0, 1)):
        if (flags & svga.FLAG_TILE_ALIGNED) and wl.tile_q < 128:
            continue
        o = torch.full_like(q, float("nan"))
        lse = torch.full((wl.heads, wl.tokens), float("nan"), device="cuda")
        svga.svga_sparse_attention_fwd_part(q if flags & svga.FLAG_QO_FRAME_MAJOR else qp,
                                            k if flags & svga.FLAG_KV_FRAME_MAJOR else kp,
                                            v if flags & svga.FLAG_KV_FRAME_MAJOR else vp,
                                            o, lse, prob, wrong, scale, flags, part, parts)
        torch.cuda.synchronize()
        assert wrong.device_status() == 1, (flags, wrong.device_status())
        assert bool(torch.isnan(o.float()).all()), "O was written"
        assert bool(torch.isnan(lse).all()), "lse was written"

    # the next call with the right map on the same context: same bits as before
    o = torch.empty_like(q)
    lse = torch.empty_like(lse_ref)
    svga.svga_sparse_attention_fwd(qp, kp, vp, o, lse, prob, right, scale)
    torch.cuda.synchronize()
    assert right.device_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)

    # the permutations that read the orders from a plan refuse it as well
    for fn in (svga.svga_permute_tokens_mapped, svga.svga_unpermute_tokens_mapped):
        wrong.status.zero_()
        dst = torch.full_like(q, float("nan"))
        fn(q, dst, prob, wrong)
        torch.cuda.synchronize()
        if big == "mid_no_anchor":
            # the orders do not depend on the anchor: the map is valid for a permutation
            assert wrong.device_status() == 0
            assert not bool(torch.isnan(dst.float()).any())
        else:
            assert wrong.device_status() == 1
            assert bool(torch.isnan(dst.float()).all()), "dst was written"
    # and accept the right one, bit-identical to the host-ordered permutation
    dst = torch.empty_like(q)
    svga.svga_permute_tokens_mapped(q, dst, prob, right)
    torch.cuda.synchronize()
    assert right.device_status() == 0 and torch.equal(dst, qp)


@pytest.mark.parametrize("name", ["mid", "headline"])
def test_plan_items_match_the_cpu_restatement(name):
    """The work items of the built plan (the order the parts of a split problem are dealt
    from) equal the CPU restatement the multi-rank bookkeeping tests use: items longest
    first from the oracle's tile classes, with their visited-chunk counts."""
    import numpy as np
    from tests.test_multirank import plan_items_cpu
    wl = C.ALL[name]()
    bmap = svga.build_block_map(svga.ProblemSpec.from_workload(wl))
    torch.cuda.synchronize()
    n_qblk = -(-wl.tokens // 128)
    n_items = wl.heads * (-(-n_qblk // 2))
    raw = bmap.plan[64 + 16 * wl.heads: 64 + 16 * (wl.heads + n_items)].cpu().numpy()
    items = np.frombuffer(raw.tobytes(), dtype=np.int32).reshape(n_items, 4)
    want, _ = plan_items_cpu(wl, with_lengths=True)
    got = [(int(h), int(b0), int(n)) for h, b0, _, n in items]
    assert got == want
