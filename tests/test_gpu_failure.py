"""Failure path on the GPU, without a fault: a K load that never arrives (the test hook
SVGA_FLAG_TEST_STALL) makes the attention kernel's bounded waits run out.  Every role
then stops, the copies in flight are drained, TMEM is released and the status word reads
SVGA_ERR_TIMEOUT; the CUDA context stays usable and the next normal call is exact."""
import math
import time

import pytest
import torch

from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_spatio_attn_b200 import svga  # noqa: E402


@pytest.mark.parametrize("frame_major", [False, True], ids=["tile-load", "row-gather"])
def test_stalled_load_times_out_and_context_survives(frame_major):
    """tile-load: permuted inputs, every chunk loaded by the TMA producer; row-gather:
    frame-major inputs, the temporal head's chunks gathered row by row."""
    # two work items: one wave of CTAs, about one second of waiting
    wl = C.tiny().with_orders(C.ORDER_TEMPORAL_MAJOR)
    q, k, v = (x.cuda() for x in make_qkv(wl))
    prob = svga.ProblemSpec.from_workload(wl)
    bmap = svga.build_block_map(prob)
    if frame_major:
        qp, kp, vp = q, k, v
        flags = svga.FLAG_QO_FRAME_MAJOR | svga.FLAG_KV_FRAME_MAJOR
    else:
        qp, kp, vp = (torch.empty_like(x) for x in (q, k, v))
        for s, d in ((q, qp), (k, kp), (v, vp)):
            svga.svga_permute_tokens(s, d, prob)
        flags = 0
    scale = 1.0 / math.sqrt(wl.head_dim)
    o_ref = torch.empty_like(q)
    svga.svga_sparse_attention_fwd(qp, kp, vp, o_ref, None, prob, bmap, scale, flags)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0

    o = torch.zeros_like(q)
    t0 = time.monotonic()
    svga.svga_sparse_attention_fwd(qp, kp, vp, o, None, prob, bmap, scale,
                                   flags | svga.FLAG_TEST_STALL)
    torch.cuda.synchronize()
    waited = time.monotonic() - t0
    assert bmap.device_status() == 7          # SVGA_ERR_TIMEOUT
    assert 0.5 < waited < 30.0, waited
    assert not o.any()                        # no output row was stored

    # the context is intact: the next call runs normally and gives the same result
    o2 = torch.empty_like(q)
    svga.svga_sparse_attention_fwd(qp, kp, vp, o2, None, prob, bmap, scale, flags)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    assert torch.equal(o2, o_ref)
