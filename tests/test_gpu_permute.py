"""Token permutation kernels: bit-exact against the oracle's order maps, and exact inverses."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_spatio_attn_b200 import configs as C

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_spatio_attn_b200 import svga  # noqa: E402
from tests.helpers import problem_of  # noqa: E402


def rand_bf16(H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(H, N, d, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("wl,order", [
    (C.tiny(), [C.ORDER_TEMPORAL_MAJOR, C.ORDER_TEMPORAL_MAJOR_STRICT]),
    (C.mid(), None),
    (C.mid(), [C.ORDER_TEMPORAL_MAJOR_STRICT, C.ORDER_TEMPORAL_MAJOR, C.ORDER_FRAME_MAJOR,
               C.ORDER_TEMPORAL_MAJOR_STRICT]),
    (C.headline(), None),
], ids=["tiny", "mid", "mid-mixed", "headline"])
def test_permute_matches_oracle_and_inverts(wl, order):
    order = wl.order if order is None else order
    prob = problem_of(wl, order)
    x = rand_bf16(wl.heads, wl.tokens, wl.head_dim, 7)
    xd = x.cuda()
    y = torch.empty_like(xd)
    z = torch.empty_like(xd)
    svga.svga_permute_tokens(xd, y, prob)
    svga.svga_unpermute_tokens(y, z, prob)
    torch.cuda.synchronize()
    assert torch.equal(z, xd), "unpermute(permute(x)) != x"
    yc = y.cpu()
    for h in range(wl.heads):
        perm = torch.from_numpy(oracle.permutation(order[h], wl.frames, wl.tokens_per_frame))
        assert torch.equal(yc[h].view(torch.int16), x[h][perm].view(torch.int16)), f"head {h}"


def test_permute_rejects_overlap():
    wl = C.tiny()
    prob = problem_of(wl)
    x = torch.zeros(2 * wl.heads, wl.tokens, wl.head_dim, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(svga.SvgaError):
        svga.svga_permute_tokens(x[:2], x[1:3], prob)
