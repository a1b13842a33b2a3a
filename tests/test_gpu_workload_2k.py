"""The 2K workload at full size against the fp64 oracle: 21 frames x 90x160 = 302,400
tokens, 10 heads, d = 128, structured inputs, with the masks the online classifier picks
for them (heads 0-4 spatial |df| <= 3, heads 5-9 temporal |ds| <= 2,400 in anchor-first
order, all with the frame-0 anchor).  Permute -> block-sparse attention -> unpermute on
the GPU; sampled rows (whole 128-row blocks, the ragged last block, spread rows) of two
spatial and two temporal heads are compared within the attention tolerance."""
import math

import numpy as np
import pytest
import torch

from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from tests.helpers import (assert_attn_close, lse_to_frame_major, oracle_rows,  # noqa: E402
                           run_sparse_path, sample_rows)


def test_2k_sparse_attention_sampled_rows():
    wl = C.twok()
    q, k, v = make_qkv(wl)
    o, lse, _ = run_sparse_path(wl, q.cuda(), k.cuda(), v.cuda())
    rows = sample_rows(wl, 128, seed=5)
    idx = torch.from_numpy(rows.astype(np.int64)).cuda()
    on = o.index_select(1, idx).float().cpu().numpy()
    lse_fm = lse_to_frame_major(lse.cpu().numpy(), wl, wl.order)
    for h in (0, 4, 5, 9):
        ro, rl = oracle_rows(wl, q, k, v, h, rows)
        assert_attn_close(on[h], ro, lse_fm[h, rows], rl, what=f"2k head {h}")
