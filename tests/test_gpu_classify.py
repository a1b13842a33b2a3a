"""Online head classification on the GPU (svga_classify_heads, through the C ABI) against
the fp64 oracle on the same sampled query rows.

The classifier's deviation values come from fp32 outputs of bf16 products, compared with
the oracle's fp64 values: each MSE within 2e-2 relative.  Types must agree unless the two
deviations are within 1e-2 of each other (relative), where both answers are correct."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200.inputs import default_sample_rows, make_qkv

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_spatio_attn_b200 import svga  # noqa: E402

MSE_REL = 2e-2
TIE_REL = 1e-2


def check(wl, q, k, v, n_rows, w_s, w_t, explicit_rows):
    prob = svga.ProblemSpec.from_workload(wl)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    rows = default_sample_rows(wl.tokens, n_rows)
    types, mse = svga.svga_classify_heads(qd, kd, vd, prob, w_s, w_t,
                                          rows.cuda() if explicit_rows else None, n_rows,
                                          1.0 / math.sqrt(wl.head_dim))
    F, S = wl.frames, wl.tokens_per_frame
    for h in range(wl.heads):
        t, ms, mt = oracle.classify(q[h].float().numpy(), k[h].float().numpy(),
                                    v[h].float().numpy(), F, S, 1.0 / math.sqrt(wl.head_dim),
                                    w_s[h], w_t[h], wl.anchor_frame0, rows.numpy())
        assert abs(mse[h][0] - ms) <= MSE_REL * ms, (h, mse[h][0], ms)
        assert abs(mse[h][1] - mt) <= MSE_REL * mt, (h, mse[h][1], mt)
        if abs(ms - mt) > TIE_REL * max(ms, mt):
            assert types[h] == t, (h, types[h], t, ms, mt)
    return types


def test_classify_structured_small():
    wl = C.Workload("struct_small", 7, 6, 10, 64, [0, 0, 1, 1], [1, 1, 40, 40], [0] * 4,
                    seed=4, structured=True)
    q, k, v = make_qkv(wl)
    types = check(wl, q, k, v, 60, [1] * 4, [10] * 4, explicit_rows=True)
    assert types == [0, 0, 1, 1]


def test_classify_mid_default_rule():
    """iid inputs (deviations nearly tie): the values are pinned, the library's own default
    row rule (rows = NULL) is checked against the same rule evaluated here."""
    wl = C.mid()
    q, k, v = make_qkv(wl)
    check(wl, q, k, v, -(-wl.tokens // 100), [2] * 4, [160] * 4, explicit_rows=False)


def test_classify_2k_structured_subset():
    """The 2K workload's structured inputs on 48 sampled rows per head, all 10 heads:
    frame-local heads come out spatial, same-position heads temporal."""
    wl = C.twok()
    q, k, v = make_qkv(wl)
    types = check(wl, q, k, v, 48, wl.cand_spatial, wl.cand_temporal, explicit_rows=False)
    assert types == [0] * 5 + [1] * 5


def test_classify_2k_one_percent():
    """The full 1% sample (3,024 rows per head) on the GPU: the expected 5/5 split."""
    wl = C.twok()
    q, k, v = make_qkv(wl)
    prob = svga.ProblemSpec.from_workload(wl)
    n = -(-wl.tokens // 100)
    types, mse = svga.svga_classify_heads(q.cuda(), k.cuda(), v.cuda(), prob, wl.cand_spatial,
                                          wl.cand_temporal, None, n, 1.0 / math.sqrt(128))
    assert types == [0] * 5 + [1] * 5
    assert all(m[0] > 0 and m[1] > 0 for m in mse)
