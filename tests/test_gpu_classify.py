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


def check_autotune(wl, q, k, v, n_rows, cands, budget, heads=None):
    """GPU band selection against oracle.select_band on the same rows: every eligible
    candidate's deviation within 2e-2 relative, and the same choice unless the two best
    eligible deviations lie within 1e-2 of each other."""
    prob = svga.ProblemSpec.from_workload(wl)
    rows = default_sample_rows(wl.tokens, n_rows)
    scale = 1.0 / math.sqrt(wl.head_dim)
    types, bands, mse = svga.svga_autotune_heads(q.cuda(), k.cuda(), v.cuda(), prob, cands,
                                                 budget, None, n_rows, scale)
    F, S = wl.frames, wl.tokens_per_frame
    for h in (range(wl.heads) if heads is None else heads):
        best, mses, fracs = oracle.select_band(q[h].float().numpy(), k[h].float().numpy(),
                                               v[h].float().numpy(), F, S, scale, cands,
                                               wl.anchor_frame0, rows.numpy(), budget)
        for c, (g, m) in enumerate(zip(mse[h], mses)):
            assert abs(g - m) <= MSE_REL * m, (h, c, g, m)
        elig = sorted(m for m, f in zip(mses, fracs) if f <= budget)
        if len(elig) < 2 or elig[1] - elig[0] > TIE_REL * elig[1]:
            assert (types[h], bands[h]) == tuple(cands[best]), (h, types[h], bands[h], best)
    return types, bands


def test_autotune_small_against_oracle():
    wl = C.Workload("struct_small", 7, 6, 10, 64, [0, 0, 1, 1], [1, 1, 40, 40], [0] * 4,
                    seed=4, structured=True)
    q, k, v = make_qkv(wl)
    cands = [(0, 0), (0, 1), (0, 2), (1, 10), (1, 20), (1, 40)]
    types, bands = check_autotune(wl, q, k, v, 60, cands, 0.6)
    assert types == [0, 0, 1, 1]


def test_autotune_budget_excludes_wide_bands():
    """A budget that only the narrow candidates meet: no head takes a wider one."""
    wl = C.Workload("struct_small", 7, 6, 10, 64, [0, 0, 1, 1], [1, 1, 40, 40], [0] * 4,
                    seed=4, structured=True)
    q, k, v = make_qkv(wl)
    prob = svga.ProblemSpec.from_workload(wl)
    cands = [(0, 0), (0, 3), (1, 5), (1, 40)]
    fr = [svga.svga_kept_fraction(prob, t, b) for t, b in cands]
    budget = max(fr[0], fr[2]) + 1e-9
    assert fr[1] > budget and fr[3] > budget
    types, bands = check_autotune(wl, q, k, v, 60, cands, budget)
    assert all((t, b) in ((0, 0), (1, 5)) for t, b in zip(types, bands))
    with pytest.raises(svga.SvgaError):   # nothing eligible
        svga.svga_autotune_heads(q.cuda(), k.cuda(), v.cuda(), prob, cands, min(fr) / 2, None,
                                 60, 0.125)


def test_autotune_2k_structured():
    """2K structured inputs, bands around the classifier's candidates under the pages'
    kept budget (38.87 %): frame-local heads pick a spatial band, same-position heads a
    temporal one; heads 0 and 9 checked against the oracle on 48 rows."""
    wl = C.twok()
    q, k, v = make_qkv(wl)
    cands = [(0, 2), (0, 3), (0, 4), (1, 1200), (1, 2400), (1, 4800)]
    types, bands = check_autotune(wl, q, k, v, 48, cands, 0.3887, heads=(0, 9))
    assert types == [0] * 5 + [1] * 5
    assert all(b in (2, 3) for b in bands[:5]) and all(b in (1200, 2400) for b in bands[5:])

