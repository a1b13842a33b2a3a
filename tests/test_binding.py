"""The Python binding checks what a pointer cannot tell the C ABI (dtype, shape,
contiguity, device) before anything reaches the library (CPU only: every call here is
rejected before a launch)."""
import pytest
import torch

from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200 import svga


@pytest.fixture(scope="module")
def prob():
    return svga.ProblemSpec.from_workload(C.tiny())


def qkvo(prob, **kw):
    shape = (prob.heads, prob.tokens, prob.head_dim)
    t = {n: torch.zeros(shape, dtype=torch.bfloat16) for n in "qkvo"}
    t.update(kw)
    return t


def attn(prob, lse=None, **kw):
    t = qkvo(prob, **kw)
    return svga.svga_sparse_attention_fwd(t["q"], t["k"], t["v"], t["o"], lse, prob, None, 0.1)


def rejected(fn, status, words):
    with pytest.raises(svga.SvgaError) as e:
        fn()
    assert e.value.status == status and words in str(e.value), str(e.value)


def test_attention_tensor_checks(prob):
    H, N, d = prob.heads, prob.tokens, prob.head_dim
    rejected(lambda: attn(prob, k=torch.zeros(H, N, d)), 1, "k must be torch.bfloat16")
    rejected(lambda: attn(prob, v=torch.zeros(H, N - 1, d, dtype=torch.bfloat16)), 2,
             "v has shape")
    rejected(lambda: attn(prob, o=torch.zeros(H, d, N, dtype=torch.bfloat16).transpose(1, 2)),
             1, "o must be contiguous")
    rejected(lambda: attn(prob, q=None), 1, "q is None")
    rejected(lambda: attn(prob, lse=torch.zeros(H, N, dtype=torch.float64)), 1,
             "lse must be torch.float32")
    rejected(lambda: attn(prob, lse=torch.zeros(H, N + 1)), 2, "lse has shape")
    rejected(lambda: attn(prob), 1, "q must be on a CUDA device")   # all else right


def test_permute_dense_classify_and_routed_checks(prob):
    H, N, d = prob.heads, prob.tokens, prob.head_dim
    x = torch.zeros(H, N, d, dtype=torch.bfloat16)
    rejected(lambda: svga.svga_permute_tokens(x, x[:, :, :32], prob), 2, "dst has shape")
    rejected(lambda: svga.svga_unpermute_tokens(x.float(), x, prob), 1, "src must be")
    rejected(lambda: svga.svga_permute_tokens_mapped(x, x, prob, None), 1, "CUDA device")
    rejected(lambda: svga.svga_dense_attention_fwd(x[0], x, x, x, None, 0.1), 2,
             "[heads, tokens, head_dim]")
    rejected(lambda: svga.svga_dense_attention_fwd(x, x, x[:1], x, None, 0.1), 2, "v has shape")
    rejected(lambda: svga.svga_dense_attention_fwd(x, x, x, x, None, 0.1,
                                                   status=torch.zeros(2, dtype=torch.int32)),
             2, "status has 2 elements")
    rows = torch.arange(4, dtype=torch.int64)
    rejected(lambda: svga.svga_classify_heads(x, x, x, prob, [1] * H, [1] * H, rows, 4, 0.1), 1,
             "rows must be torch.int32")
    rejected(lambda: svga.svga_classify_heads(x, x, x, prob, [1] * H, [1] * H,
                                              rows.to(torch.int32), 5, 0.1), 2,
             "rows has 4 elements")
    types = torch.zeros(H + 1, dtype=torch.int32)
    rejected(lambda: svga.svga_build_block_map_routed(prob, types, [1] * H, [1] * H, None), 2,
             "head_type_dev has")
    rejected(lambda: svga.svga_classify_heads_async(x, x, x, prob, [1] * H, [1] * H, None, 4,
                                                    0.1, types[:H],
                                                    mse_dev=torch.zeros(H, 3)), 2,
             "mse_dev has")
