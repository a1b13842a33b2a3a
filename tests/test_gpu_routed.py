"""Routed pipeline through the C ABI: online classification -> block map -> permutation
-> block-sparse attention -> inverse permutation with the head types kept on the device.

Checked against the same layer routed through the host (types returned by
svga_classify_heads, problem built from them): identical types, deviations, maps and
outputs bit for bit.  The whole routed layer is then captured once in a CUDA graph and
replayed on new inputs, equal to an eager run on those inputs.  The classifier itself is
checked against the oracle in test_gpu_classify.py, the attention in test_gpu_attention.py."""
import math

import numpy as np
import pytest
import torch

from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_spatio_attn_b200 import svga  # noqa: E402

W_S, W_T = 2, 160


def struct_mid(seed=7):
    """13 frames x 24x40 = 12,480 tokens, d = 128; heads 0-1 favour frame-local keys,
    heads 2-3 same-position keys (structured inputs), so the classifier has an answer."""
    return C.Workload("struct_mid", 13, 24, 40, 128, [0, 0, 1, 1], [W_S, W_S, W_T, W_T],
                      [0, 0, 1, 1], seed=seed, structured=True)


class Layer:
    """Buffers of one routed attention layer (all preallocated, graph-capturable)."""

    def __init__(self, wl):
        self.wl = wl
        H, N, d = wl.heads, wl.tokens, wl.head_dim
        self.prob = svga.ProblemSpec.from_workload(wl)
        self.n_rows = -(-N // 100)
        self.scale = 1.0 / math.sqrt(d)
        self.ws = [W_S] * H
        self.wt = [W_T] * H
        self.cws = torch.empty(svga.svga_classify_size(self.prob, self.n_rows), dtype=torch.uint8,
                               device="cuda")
        self.types = torch.empty(H, dtype=torch.int32, device="cuda")
        self.mse = torch.empty(H, 2, dtype=torch.float32, device="cuda")
        self.cstatus = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.bmap = svga.BlockMap(self.prob)
        mk = lambda: torch.empty(H, N, d, dtype=torch.bfloat16, device="cuda")  # noqa: E731
        self.q, self.k, self.v = mk(), mk(), mk()
        self.qp, self.kp, self.vp, self.op, self.o = mk(), mk(), mk(), mk(), mk()

    def run(self):
        p, m = self.prob, self.bmap
        svga.svga_classify_heads_async(self.q, self.k, self.v, p, self.ws, self.wt, None,
                                       self.n_rows, self.scale, self.types, self.mse,
                                       self.cstatus, self.cws)
        svga.svga_build_block_map_routed(p, self.types, self.ws, self.wt, m)
        for s, d in ((self.q, self.qp), (self.k, self.kp), (self.v, self.vp)):
            svga.svga_permute_tokens_mapped(s, d, p, m)
        svga.svga_sparse_attention_fwd(self.qp, self.kp, self.vp, self.op, None, p, m, self.scale)
        svga.svga_unpermute_tokens_mapped(self.op, self.o, p, m)


def host_routed(wl, q, k, v):
    """The same layer with the classifier's types brought to the host first."""
    H = wl.heads
    prob0 = svga.ProblemSpec.from_workload(wl)
    n_rows = -(-wl.tokens // 100)
    scale = 1.0 / math.sqrt(wl.head_dim)
    types, mse = svga.svga_classify_heads(q, k, v, prob0, [W_S] * H, [W_T] * H, None, n_rows,
                                          scale)
    wl2 = C.Workload(**{**wl.__dict__, "head_type": list(types),
                        "band": [W_S if t == 0 else W_T for t in types],
                        "order": [C.ORDER_FRAME_MAJOR if t == 0 else C.ORDER_TEMPORAL_MAJOR
                                  for t in types]})
    prob = svga.ProblemSpec.from_workload(wl2)
    bmap = svga.build_block_map(prob)
    qp, kp, vp, op, o = (torch.empty_like(q) for _ in range(5))
    for s, d in ((q, qp), (k, kp), (v, vp)):
        svga.svga_permute_tokens(s, d, prob)
    svga.svga_sparse_attention_fwd(qp, kp, vp, op, None, prob, bmap, scale)
    svga.svga_unpermute_tokens(op, o, prob)
    torch.cuda.synchronize()
    return types, mse, bmap, o


def csr(bmap, which):
    ptr = getattr(bmap, f"{which}_ptr")
    n = int(ptr[-1].item())
    return ptr.cpu(), getattr(bmap, f"{which}_idx")[:n].cpu()


def test_routed_layer_equals_host_routed_layer():
    wl = struct_mid()
    q, k, v = (x.cuda() for x in make_qkv(wl))
    types_h, mse_h, bmap_h, o_h = host_routed(wl, q, k, v)
    assert types_h == [0, 0, 1, 1]
    layer = Layer(wl)
    layer.q.copy_(q)
    layer.k.copy_(k)
    layer.v.copy_(v)
    layer.run()
    torch.cuda.synchronize()
    assert layer.cstatus.item() == 0 and layer.bmap.device_status() == 0
    assert layer.types.cpu().tolist() == types_h
    np.testing.assert_array_equal(layer.mse.cpu().numpy(), np.array(mse_h, np.float32))
    assert torch.equal(layer.bmap.cls, bmap_h.cls)
    for which in ("full", "bnd"):
        for a, b in zip(csr(layer.bmap, which), csr(bmap_h, which)):
            assert torch.equal(a, b)
    assert torch.equal(layer.o, o_h)


def test_routed_layer_replays_from_one_cuda_graph():
    wl = struct_mid()
    layer = Layer(wl)
    q1, k1, v1 = make_qkv(wl)
    q2, k2, v2 = make_qkv(struct_mid(seed=8))
    for dst, src in ((layer.q, q1), (layer.k, k1), (layer.v, v1)):
        dst.copy_(src)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer.run()                          # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer.run()
    for dst, src in ((layer.q, q2), (layer.k, k2), (layer.v, v2)):
        dst.copy_(src)
    graph.replay()
    torch.cuda.synchronize()
    o_graph, t_graph = layer.o.clone(), layer.types.clone()
    assert layer.cstatus.item() == 0 and layer.bmap.device_status() == 0
    layer.run()                              # eager, same inputs
    torch.cuda.synchronize()
    assert torch.equal(t_graph, layer.types)
    assert torch.equal(o_graph, layer.o)
    del graph


def test_routed_map_flags_an_invalid_device_type():
    wl = struct_mid()
    prob = svga.ProblemSpec.from_workload(wl)
    bmap = svga.BlockMap(prob)
    types = torch.tensor([0, 5, 1, 1], dtype=torch.int32, device="cuda")
    svga.svga_build_block_map_routed(prob, types, [W_S] * 4, [W_T] * 4, bmap)
    torch.cuda.synchronize()
    assert bmap.device_status() == 1
