"""svga_build_block_map_static: the block-map build for callers that cannot allocate
device memory (no workspace argument; its scratch is a static device array inside the
library).  Called through the C ABI and checked against svga_build_block_map on two
calls in a row: block maps are integer data, so the outputs must match bit for bit.

This file sorts last so that a run stopping at the first failure has already run every
other test; it also passes on its own in a fresh process."""
import ctypes

import pytest
import torch

from block_sparse_spatio_attn_b200 import configs as C

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_spatio_attn_b200 import svga  # noqa: E402


def _zeroed_map(prob):
    m = svga.BlockMap(prob)
    for t in (m.cls, m.full_ptr, m.bnd_ptr, m.full_idx, m.bnd_idx, m.plan):
        t.zero_()
    return m


def _build_static(prob, bmap):
    lib = svga.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.svga_build_block_map_static(ctypes.byref(prob.c), ctypes.byref(bmap.c), stream)


def _same(a, b):
    torch.cuda.synchronize()
    for name in ("cls", "full_ptr", "bnd_ptr", "full_idx", "bnd_idx", "plan"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    assert a.device_status() == 0 and b.device_status() == 0


def test_static_scratch_build_matches_workspace_build_twice():
    cases = [svga.ProblemSpec.from_workload(C.mid()),
             svga.ProblemSpec.from_workload(C.headline())]
    for prob in cases:  # two calls in a row, different problems: no stale scratch state
        ref = _zeroed_map(prob)
        svga.svga_build_block_map(prob, ref)
        got = _zeroed_map(prob)
        assert _build_static(prob, got) == svga.SVGA_OK, svga.load().svga_last_error()
        _same(got, ref)
    # and the same problem again right after, on the same stream
    prob = cases[0]
    ref = _zeroed_map(prob)
    svga.svga_build_block_map(prob, ref)
    got = _zeroed_map(prob)
    assert _build_static(prob, got) == svga.SVGA_OK
    _same(got, ref)


def test_static_scratch_rejects_problems_beyond_its_size():
    wl = C.headline()
    big = svga.ProblemSpec(4096, wl.frames, wl.grid_h, wl.grid_w, wl.head_dim,
                           [0] * 4096, [3] * 4096, [0] * 4096)
    need = svga.svga_block_map_size(big)["workspace_bytes"]
    assert need > (1 << 20)
    m = svga.BlockMapC(1 << 12, 1 << 12, 1 << 12, 1 << 12, 1 << 12, 0, 0, 1 << 12, 1 << 30, None)
    lib = svga.load()
    rc = lib.svga_build_block_map_static(ctypes.byref(big.c), ctypes.byref(m), None)
    assert rc == 5  # SVGA_ERR_WORKSPACE, rejected on the host before any launch
    assert b"static" in lib.svga_last_error()
