"""The C-ABI library: loads without a GPU, exports every symbol the header declares, and
rejects bad arguments on the host before any launch (CPU only: no compute call)."""
import ctypes
import os
import re

import pytest

from block_sparse_spatio_attn_b200 import configs as C
from block_sparse_spatio_attn_b200 import svga

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "svga.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(svga_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_spatio_attn_b200 import build
    build.build()
    return svga.load()


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
    assert set(names) == set(svga.EXPORTED)


def test_version_and_status_strings(lib):
    assert svga.version() == 1
    assert svga.status_string(0) == "SVGA_OK"
    assert svga.status_string(7) == "SVGA_ERR_TIMEOUT"


def test_block_map_sizes_headline(lib):
    wl = C.headline()
    s = svga.svga_block_map_size(svga.ProblemSpec.from_workload(wl))
    nq = -(-75600 // 128)
    assert s["cls_bytes"] == 10 * nq * nq
    assert s["ptr_bytes"] == 4 * (10 * nq + 1)
    assert s["full_cap"] == s["bnd_cap"] == 10 * nq * nq
    n_items = 10 * ((nq + 1) // 2)
    hdr = (64 + 16 * (10 + n_items) + 255) // 256 * 256
    assert s["plan_bytes"] == hdr + 4 * n_items * nq


def _bad(lib, **kw):
    wl = C.tiny()
    d = dict(heads=wl.heads, num_frames=wl.frames, grid_h=wl.grid_h, grid_w=wl.grid_w,
             head_dim=wl.head_dim, head_type=wl.head_type, band=wl.band, order=wl.order,
             anchor_frame0=1, tile_q=64, tile_k=64)
    d.update(kw)
    return svga.ProblemSpec(**d)


@pytest.mark.parametrize("kw,status", [
    (dict(heads=0, head_type=[], band=[], order=[]), 2),
    (dict(head_dim=96), 4),
    (dict(tile_q=32), 4),
    (dict(tile_k=512), 4),
    (dict(band=[-1, 8]), 1),
    (dict(head_type=[0, 5]), 1),
    (dict(order=[0, 3]), 1),
    (dict(anchor_frame0=2), 1),
    (dict(num_frames=0), 2),
    (dict(grid_h=300, grid_w=300), 2),
    # 64 heads x 1,105,425 tokens: 4.8e9 tiles overflow the int32 list offsets
    (dict(heads=64, num_frames=17, grid_h=255, grid_w=255, head_type=[0] * 64,
          band=[1] * 64, order=[0] * 64, tile_q=128, tile_k=128), 2),
    # tile 256 in k: 1.1e9 tiles fit, but 2.4e9 plan entries (128-key chunks) do not
    (dict(heads=64, num_frames=17, grid_h=255, grid_w=255, head_type=[0] * 64,
          band=[1] * 64, order=[0] * 64, tile_q=256, tile_k=256), 2),
])
def test_problem_validation(lib, kw, status):
    with pytest.raises(svga.SvgaError) as e:
        svga.svga_block_map_size(_bad(lib, **kw))
    assert e.value.status == status


@pytest.mark.parametrize("kw,status", [
    (dict(frame_pad=-64), 1),
    (dict(frame_pad=32), 1),                              # not a multiple of the tiles
    (dict(frame_pad=64, tile_q=128), 1),                  # multiple of 64, not of 128
    (dict(frame_pad=65536 + 64), 1),
    # 4,096 tokens per frame at stride 65,536: 1,024 frames hold 2^26 positions
    (dict(frame_pad=65536, num_frames=1024, grid_h=64, grid_w=64), 2),
])
def test_frame_pad_validation(lib, kw, status):
    with pytest.raises(svga.SvgaError) as e:
        svga.svga_block_map_size(_bad(lib, **kw))
    assert e.value.status == status


def test_padded_rows_and_sizes(lib):
    """The padded layout's row count (frames x S rounded up to frame_pad) drives every
    tile count: headline spatial frames of 3,600 tokens at stride 3,712 (29 tiles of
    128)."""
    wl = C.headline()
    prob = svga.ProblemSpec.from_workload(wl, frame_pad=128)
    assert prob.rows == 21 * 3712 and prob.tokens == 75600
    assert svga.ProblemSpec.from_workload(wl).rows == 75600
    assert svga.ProblemSpec.from_workload(wl, frame_pad=256).rows == 21 * 3840
    s = svga.svga_block_map_size(prob)
    nq = 21 * 29
    assert s["cls_bytes"] == 10 * nq * nq
    n_items = 10 * ((nq + 1) // 2)
    hdr = (64 + 16 * (10 + n_items) + 255) // 256 * 256
    assert s["plan_bytes"] == hdr + 4 * n_items * nq


def test_padded_layout_flag_checks(lib):
    """The padded layout excludes the frame-major q / o and k / v forms and the snapped
    tile-aligned mask (its other reading): refused on the host."""
    P = ctypes.c_void_p
    m = svga.BlockMapC()
    m.plan, m.plan_bytes, m.status = 4096, 1 << 30, None   # never dereferenced here
    prob = svga.ProblemSpec.from_workload(C.mid(), frame_pad=128)
    for flags in (svga.FLAG_QO_FRAME_MAJOR, svga.FLAG_KV_FRAME_MAJOR, svga.FLAG_TILE_ALIGNED):
        rc = lib.svga_sparse_attention_fwd(P(4096), P(4096), P(4096), P(4096), None,
                                           ctypes.byref(prob.c), ctypes.byref(m),
                                           ctypes.c_float(0.1), flags, P(0))
        assert rc == 4 and b"frame_pad" in lib.svga_last_error(), flags
    rc = lib.svga_sparse_attention_fwd(P(4096), P(4096), P(4096), P(4096), None,
                                       ctypes.byref(prob.c), ctypes.byref(m),
                                       ctypes.c_float(-1.0), svga.FLAG_NAIVE_B1, P(0))
    assert rc == 1 and b"scale" in lib.svga_last_error()   # accepted up to the last check


def test_pointer_validation_before_launch(lib):
    prob = _bad(lib)
    P = ctypes.c_void_p
    st = P(0)
    # NULL and misaligned tensors are rejected on the host, before any CUDA call
    rc = lib.svga_permute_tokens(None, P(4096), ctypes.byref(prob.c), st)
    assert rc == 1
    rc = lib.svga_permute_tokens(P(4096 + 8), P(1 << 20), ctypes.byref(prob.c), st)
    assert rc == 3
    rc = lib.svga_permute_tokens(P(4096), P(4096 + 256), ctypes.byref(prob.c), st)
    assert rc == 1 and b"overlap" in lib.svga_last_error()
    rc = lib.svga_dense_attention_fwd(P(4096), P(4096), P(4096), P(4096), None, 2, 192, 80,
                                      ctypes.c_float(0.1), None, st)
    assert rc == 4
    rc = lib.svga_dense_attention_fwd(P(4096), P(4096), P(4096), P(4096), None, 2, 192, 64,
                                      ctypes.c_float(-1.0), None, st)
    assert rc == 1
    m = svga.BlockMapC()
    rc = lib.svga_sparse_attention_fwd(P(4096), P(4096), P(4096), P(4096), None,
                                       ctypes.byref(prob.c), ctypes.byref(m),
                                       ctypes.c_float(0.1), 0, st)
    assert rc == 1
    rc = lib.svga_build_block_map(ctypes.byref(prob.c), ctypes.byref(m), None, 0, st)
    assert rc == 1


def test_classify_size_validation(lib):
    prob = svga.ProblemSpec.from_workload(C.tiny())
    assert svga.svga_classify_size(prob, 2) > 0
    with pytest.raises(svga.SvgaError):
        svga.svga_classify_size(prob, 0)
    with pytest.raises(svga.SvgaError):
        svga.svga_classify_size(prob, 193)


def test_sparse_forward_flag_and_part_checks_on_the_host(lib):
    """Every flag combination is checked on the host before any CUDA call: unknown bits
    and NAIVE with TILE_ALIGNED are rejected, TILE_ALIGNED needs tile_q >= 128, and the
    accepted combinations (the frame-major ones included) get as far as the last host
    check, the scale."""
    P = ctypes.c_void_p
    m = svga.BlockMapC()
    m.plan, m.plan_bytes, m.status = 4096, 1 << 30, None   # never dereferenced here

    def call(flags, scale=0.1, part=0, n=1, wl=C.mid()):
        prob = svga.ProblemSpec.from_workload(wl)
        return lib.svga_sparse_attention_fwd_part(
            P(4096), P(4096), P(4096), P(4096), None, ctypes.byref(prob.c), ctypes.byref(m),
            ctypes.c_float(scale), flags, part, n, P(0))

    assert call(1 << 8) == 1 and b"unknown flags" in lib.svga_last_error()
    assert call(svga.FLAG_NAIVE_B1 | svga.FLAG_TILE_ALIGNED) == 1
    assert b"exclude" in lib.svga_last_error()
    assert call(svga.FLAG_TILE_ALIGNED, wl=C.mid().with_tile(64, 64)) == 4
    fm = svga.FLAG_QO_FRAME_MAJOR | svga.FLAG_KV_FRAME_MAJOR
    for flags in (0, svga.FLAG_NAIVE_B1, svga.FLAG_TILE_ALIGNED, svga.FLAG_QO_FRAME_MAJOR,
                  svga.FLAG_KV_FRAME_MAJOR, fm, fm | svga.FLAG_NAIVE_B1,
                  fm | svga.FLAG_TILE_ALIGNED, fm | svga.FLAG_TEST_STALL, svga.FLAG_CTA_PAIR,
                  svga.FLAG_CTA_PAIR | svga.FLAG_QO_FRAME_MAJOR | svga.FLAG_NAIVE_B1,
                  svga.FLAG_CTA_PAIR | svga.FLAG_TEST_STALL):
        assert call(flags, scale=-1.0) == 1, flags
        assert b"scale" in lib.svga_last_error(), flags
    assert call(0, part=2, n=2) == 1 and b"part" in lib.svga_last_error()
    assert call(0, part=0, n=5000) == 1


C_PROGRAM = r"""
#include <stdio.h>
#include "svga.h"
int main(void)
{
    int type[2] = {SVGA_HEAD_SPATIAL, SVGA_HEAD_TEMPORAL}, band[2] = {1, 8};
    int order[2] = {SVGA_ORDER_FRAME_MAJOR, SVGA_ORDER_TEMPORAL_MAJOR};
    svga_problem p = {2, 3, 8, 8, 64, type, band, order, 1, 64, 64, 0};
    size_t cls = 0, ptr = 0, plan = 0, ws = 0;
    int64_t fcap = 0, bcap = 0, rows = 0, rows_pad = 0;
    svga_status rc = svga_block_map_size(&p, &cls, &ptr, &fcap, &bcap, &plan, &ws);
    svga_status rr = svga_problem_rows(&p, &rows);
    p.frame_pad = 128;
    rr = rr == SVGA_OK ? svga_problem_rows(&p, &rows_pad) : rr;
    p.frame_pad = 0;
    p.head_dim = 96;
    svga_status bad = svga_block_map_size(&p, &cls, &ptr, &fcap, &bcap, &plan, &ws);
    printf("%d %d %zu %zu %lld %lld %lld %s %s\n", svga_version(), (int)rc, cls, ptr,
           (long long)fcap, (long long)rows, (long long)rows_pad, svga_status_string(bad),
           svga_last_error());
    return rc == SVGA_OK && rr == SVGA_OK && bad == SVGA_ERR_UNSUPPORTED ? 0 : 1;
}
"""


def test_header_is_plain_c_and_the_library_links_from_c(lib, tmp_path):
    """A C99 program includes include/svga.h (pedantic, no warnings), links libsvga.so
    and calls host-side entry points: the ABI needs no C++ and no Python."""
    import subprocess
    src = tmp_path / "use_svga.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_svga"
    libdir = os.path.join(ROOT, "block_sparse_spatio_attn_b200")
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L", libdir, "-lsvga", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    ver, rc, cls, ptr, fcap, rows, rows_pad, bad = r.stdout.split()[:8]
    assert int(ver) == lib.svga_version() and int(rc) == 0
    assert (int(cls), int(ptr), int(fcap)) == (2 * 3 * 3, 4 * (2 * 3 + 1), 2 * 3 * 3)
    assert (int(rows), int(rows_pad)) == (3 * 64, 3 * 128)   # frames of 64 at stride 128
    assert bad == "SVGA_ERR_UNSUPPORTED" and "head_dim 96" in r.stdout


def test_undersized_plan_is_rejected_on_the_host(lib):
    """A plan smaller than svga_block_map_size's plan_bytes (the worst case) is refused
    before any launch by every call that builds or reads a map: a build into it would
    have to drop entries its items still count, and a kernel reading it would run past
    its end.  With the full size the same calls get past the map checks."""
    P = ctypes.c_void_p
    prob = svga.ProblemSpec.from_workload(C.mid())
    s = svga.svga_block_map_size(prob)
    fake = 1 << 20   # aligned, never dereferenced: every call below stops on the host

    def bmap(plan_bytes):
        return svga.BlockMapC(fake, fake, fake, fake, fake, s["full_cap"], s["bnd_cap"], fake,
                              plan_bytes, None)

    small = bmap(s["plan_bytes"] - 4)
    st = P(0)
    assert lib.svga_build_block_map(ctypes.byref(prob.c), ctypes.byref(small), P(fake),
                                    s["workspace_bytes"], st) == 5
    assert b"plan" in lib.svga_last_error()
    assert lib.svga_build_block_map_static(ctypes.byref(prob.c), ctypes.byref(small), st) == 5
    wsp = (ctypes.c_int32 * prob.heads)(*([2] * prob.heads))
    assert lib.svga_build_block_map_routed(ctypes.byref(prob.c), P(fake), wsp, wsp,
                                           ctypes.byref(small), P(fake), s["workspace_bytes"],
                                           st) == 5
    assert lib.svga_sparse_attention_fwd(P(fake), P(fake), P(fake), P(fake), None,
                                         ctypes.byref(prob.c), ctypes.byref(small),
                                         ctypes.c_float(0.1), 0, st) == 1
    assert b"smaller than svga_block_map_size" in lib.svga_last_error()
    assert lib.svga_permute_tokens_mapped(P(fake), P(1 << 32), ctypes.byref(prob.c),
                                          ctypes.byref(small), st) == 1
    assert lib.svga_unpermute_tokens_mapped(P(fake), P(1 << 32), ctypes.byref(prob.c),
                                            ctypes.byref(small), st) == 1
    # a misaligned plan is refused too
    mis = svga.BlockMapC(fake, fake, fake, fake, fake, 0, 0, fake + 16, s["plan_bytes"], None)
    assert lib.svga_sparse_attention_fwd(P(fake), P(fake), P(fake), P(fake), None,
                                         ctypes.byref(prob.c), ctypes.byref(mis),
                                         ctypes.c_float(0.1), 0, st) == 3
    # the full size passes the map checks and stops at the next host check (the scale)
    full = bmap(s["plan_bytes"])
    assert lib.svga_sparse_attention_fwd(P(fake), P(fake), P(fake), P(fake), None,
                                         ctypes.byref(prob.c), ctypes.byref(full),
                                         ctypes.c_float(-1.0), 0, st) == 1
    assert b"scale" in lib.svga_last_error()
