"""Block map on the GPU against the oracle: classes and CSR lists bit-exact; the plan
is a faithful longest-first re-packing of the lists."""
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
from tests.test_oracle_tile_counts import HEADLINE, TWOK  # noqa: E402


def oracle_flat_map(wl, order, tq, tk, heads=None):
    """Oracle maps of the selected heads, concatenated into one flat CSR."""
    F, S = wl.frames, wl.tokens_per_frame
    heads = range(wl.heads) if heads is None else heads
    cls, fptr, fidx, bptr, bidx = [], [0], [], [0], []
    for h in heads:
        m = oracle.tile_map(wl.head_type[h], wl.band[h], wl.anchor_frame0, order[h], F, S, tq, tk)
        cls.append(m["cls"])
        fptr.extend((m["full_ptr"][1:] + fptr[-1]).tolist())
        bptr.extend((m["bnd_ptr"][1:] + bptr[-1]).tolist())
        fidx.append(m["full_idx"])
        bidx.append(m["bnd_idx"])
    return (np.stack(cls), np.array(fptr, np.int32), np.concatenate(fidx),
            np.array(bptr, np.int32), np.concatenate(bidx))


def gpu_map(wl, order, tq, tk):
    prob = problem_of(wl, order, tq, tk)
    bmap = svga.build_block_map(prob)
    torch.cuda.synchronize()
    assert bmap.device_status() == 0
    N = wl.tokens
    nq, nk = -(-N // tq), -(-N // tk)
    cls = bmap.cls[: wl.heads * nq * nk].cpu().numpy().reshape(wl.heads, nq, nk)
    fptr = bmap.full_ptr.cpu().numpy()
    bptr = bmap.bnd_ptr.cpu().numpy()
    fidx = bmap.full_idx[: fptr[-1]].cpu().numpy()
    bidx = bmap.bnd_idx[: bptr[-1]].cpu().numpy()
    return bmap, cls, fptr, fidx, bptr, bidx


CASES = [
    (C.tiny(), None, 64, 64),
    (C.tiny(), [C.ORDER_TEMPORAL_MAJOR] * 2, 64, 64),
    (C.tiny(), [C.ORDER_TEMPORAL_MAJOR_STRICT] * 2, 128, 64),
    (C.mid(), None, 128, 128),
    (C.mid(), None, 64, 64),
    (C.mid(), None, 256, 128),
    (C.mid(), None, 128, 256),
    (C.mid(), [C.ORDER_FRAME_MAJOR] * 4, 256, 256),
    (C.mid(), [C.ORDER_TEMPORAL_MAJOR_STRICT] * 4, 64, 128),
]


@pytest.mark.parametrize("wl,order,tq,tk", CASES,
                         ids=[f"{w.name}-{o}-{a}x{b}" for w, o, a, b in CASES])
def test_map_bit_exact(wl, order, tq, tk):
    order = wl.order if order is None else order
    _, cls, fptr, fidx, bptr, bidx = gpu_map(wl, order, tq, tk)
    rc, rfp, rfi, rbp, rbi = oracle_flat_map(wl, order, tq, tk)
    np.testing.assert_array_equal(cls, rc)
    np.testing.assert_array_equal(fptr, rfp)
    np.testing.assert_array_equal(fidx, rfi)
    np.testing.assert_array_equal(bptr, rbp)
    np.testing.assert_array_equal(bidx, rbi)


@pytest.mark.parametrize("order,heads", [(None, [0, 5]),
                                         ([C.ORDER_FRAME_MAJOR] * 10, [5]),
                                         ([C.ORDER_TEMPORAL_MAJOR_STRICT] * 10, [5])])
def test_map_bit_exact_headline(order, heads):
    wl = C.headline()
    order = wl.order if order is None else order
    _, cls, fptr, fidx, bptr, bidx = gpu_map(wl, order, 128, 128)
    nq = cls.shape[1]
    for h in heads:
        m = oracle.tile_map(wl.head_type[h], wl.band[h], 1, order[h], wl.frames,
                            wl.tokens_per_frame, 128, 128)
        np.testing.assert_array_equal(cls[h], m["cls"])
        r0 = h * nq
        np.testing.assert_array_equal(fptr[r0:r0 + nq + 1] - fptr[r0], m["full_ptr"])
        np.testing.assert_array_equal(fidx[fptr[r0]:fptr[r0 + nq]], m["full_idx"])
        np.testing.assert_array_equal(bidx[bptr[r0]:bptr[r0 + nq]], m["bnd_idx"])


def decode_plan(bmap, wl, tq, tk):
    plan = bmap.plan.cpu().numpy()
    hdr = plan[:64].view(np.int32)
    assert hdr[0] == 0x53564741
    heads, N = hdr[1], hdr[2]
    kn, n_qblk, n_kc, n_items = hdr[8], hdr[9], hdr[10], hdr[11]
    info = plan[64:64 + 16 * heads].view(np.int32).reshape(heads, 4)
    items = plan[64 + 16 * heads:64 + 16 * (heads + n_items)].view(np.int32).reshape(n_items, 4)
    off = (64 + 16 * (heads + n_items) + 255) // 256 * 256
    ents = plan[off:].view(np.uint32)
    return dict(heads=heads, N=N, kn=kn, n_qblk=n_qblk, n_kc=n_kc, items=items, info=info,
                entries=ents)


@pytest.mark.parametrize("wl,tq,tk", [(C.mid(), 128, 128), (C.mid(), 64, 64),
                                      (C.mid(), 256, 256), (C.tiny(), 64, 64)],
                         ids=["mid128", "mid64", "mid256", "tiny64"])
def test_plan_repacks_the_lists(wl, tq, tk):
    bmap, cls, *_ = gpu_map(wl, wl.order, tq, tk)
    P = decode_plan(bmap, wl, tq, tk)
    kn = min(tk, 128)
    assert P["kn"] == kn
    np.testing.assert_array_equal(P["info"][:, 0], wl.head_type)
    np.testing.assert_array_equal(P["info"][:, 1], wl.band)
    np.testing.assert_array_equal(P["info"][:, 2], wl.order)
    items = P["items"]
    n_pairs = (P["n_qblk"] + 1) // 2
    # every (head, block pair) exactly once, longest first
    assert sorted((int(h), int(b)) for h, b in items[:, :2]) == \
        [(h, 2 * p) for h in range(wl.heads) for p in range(n_pairs)]
    assert (np.diff(items[:, 3]) <= 0).all()
    nq = cls.shape[1]

    def block_flags(h, b, c):
        if b >= P["n_qblk"]:
            return 0
        qt = {64: [2 * b, min(2 * b + 1, nq - 1)], 128: [b], 256: [b // 2]}[tq]
        j = c // (tk // kn)
        xs = [cls[h, i, j] for i in qt]
        if all(x == 0 for x in xs):
            return 0
        return 1 | (2 if all(x == 1 for x in xs) else 0)

    for h, b0, off, cnt in items:
        ents = P["entries"][off:off + cnt]
        expect = []
        for c in range(P["n_kc"]):
            a, b = block_flags(h, b0, c), block_flags(h, b0 + 1, c)
            if a | b:
                expect.append(c | (a << 24) | (b << 26))
        np.testing.assert_array_equal(ents, np.array(expect, np.uint32))


# ------------------------------------------------- host-side map validator
@pytest.mark.parametrize("wl,order,tq,tk", [
    (C.tiny(), None, 64, 64),
    (C.mid(), None, 128, 128),
    (C.mid(), [C.ORDER_TEMPORAL_MAJOR_STRICT] * 4, 64, 256),
    (C.mid(), [C.ORDER_FRAME_MAJOR] * 4, 256, 64),
    (C.headline(), None, 128, 128),
], ids=["tiny", "mid", "mid-strict-64x256", "mid-fm-256x64", "headline"])
def test_validator_accepts_built_maps(wl, order, tq, tk):
    prob = problem_of(wl, order, tq, tk)
    bmap = svga.build_block_map(prob)
    svga.svga_validate_block_map(prob, bmap)


def _corrupted(what):
    wl = C.mid()
    prob = problem_of(wl, None, 128, 128)
    bmap = svga.build_block_map(prob)
    torch.cuda.synchronize()
    if what == "class":           # a full tile turned boundary: lists no longer agree
        k = int(torch.nonzero(bmap.cls == 1)[0].item())
        bmap.cls[k] = 2
    elif what == "order":         # two entries of a full list swapped
        r = int(torch.nonzero(bmap.full_ptr[1:] - bmap.full_ptr[:-1] >= 2)[0].item())
        a = int(bmap.full_ptr[r].item())
        x, y = bmap.full_idx[a].item(), bmap.full_idx[a + 1].item()
        bmap.full_idx[a], bmap.full_idx[a + 1] = y, x
    elif what == "offset":        # a CSR offset decreasing
        bmap.bnd_ptr[5] = bmap.bnd_ptr[4] - 1
    elif what == "plan_flag":     # the full flag of a plan entry flipped
        head = bmap.plan[:64].cpu().numpy().view(np.int32)
        hdr = (64 + 16 * (int(head[1]) + int(head[11])) + 255) // 256 * 256
        ent = bmap.plan[hdr:hdr + 4].view(torch.int32)
        ent ^= 1 << 25
    elif what == "status":
        bmap.status.fill_(3)
    torch.cuda.synchronize()
    return prob, bmap


@pytest.mark.parametrize("what,msg", [("class", "list"), ("order", "ascending"),
                                      ("offset", "decrease"), ("plan_flag", "plan entry"),
                                      ("status", "status word")])
def test_validator_rejects_corrupted_maps(what, msg):
    prob, bmap = _corrupted(what)
    with pytest.raises(svga.SvgaError) as e:
        svga.svga_validate_block_map(prob, bmap)
    assert e.value.status == 1 and msg in str(e.value), str(e.value)


def _pinned(rows, name):
    """(full, boundary, empty) of the named row of an independent tile-count table."""
    return tuple(next(c[7:10] for c in rows if c[0] == name))


@pytest.mark.parametrize("name", ["headline", "2k"])
def test_map_counts_equal_the_independent_integers(name):
    """The GPU map of the whole workload (tile 128x128) has, head by head, the (full,
    boundary, empty) tile counts that were computed independently of this library and
    that the oracle reproduces (tests/test_oracle_tile_counts.py): spatial heads
    frame-major, temporal heads in the anchor-first temporal-major order."""
    if name == "headline":
        rows, sp, tp = HEADLINE, "headline spatial FM 128", "headline temporal anchor-first 128"
    else:
        rows, sp, tp = TWOK, "2k spatial FM 128", "2k temporal anchor-first 128"
    expect = {C.SPATIAL: _pinned(rows, sp), C.TEMPORAL: _pinned(rows, tp)}
    wl = C.ALL[name]()
    _, cls, *_ = gpu_map(wl, None, 128, 128)
    for h in range(wl.heads):
        got = tuple(int((cls[h] == c).sum()) for c in (1, 2, 0))
        assert got == expect[wl.head_type[h]], (name, h, got)
