"""Multi-process host logic of bench.py on CPU: two gloo ranks, the timing taken as the
maximum over ranks and the weak-scaling throughput built from it."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r is slower on the first timer, faster on the second
        local = [10.0 + rank, 5.0 - rank]
        got = bench.max_over_ranks(local, torch.device("cpu"))
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_gloo_two_ranks():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert out[0] == out[1] == [11.0, 5.0]


def test_weak_scaling_value_and_single_process_identity():
    import bench
    # 1e13 FLOP per rank, 2 ranks, 10 ms per step -> 2000 TFLOP/s for the job
    assert abs(bench.weak_scaling_value(1e13, 2, 10.0) - 2000.0) < 1e-9
    assert bench.max_over_ranks([3.0, 4.0], torch.device("cpu")) == [3.0, 4.0]


def test_job_value_weak_and_strong():
    import bench
    # replicas: every rank its own problem; split: the ranks share one problem
    assert abs(bench.job_value(1e13, 4, 10.0, split=False) - 4000.0) < 1e-9
    assert abs(bench.job_value(1e13, 4, 2.5, split=True) - 4000.0) < 1e-9
    assert bench.job_value(1e13, 1, 10.0, True) == bench.job_value(1e13, 1, 10.0, False)


def test_closed_form_kept_pairs_match_the_oracle():
    """bench.py's FLOP accounting (closed form per head and per row) equals the oracle's
    pair counts."""
    import numpy as np

    import bench
    import oracle
    from block_sparse_spatio_attn_b200 import configs as C
    wl = C.mid()
    F, S = wl.frames, wl.tokens_per_frame
    for t, w in [(0, 2), (1, 160)]:
        assert bench.kept_pairs(t, w, 1, F, S) == oracle.kept_count(t, w, 1, F, S)
    wl = C.tiny()
    m = [oracle.mask(t, w, 1, wl.frames, wl.tokens_per_frame)
         for t, w in zip(wl.head_type, wl.band)]
    for h in range(wl.heads):
        for r in (0, 7, 64, 100, 191):
            assert bench.kept_keys_of_row(wl, h, r) == int(m[h][r].sum())


# ------------------------------------------------ one problem split over two ranks
def plan_items_cpu(wl, with_lengths=False):
    """The attention plan's work items restated on the CPU from the oracle's tile classes:
    one item per (head, pair of 128-row query blocks), its length the number of key chunks
    either block visits, items sorted longest first (ties: lower head, then lower pair).
    Tiles of 128 x 128, so block b is q-tile b and chunk c is k-tile c."""
    import oracle
    assert wl.tile_q == wl.tile_k == 128
    N = wl.tokens
    n_qblk = -(-N // 128)
    n_pairs = -(-n_qblk // 2)
    items, cache = [], {}
    for h in range(wl.heads):
        key = (wl.head_type[h], wl.band[h], wl.order[h])
        if key not in cache:
            cache[key] = oracle.tile_map(*key[:2], wl.anchor_frame0, key[2], wl.frames,
                                         wl.tokens_per_frame, 128, 128)["cls"]
        cls = cache[key]
        for p in range(n_pairs):
            rows = cls[2 * p: min(n_qblk, 2 * p + 2)]
            items.append((int((rows != 0).any(axis=0).sum()), h * n_pairs + p, h, 2 * p))
    items.sort(key=lambda x: (-x[0], x[1]))
    if with_lengths:
        return [(h, b0, n) for n, _, h, b0 in items], n_qblk
    return [(h, b0) for _, _, h, b0 in items], n_qblk


def owned_blocks(items, n_qblk, part, num_parts):
    """(head, query block) pairs of `part`: the items are dealt in snake order, group g of
    num_parts consecutive items giving part r its r-th item when g is even and its
    (num_parts-1-r)-th when g is odd; an item holds blocks b0 and b0+1 (if it exists)."""
    out = []
    for g in range(-(-len(items) // num_parts)):
        i = g * num_parts + (num_parts - 1 - part if g % 2 else part)
        if i < len(items):
            h, b0 = items[i]
            out += [(h, b) for b in (b0, b0 + 1) if b < n_qblk]
    return out


def _split_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_spatio_attn_b200 import configs as C
        wl = C.mid()
        items, n_qblk = plan_items_cpu(wl)
        mine = owned_blocks(items, n_qblk, rank, world)
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        out[rank] = {"gathered": gathered, "n_qblk": n_qblk, "heads": wl.heads,
                     "lengths": [n for n in (len(x) for x in gathered)]}
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_split_rows_are_disjoint_and_cover_every_row_gloo_two_ranks():
    """Two gloo ranks each derive, from the plan restated on the CPU, the query blocks
    their part of one split problem writes; the parts are disjoint and together hold
    every (head, 128-row block) exactly once.  The rank-to-part rule is the one
    svga_sparse_attention_fwd_part documents (snake deal of the longest-first items)."""
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_split_worker, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert out[0]["gathered"] == out[1]["gathered"]
    parts = out[0]["gathered"]
    sets = [set(p) for p in parts]
    assert all(len(s) == len(p) for s, p in zip(sets, parts)), "a part holds a block twice"
    assert not (sets[0] & sets[1]), "two parts write the same rows"
    every = {(h, b) for h in range(out[0]["heads"]) for b in range(out[0]["n_qblk"])}
    assert sets[0] | sets[1] == every
    # the snake deal keeps the parts' work within one item of each other
    assert abs(len(parts[0]) - len(parts[1])) <= 2


def test_snake_deal_balances_work_on_the_headline_plan():
    """The same restatement at the headline size, 8 parts: every block owned once, and the
    parts' visited-chunk totals within one item of each other."""
    from block_sparse_spatio_attn_b200 import configs as C
    wl = C.headline()
    items, n_qblk = plan_items_cpu(wl, with_lengths=True)
    length = {(h, b0): n for h, b0, n in items}
    pairs = [(h, b0) for h, b0, _ in items]
    seen, work = [], []
    for r in range(8):
        mine = owned_blocks(pairs, n_qblk, r, 8)
        seen += mine
        work.append(sum(length[(h, b)] for h, b in mine if (h, b) in length))
    assert sorted(seen) == sorted((h, b) for h in range(wl.heads) for b in range(n_qblk))
    assert max(work) - min(work) <= max(n for _, _, n in items)
