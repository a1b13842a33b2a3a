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
