"""Benchmark of the block-sparse spatio-temporal attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl svga|reference]
                    [--config headline|mid|tiny|permstudy|2k] [--tile 128x128]
                    [--order fm|tm|strict] [--split] [--mode full|attn|parts|classify]

One step = one pass of the hot path over the workload's Q/K/V already in HBM: K and V
permuted into each head's token order, then the block-sparse attention, which takes Q
frame-major (gathering the rows of temporal-major heads itself) and writes O
frame-major; the same step with Q permuted and O unpermuted by separate kernels is
timed beside it.  The block map depends on the problem only and is built once before
timing (its build time is reported separately), as it would be cached across layers and
denoising steps.  Metric: effective TFLOP/s on kept pairs, FLOP = sum over heads of
4 * kept_pairs * head_dim, and ms per step.  Under torchrun every rank runs the same
workload on its own GPU (weak scaling; value = FLOP of all ranks / max time over ranks),
or with --split the ranks share one problem (strong scaling).

--mode attn / classify only launch the attention kernel / the classifier (for ncu
captures); --mode parts times each part of a split problem alone.
--impl reference times the fp64 CPU oracle (the only reference this method has) on a
bounded sample of query rows per step, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_spatio_attn_b200 import configs as C  # noqa: E402
from block_sparse_spatio_attn_b200.inputs import make_qkv  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "sparse attn fwd ms + TFLOP/s on kept pairs (75.6K tok, 10 heads, d=128)"


# ------------------------------------------------------------------- accounting
def kept_pairs(type_: int, band: int, anchor: int, F: int, S: int) -> int:
    """Kept (q, k) pairs of one head (closed form of the spatial / temporal masks)."""
    if type_ == C.SPATIAL:
        tot = 0
        for fq in range(F):
            lo, hi = max(0, fq - band), min(F - 1, fq + band)
            tot += (hi - lo + 1) + (1 if (anchor and lo > 0) else 0)
        return S * S * tot
    c = sum(min(S - 1, s + band) - max(0, s - band) + 1 for s in range(S))
    return F * S * S + F * (F - 1) * c if anchor else F * F * c


def kept_keys_of_row(wl, h: int, t: int) -> int:
    """Kept keys of frame-major query token t of head h."""
    F, S = wl.frames, wl.tokens_per_frame
    f, s = divmod(t, S)
    w = wl.band[h]
    if wl.head_type[h] == C.SPATIAL:
        lo, hi = max(0, f - w), min(F - 1, f + w)
        return S * ((hi - lo + 1) + (1 if (wl.anchor_frame0 and lo > 0) else 0))
    c = min(S - 1, s + w) - max(0, s - w) + 1
    return S + (F - 1) * c if wl.anchor_frame0 else F * c


def kept_flops(wl) -> float:
    F, S, d = wl.frames, wl.tokens_per_frame, wl.head_dim
    return float(sum(4 * kept_pairs(t, w, wl.anchor_frame0, F, S) * d
                     for t, w in zip(wl.head_type, wl.band)))


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings (the job is as slow as its slowest rank);
    identity on a single process."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def weak_scaling_value(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """TFLOP/s of the whole job: every rank runs the full workload (weak scaling)."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def job_value(flops_per_problem: float, world: int, ms_per_step: float, split: bool) -> float:
    """TFLOP/s of the whole job: with `split` the ranks share one problem (strong
    scaling), otherwise every rank runs its own (weak scaling)."""
    return weak_scaling_value(flops_per_problem, 1 if split else world, ms_per_step)


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def code_digest(src_path: str) -> str:
    """sha256 of a C++/CUDA source with its // comments and blank lines removed, so that
    an edit of the comments alone keeps the digest."""
    lines = []
    for line in open(src_path, encoding="utf-8"):
        code = line.split("//", 1)[0].rstrip()
        if code:
            lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def traffic_from_profile(kernel_src: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if it
    was taken on the current kernel code (code_sha256 recorded in the summary)."""
    path = os.path.join(ROOT, "profiles", "attention_headline_ncu.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m_sha = re.search(r"code_sha256:\s*([0-9a-f]{64})", txt)
    m_b = re.search(r"dram_bytes_per_full_launch:\s*([0-9.eE+]+)", txt)
    if not (m_sha and m_b):
        return None
    return float(m_b.group(1)) if code_digest(kernel_src) == m_sha.group(1) else None


# ------------------------------------------------------------------ clock sampler
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self, gpu_index: int):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = []
        with open(self.f.name) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((int(parts[0]), float(parts[1]), float(parts[2]),
                                 float(parts[3]) if parts[3] not in ("[N/A]", "N/A") else 0.0,
                                 parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.f.name)
        idx = {r[0] for r in rows}
        gi = gpu_index if gpu_index in idx else (min(idx) if idx else None)
        rows = [r for r in rows if r[0] == gi]
        if not rows:
            return None
        load = [r for r in rows if r[3] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[4]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in load), "sm_max_mhz": rows[0][2],
                "reasons": reasons, "samples": len(load)}


# --------------------------------------------------------------------- svga arm
def run_svga(args, rank, world, local_rank):
    from block_sparse_spatio_attn_b200 import svga
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    split = bool(args.split) and world > 1
    part, n_parts = (rank, world) if split else (0, 1)
    wl = C.ALL[args.config]()
    if args.tile:
        tq, tk = (int(x) for x in args.tile.lower().split("x"))
        wl = wl.with_tile(tq, tk)
    if args.order:
        wl = wl.with_orders({"fm": C.ORDER_FRAME_MAJOR, "tm": C.ORDER_TEMPORAL_MAJOR,
                             "strict": C.ORDER_TEMPORAL_MAJOR_STRICT}[args.order])
    H, N, d = wl.heads, wl.tokens, wl.head_dim
    scale = 1.0 / math.sqrt(d)
    q, k, v = make_qkv(wl)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    stream = torch.cuda.current_stream(dev)
    classify = None
    if wl.classify_fraction > 0:
        # online head classification (routing: outside the timed step, timed on its own)
        n_rows = max(1, int(math.ceil(wl.tokens * wl.classify_fraction)))
        prob0 = svga.ProblemSpec.from_workload(wl)
        ws = torch.empty(svga.svga_classify_size(prob0, n_rows), dtype=torch.uint8, device=dev)
        types, mse = svga.svga_classify_heads(qd, kd, vd, prob0, wl.cand_spatial,
                                              wl.cand_temporal, None, n_rows, scale, ws)
        t0 = time.perf_counter()
        for _ in range(3):
            types, mse = svga.svga_classify_heads(qd, kd, vd, prob0, wl.cand_spatial,
                                                  wl.cand_temporal, None, n_rows, scale, ws)
        classify_ms = (time.perf_counter() - t0) / 3 * 1e3
        band = [wl.cand_spatial[h] if types[h] == C.SPATIAL else wl.cand_temporal[h]
                for h in range(H)]
        order = [C.ORDER_FRAME_MAJOR if t == C.SPATIAL else C.ORDER_TEMPORAL_MAJOR for t in types]
        wl = C.Workload(**{**wl.__dict__, "head_type": list(types), "band": band,
                           "order": order})
        classify = {"ms": classify_ms, "rows_per_head": n_rows, "types": list(types),
                    "mse": [[round(a, 9), round(b, 9)] for a, b in mse]}
        if args.mode != "classify":
            # band selection over a ladder around the classifier's candidates, under the
            # pages' kept budget (38.87 % of the pairs)
            cands = [(C.SPATIAL, 2), (C.SPATIAL, 3), (C.SPATIAL, 4),
                     (C.TEMPORAL, 1200), (C.TEMPORAL, 2400), (C.TEMPORAL, 4800)]
            ws_at = torch.empty(svga.svga_autotune_size(prob0, n_rows, len(cands)),
                                dtype=torch.uint8, device=dev)
            at = svga.svga_autotune_heads(qd, kd, vd, prob0, cands, 0.3887, None, n_rows, scale,
                                          ws_at)
            t0 = time.perf_counter()
            for _ in range(3):
                at = svga.svga_autotune_heads(qd, kd, vd, prob0, cands, 0.3887, None, n_rows,
                                              scale, ws_at)
            classify["band_selection"] = {
                "ms": (time.perf_counter() - t0) / 3 * 1e3, "candidates": cands,
                "max_kept_fraction": 0.3887,
                "kept_fractions": [round(svga.svga_kept_fraction(prob0, t, b), 5)
                                   for t, b in cands],
                "types": at[0], "bands": at[1]}
            del ws_at
        if args.mode == "classify":
            # profiling aid: the classifier alone (Q/K/V and its workspace on the device)
            for _ in range(args.steps):
                svga.svga_classify_heads(qd, kd, vd, prob0, wl.cand_spatial, wl.cand_temporal,
                                         None, n_rows, scale, ws)
            return {"study": "online head classification", "workload": wl.name, **classify}
    elif args.mode == "classify":
        raise SystemExit(f"{wl.name} has no classifier settings (use --config 2k)")
    prob = svga.ProblemSpec.from_workload(wl)

    # block map: built once (timed on its own)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    bmap = svga.build_block_map(prob)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(3):
        svga.svga_build_block_map(prob, bmap)
    ev1.record(stream)
    torch.cuda.synchronize()
    map_ms = ev0.elapsed_time(ev1) / 3
    nq, nk = -(-N // wl.tile_q), -(-N // wl.tile_k)
    cls = bmap.cls[: H * nq * nk].view(H, nq, nk).cpu()
    visited = int((cls != 0).sum())
    boundary = int((cls == 2).sum())
    visited_flops = 4.0 * wl.tile_q * wl.tile_k * d * visited
    kflops = kept_flops(wl)
    kept_frac = kflops / (4.0 * H * N * N * d)

    qp, kp, vp, op, o = (torch.empty_like(qd) for _ in range(5))

    kernel_flag = svga.FLAG_CTA_PAIR if args.cta_pair else 0
    # One step: K and V move to each head's token order; the attention kernel gathers
    # the Q rows from frame-major memory itself and writes O rows back frame-major.
    def step(attn_evs=None):
        svga.svga_permute_tokens(kd, kp, prob)
        svga.svga_permute_tokens(vd, vp, prob)
        if attn_evs is not None:
            attn_evs[0].record(stream)
        svga.svga_sparse_attention_fwd_part(qd, kp, vp, o, None, prob, bmap, scale,
                                            svga.FLAG_QO_FRAME_MAJOR | kernel_flag, part,
                                            n_parts)
        if attn_evs is not None:
            attn_evs[1].record(stream)

    def step_separate():  # the same step with all four token permutations as kernels
        svga.svga_permute_tokens(qd, qp, prob)
        svga.svga_permute_tokens(kd, kp, prob)
        svga.svga_permute_tokens(vd, vp, prob)
        svga.svga_sparse_attention_fwd(qp, kp, vp, op, None, prob, bmap, scale)
        svga.svga_unpermute_tokens(op, o, prob)

    launches_per_step = 4 if args.cta_pair else 3  # the pair kernel, then the rest
    if args.mode == "parts":
        # study of one problem split over P GPUs: each part timed alone on this GPU,
        # which is the whole of what one of P GPUs would run (no exchange between parts)
        step_separate()
        torch.cuda.synchronize()

        def med_ms(fn, n=max(3, args.steps)):
            for _ in range(2):
                fn()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(n)]
            for a_, b_ in evs:
                a_.record(stream)
                fn()
                b_.record(stream)
            torch.cuda.synchronize()
            return statistics.median(a_.elapsed_time(b_) for a_, b_ in evs)

        single = med_ms(lambda: svga.svga_sparse_attention_fwd(qp, kp, vp, op, None, prob, bmap,
                                                               scale))
        part_ms = [med_ms(lambda r=r: svga.svga_sparse_attention_fwd_part(
            qp, kp, vp, op, None, prob, bmap, scale, 0, r, args.parts))
            for r in range(args.parts)]
        if bmap.device_status() != 0:
            raise RuntimeError(f"device status {bmap.device_status()}")
        return {"study": "one problem in parts", "workload": wl.name, "parts": args.parts,
                "single_call_ms": single, "part_ms": part_ms, "max_part_ms": max(part_ms),
                "projected_speedup": single / max(part_ms),
                "balance": min(part_ms) / max(part_ms)}
    if args.mode == "attn":
        # profiling aid: the attention kernel alone, warm-up + steps launches, no report
        step_separate()
        for _ in range(args.warmup + args.steps):   # the launch the timed step makes
            svga.svga_sparse_attention_fwd(qd, kp, vp, o, None, prob, bmap, scale,
                                           svga.FLAG_QO_FRAME_MAJOR | kernel_flag)
        torch.cuda.synchronize()
        if bmap.device_status() != 0:
            raise RuntimeError(f"device status {bmap.device_status()}")
        return None
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if bmap.device_status() != 0:
        raise RuntimeError(f"device status {bmap.device_status()} after warm-up")

    sampler = ClockSampler()
    if rank == 0:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    attn_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(attn_evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop(local_rank) if rank == 0 else None
    elapsed = t0.elapsed_time(t1)
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in attn_evs)
    elapsed, attn_ms = max_over_ranks([elapsed, attn_ms], dev)
    ms_per_step = elapsed / args.steps
    if bmap.device_status() != 0:
        raise RuntimeError(f"device status {bmap.device_status()} in the timed region")

    # -------- extras on the same GPU (not part of `value`) ------------------------
    def time_it(fn, reps):
        for _ in range(2):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    reps = max(3, min(args.steps, 10))
    step_separate()   # Q in each head's order for the comparison launches below
    dense_ms = time_it(lambda: svga.svga_dense_attention_fwd(qd, kd, vd, op, None, scale), reps)
    naive_ms = time_it(lambda: svga.svga_sparse_attention_fwd(qp, kp, vp, op, None, prob, bmap,
                                                              scale, svga.FLAG_NAIVE_B1), reps)
    perm_ms = time_it(lambda: svga.svga_permute_tokens(qd, qp, prob), reps)

    # the step forms timed alternately (order rotated each round): same clocks.  The
    # all-frame-major form is one launch that also gathers the K and V rows itself.
    def step_all_fm():
        svga.svga_sparse_attention_fwd(qd, kd, vd, o, None, prob, bmap, scale,
                                       svga.FLAG_QO_FRAME_MAJOR | svga.FLAG_KV_FRAME_MAJOR)

    forms = [(step_separate, []), (step, []), (step_all_fm, [])]
    for rnd in range(4):
        for fn, acc in forms[rnd % 3:] + forms[:rnd % 3]:
            acc.append(time_it(fn, max(3, reps // 2)))
    step_sep_ms, step_ref_ms, step_fm_ms = (statistics.median(acc) for _, acc in forms)
    dense_flops = 4.0 * H * N * N * d
    # tile-aligned traversal (B3, opt-in): every pair of a visited tile is kept
    b3 = None
    if wl.tile_q >= 128:
        # timed alternately with the exact traversal (order swapped each round), so that
        # both see the same clocks under the power cap
        b2_t, b3_t = [], []
        for rnd in range(4):
            for fl in ((0, svga.FLAG_TILE_ALIGNED) if rnd % 2 == 0 else
                       (svga.FLAG_TILE_ALIGNED, 0)):
                t = time_it(lambda: svga.svga_sparse_attention_fwd(
                    qp, kp, vp, op, None, prob, bmap, scale, fl), max(3, reps // 2))
                (b3_t if fl else b2_t).append(t)
        b3_ms, b2_paired_ms = statistics.median(b3_t), statistics.median(b2_t)
        rq = torch.clamp(N - torch.arange(nq) * wl.tile_q, max=wl.tile_q).double()
        rk = torch.clamp(N - torch.arange(nk) * wl.tile_k, max=wl.tile_k).double()
        b3_pairs = float(((cls != 0).double() * (rq[:, None] * rk[None, :])).sum())
        b3 = {"ms": b3_ms, "exact_b2_ms_alternating": b2_paired_ms,
              "kept_fraction": b3_pairs / (H * N * N),
              "tflops_on_kept": 4.0 * d * b3_pairs / (b3_ms * 1e-3) / 1e12}

    # the other reading of B3, exact: frames laid out at a stride of whole tiles (the
    # problem's frame_pad), so that no tile holds two frames; timed alternately with the
    # unpadded exact traversal
    b3_padded = None
    if wl.tile_q >= 128 and (wl.tokens_per_frame % max(wl.tile_q, wl.tile_k)) != 0:
        fpad = max(wl.tile_q, wl.tile_k)
        prob_p = svga.ProblemSpec.from_workload(wl, frame_pad=fpad)
        bmap_p = svga.build_block_map(prob_p)
        NPr = prob_p.rows
        qpp, kpp, vpp, opp = (torch.empty(H, NPr, d, dtype=torch.bfloat16, device=dev)
                              for _ in range(4))
        for src, dst in ((qd, qpp), (kd, kpp), (vd, vpp)):
            svga.svga_permute_tokens(src, dst, prob_p)
        b2_t, bp_t = [], []
        for rnd in range(4):
            for padded in ((False, True) if rnd % 2 == 0 else (True, False)):
                if padded:
                    t = time_it(lambda: svga.svga_sparse_attention_fwd(
                        qpp, kpp, vpp, opp, None, prob_p, bmap_p, scale), max(3, reps // 2))
                else:
                    t = time_it(lambda: svga.svga_sparse_attention_fwd(
                        qp, kp, vp, op, None, prob, bmap, scale), max(3, reps // 2))
                (bp_t if padded else b2_t).append(t)
        if bmap_p.device_status() != 0:
            raise RuntimeError(f"device status {bmap_p.device_status()} (padded layout)")
        nqp, nkp = -(-NPr // wl.tile_q), -(-NPr // wl.tile_k)
        cls_p = bmap_p.cls[: H * nqp * nkp].view(H, nqp, nkp).cpu()
        b3_padded = {"ms": statistics.median(bp_t),
                     "exact_b2_ms_alternating": statistics.median(b2_t),
                     "frame_pad": fpad, "rows_per_head": NPr,
                     "visited_tiles": int((cls_p != 0).sum()),
                     "boundary_tiles": int((cls_p == 2).sum()),
                     "visited_tiles_unpadded": int((cls != 0).sum()),
                     "boundary_tiles_unpadded": int((cls == 2).sum())}
        del qpp, kpp, vpp, opp, bmap_p

    # -------- end to end through the public API, host buffers ---------------------
    # Pipelined as a serving loop would run it: step i's inputs are copied in on one
    # stream while step i-1 computes on another, and outputs go out on a third; two sets
    # of device buffers alternate.  Every step's 774 MB still cross PCIe inside the
    # timed region.
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.empty_like(q).pin_memory()
    sets = [(qd, kd, vd, qp, kp, vp, op, o), tuple(torch.empty_like(qd) for _ in range(8))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_done, comp_done, out_done = ([torch.cuda.Event(), torch.cuda.Event()] for _ in range(3))

    def layer(bs):  # the step on one buffer set
        bq, bk, bv, bqp, bkp, bvp, bop, bo = bs
        svga.svga_permute_tokens(bk, bkp, prob)
        svga.svga_permute_tokens(bv, bvp, prob)
        svga.svga_sparse_attention_fwd_part(bq, bkp, bvp, bo, None, prob, bmap, scale,
                                            svga.FLAG_QO_FRAME_MAJOR, part, n_parts)

    def e2e_run(n, t0=None, t1=None):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[b])     # set b's inputs are free again
                if i == 0 and t0 is not None:
                    t0.record(s_in)
                for dst, src in zip(sets[b][:3], (qh, kh, vh)):
                    dst.copy_(src, non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if i >= 2:
                stream.wait_event(out_done[b])        # set b's output has been read out
            layer(sets[b])
            comp_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[b])
                oh.copy_(sets[b][7], non_blocking=True)
                out_done[b].record(s_out)
        if t1 is not None:
            t1.record(s_out)

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(4, min(args.steps, 12))
    e2e_run(e2e_steps, a, b)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / e2e_steps
    if bmap.device_status() != 0:
        raise RuntimeError(f"device status {bmap.device_status()} in the e2e loop")
    e2e_ms, = max_over_ranks([e2e_ms], dev)

    peaks, peak_src = read_peaks()
    timed_s = elapsed / 1e3
    sustained = timed_s >= 2.0
    peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    launch_flops = visited_flops / n_parts   # split: about 1/n of the items per rank
    achieved = launch_flops / (attn_ms * 1e-3) / 1e12
    traffic = traffic_from_profile(os.path.join(ROOT, "block_sparse_spatio_attn_b200", "csrc",
                                                "attention.cu"))
    if traffic is not None and args.config != "headline":
        traffic = None
    out = {
        "metric": METRIC, "value": job_value(kflops, world, ms_per_step, split),
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "tokens": N, "heads": H, "head_dim": d,
                   "frames": wl.frames, "grid": f"{wl.grid_h}x{wl.grid_w}",
                   "head_types": "".join("ST"[t] for t in wl.head_type), "bands": wl.band,
                   "orders": wl.order, "tile": f"{wl.tile_q}x{wl.tile_k}",
                   "attention_kernel": "cta_pair" if args.cta_pair else "one_cta",
                   "parallelism": (f"parts{world}" if split else f"replicas{world}")
                   if world > 1 else "single",
                   "l2": "inputs larger than L2 (Q,K,V %.0f MB)" % (3 * H * N * d * 2 / 1e6),
                   "step": "permute K,V + sparse attention (Q rows gathered and O rows "
                           "written frame-major by the kernel)"},
        "attn_ms": attn_ms,
        "attn_tflops_kept": kflops / (attn_ms * 1e-3) / 1e12,
        "attn_tflops_visited": achieved,
        "kept_fraction": kept_frac, "visited_fraction": visited / (H * nq * nk),
        "boundary_fraction": boundary / (H * nq * nk),
        "dense_ms": dense_ms, "dense_tflops": dense_flops / (dense_ms * 1e-3) / 1e12,
        "sparse_over_dense": attn_ms / dense_ms, "target_ratio": kept_frac + 0.15,
        "naive_b1_ms": naive_ms, "tile_aligned_b3": b3, "tile_aligned_b3_padded": b3_padded,
        "step_with_separate_permutes": {"ms": step_sep_ms, "step_ms_same_conditions": step_ref_ms},
        "step_all_frame_major": {"ms": step_fm_ms, "step_ms_same_conditions": step_ref_ms,
                                 "launches": 1,
                                 "note": "K and V rows gathered by the kernel (opt-in flag)"},
        "permute_ms_per_tensor": perm_ms, "map_build_ms": map_ms,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} {'sustained' if sustained else 'burst'} bf16",
                     "kernel": "attn_fwd_kernel<128,128>", "flops_per_launch": launch_flops},
        "e2e": {"value": job_value(kflops, world, e2e_ms, split), "unit": "TFLOP/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": 3 * H * N * d * 2,
                "d2h_bytes_per_step": H * N * d * 2,
                "pipeline": "copy-in, compute and copy-out of successive steps overlap on "
                            "three streams, two device buffer sets"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if classify is not None:
        out["classify"] = classify
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, q, k, v, args.cpu_seconds)
    return out


# ------------------------------------------------------------------ oracle arm
def as_f32(q, k, v):
    """Per-head float32 copies for the oracle (bf16 values, exact), made before timing."""
    return [tuple(np.ascontiguousarray(x[h].float().numpy()) for x in (q, k, v))
            for h in range(q.shape[0])]


def oracle_sample(wl, qkv32, rows_per_head: int, seed: int):
    """Run the oracle on `rows_per_head` rows of every head; returns (seconds, kept FLOP)."""
    import oracle
    rng = np.random.default_rng(seed)
    N = wl.tokens
    rows = np.sort(rng.choice(N, size=rows_per_head, replace=False)).astype(np.int32)
    t = time.perf_counter()
    for h in range(wl.heads):
        qh, kh, vh = qkv32[h]
        oracle.attention_rows(qh, kh, vh, wl.frames, wl.tokens_per_frame,
                              1.0 / math.sqrt(wl.head_dim), wl.head_type[h], wl.band[h],
                              wl.anchor_frame0, rows)
    dt = time.perf_counter() - t
    flops = sum(4.0 * kept_keys_of_row(wl, h, int(r)) * wl.head_dim
                for h in range(wl.heads) for r in rows)
    return dt, flops


def calibrate_rows(wl, qkv32, seconds: float) -> int:
    oracle_sample(wl, qkv32, 4, 321)  # first call pays for thread start-up
    dt, _ = oracle_sample(wl, qkv32, 16, 123)
    return max(16, min(wl.tokens, int(16 * seconds / max(dt, 1e-3))))


def cpu_baseline(wl, q, k, v, seconds: float):
    import oracle
    qkv32 = as_f32(q, k, v)
    rows = calibrate_rows(wl, qkv32, seconds)
    dt, fl = oracle_sample(wl, qkv32, rows, 7)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{rows} query rows per head x {wl.heads} heads of {wl.name} "
                      f"(fp64 C + OpenMP), {dt:.1f} s"}


def run_reference(args, rank, world):
    import oracle
    if rank != 0:
        return None
    wl = C.ALL[args.config]()
    q, k, v = make_qkv(wl)
    qkv32 = as_f32(q, k, v)
    rows = calibrate_rows(wl, qkv32, args.ref_step_seconds)
    for i in range(args.warmup):
        oracle_sample(wl, qkv32, rows, 1000 + i)
    tot_t, tot_f = 0.0, 0.0
    for i in range(args.steps):
        dt, fl = oracle_sample(wl, qkv32, rows, i)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    sample = f"{rows} query rows per head x {wl.heads} heads per step of {wl.name}"
    return {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "tokens": wl.tokens, "heads": wl.heads,
                       "head_dim": wl.head_dim, "tile": f"{wl.tile_q}x{wl.tile_k}"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="svga", choices=["svga", "reference"])
    ap.add_argument("--config", default="headline", choices=sorted(C.ALL))
    ap.add_argument("--tile", default="", help="block-map tile, e.g. 64x64, 128x256")
    ap.add_argument("--order", default="", choices=["", "fm", "tm", "strict"],
                    help="token order of the temporal heads (default: the workload's)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--parts", type=int, default=8, help="number of parts for --mode parts")
    ap.add_argument("--split", action="store_true",
                    help="under torchrun, the ranks share one problem (each runs its part of "
                         "the work items) instead of running one problem each")
    ap.add_argument("--cta-pair", action="store_true",
                    help="run the work items on CTA pairs (SVGA_FLAG_CTA_PAIR)")
    ap.add_argument("--mode", default="full", choices=["full", "attn", "parts", "classify"],
                    help="attn: only launch the attention kernel (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    pg = world > 1 and args.impl == "svga"   # the oracle arm runs on rank 0 alone
    if pg:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.impl == "reference":
            out = run_reference(args, rank, world)
        else:
            out = run_svga(args, rank, world, local_rank)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if pg:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
