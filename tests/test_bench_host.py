"""Host logic of bench.py that needs no GPU: the digest that decides whether the
committed ncu traffic figure still describes the kernel source."""


def test_code_digest_ignores_comments_and_blank_lines(tmp_path):
    import bench
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text("int f(int x)  // doubles\n{\n    return 2 * x;\n}\n")
    b.write_text("// a new header comment\n\nint f(int x)\n{\n\n    return 2 * x;  // same\n}\n")
    c.write_text("int f(int x)\n{\n    return 3 * x;\n}\n")
    assert bench.code_digest(str(a)) == bench.code_digest(str(b))
    assert bench.code_digest(str(a)) != bench.code_digest(str(c))


def test_traffic_needs_a_matching_digest(tmp_path, monkeypatch):
    import bench
    src = tmp_path / "k.cu"
    src.write_text("__global__ void k() {}\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    summary = prof / "attention_headline_ncu.md"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    summary.write_text(f"code_sha256: {bench.code_digest(str(src))}\n"
                       "dram_bytes_per_full_launch: 3.5e9\n")
    assert bench.traffic_from_profile(str(src)) == 3.5e9
    src.write_text("__global__ void k() { int x = 1; (void)x; }\n")
    assert bench.traffic_from_profile(str(src)) is None


def test_flop_accounting_matches_the_mask_on_random_problems():
    """bench.py's kept-pair and per-row kept-key counts (closed forms, the metric's FLOP)
    against the mask written out with numpy, on random small problems."""
    import numpy as np

    import bench
    from block_sparse_spatio_attn_b200 import configs as C
    rng = np.random.default_rng(7)
    for _ in range(200):
        F, S = int(rng.integers(1, 8)), int(rng.integers(1, 30))
        t = int(rng.integers(0, 2))
        w, a = int(rng.integers(0, 10)), int(rng.integers(0, 2))
        tok = np.arange(F * S)
        f, s = tok // S, tok % S
        near = (np.abs(f[:, None] - f[None, :]) if t == C.SPATIAL
                else np.abs(s[:, None] - s[None, :])) <= w
        m = near | (bool(a) & (f[None, :] == 0))
        assert bench.kept_pairs(t, w, a, F, S) == int(m.sum())
        wl = C.Workload("r", F, 1, S, 64, [t], [w], [0], seed=0, anchor_frame0=a)
        for r in rng.choice(F * S, size=min(5, F * S), replace=False):
            assert bench.kept_keys_of_row(wl, 0, int(r)) == int(m[r].sum())


def test_reference_arm_rank_contract():
    """bench.py --impl reference: rank 0 prints one JSON line with the oracle's figures,
    any other rank exits 0 without work or output (the torchrun launch)."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config",
           "tiny", "--steps", "1", "--warmup", "3", "--ref-step-seconds", "0.2"]
    outs = {}
    for rank in (0, 1):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1")
        r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=300, cwd=root)
        assert r.returncode == 0, r.stderr[-2000:]
        outs[rank] = [l for l in r.stdout.splitlines() if l.strip()]
    assert outs[1] == []
    assert len(outs[0]) == 1
    line = json.loads(outs[0][0])
    assert line["impl"] == "reference" and line["value"] > 0 and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["gpu_launches"] == 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
