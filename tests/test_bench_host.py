"""Host-side pieces of the benchmark (CPU): the algorithmic work counts that
the roofline divides by, and the CPU reference arm's JSON line."""
import json
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_lsa_work_counts_every_visible_bucket_once():
    """scores = sum over queries of the buckets of the cluster blocks before
    the query's own (brute force over positions)."""
    import bench
    from workloads import LSA_WORKLOADS
    wl = LSA_WORKLOADS["lsa_t8k"].with_(T=3000)
    w = bench.lsa_work(wl)
    nb = wl.T // wl.n_cluster
    want = sum(min(nb, p // wl.n_cluster) * wl.n_buckets for p in range(wl.T))
    assert w["scores"] == want
    assert w["score_bytes"] == 4 * want
    assert w["score_flops"] == 2.0 * wl.d * want


def test_two_stage_work_matches_a_direct_count():
    """Candidate keys of the two-stage prefill: per query the visible keys of
    block 0, its own block and keep - 2 other complete blocks (all of them
    while fewer exist)."""
    import bench
    from workloads import WORKLOADS
    wl = WORKLOADS["two_stage_t64k"].with_(T=5000, keep_blocks=8)
    B, keep = wl.block_size, wl.keep_blocks
    cand = 0
    for p in range(wl.T):
        cur = p // B
        others = min(cur - 1, keep - 2) if cur >= 1 else 0
        cand += (B if cur >= 1 else 0) + others * B + (p % B + 1)
    assert bench.two_stage_work(wl)["cand"] == cand


def test_lsa_reference_arm_prints_one_json_line():
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "lsa_t8k", "--steps", "1", "--warmup", "0", "--ref-rows", "16"],
                       capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["config"]["workload"] == "lsa_t8k"


def test_timing_rows_cover_every_stratum_once():
    import bench
    for T, n in ((65536, 96), (1000, 7), (64, 64)):
        for seed in (0, 3):
            r = bench.timing_rows(T, n, seed)
            assert len(r) == n and (r >= 0).all() and (r < T).all()
            assert (((r * n) // T) == list(range(n))).all(), (T, n, seed)


def test_two_stage_reference_arm_reports_measured_and_extrapolated_time():
    """The reference arm's ms_per_step is the wall time it measured; the full
    workload's time is an extrapolation, reported apart and larger."""
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--T", "4096",
                        "--steps", "1", "--warmup", "0", "--ref-rows", "4"],
                       capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["config"]["T"] == 4096 and d["config"]["rows_per_step"] == 4
    assert 0 < d["ms_per_step"] < d["extrapolated_full_step_ms"]
    assert abs(d["value"] - 4096 / (d["extrapolated_full_step_ms"] * 1e-3)) <= 1e-3 * d["value"] + 1e-3
    assert d["cpu_baseline"]["cores"] > 0 and d["cpu_baseline"]["value"] == d["value"]
