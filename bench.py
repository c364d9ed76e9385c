#!/usr/bin/env python
"""Benchmark of the learned top-k sparse-attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  * a two-stage prefill of T = 65,536 tokens (block keys, stage-1 block
    scores + keep, stage-2 token indexer, exact top-k = 2048, sparse MQA
    attention over 16 heads x 128) -- the headline prefill tokens/s, and
  * one decode step of 64 sequences x 131,072 cached keys (indexer, exact
    top-2048, split-K attention) -- decode microseconds per token.
L2 (126 MB) is flushed before every timed step by writing a 512 MB buffer
outside the timed events. Inputs are seeded and synthetic (workloads module).

  python bench.py --gpus N --steps K --warmup W [--impl reference]

Under torchrun (N > 1) every rank runs its own independent copy of the
workload (weak scaling; no collective on the data path); the reported time is
the max over ranks.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn prefill tokens/s (indexer+top-k+attn) @64K k=2048; decode µs/token"
LSA_METRIC = "LSA flat prefill tokens/s (clustering+bucket search+attn) @64K k=2048"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# --------------------------------------------------------- multi-rank plumbing
def rank_seed(base: int, rank: int) -> int:
    """Every rank runs its own independent copy of the workload (weak scaling)."""
    return base + 1000 * rank


def reduce_max(values, device=None):
    """Max over ranks of per-rank device-timed values (no-op on one rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def weak_scaling_value(world: int, steps: int, units_per_rank_step: int, max_ms: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return world * steps * units_per_rank_step / (max_ms * 1e-3)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                rows.append(f)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows if _isnum(r[3])), default=None)}


def _isnum(s):
    try:
        float(s)
        return True
    except ValueError:
        return False


# DRAM bytes per launch of a kernel from one ncu capture (dram__bytes_read.sum
# + dram__bytes_write.sum), captured on the two-stage workload at T_cap rows
# and scaled to the run by the number of candidate keys scored (the candidate
# scores are most of the traffic). An entry is removed when its kernel changes.
MEASURED_DRAM = {
    # the stage-2 indexer_kernel<64, 128, 1, 3> (grouped mode), two-stage workload at T = 16384
    "stage2_indexer": {"bytes": 146.940160e6 + 183.156736e6, "T_cap": 16384},
}


def measured_traffic(kernel, wl):
    m = MEASURED_DRAM.get(kernel)
    if m is None or wl.mode != "two_stage":
        return None
    return round(m["bytes"] * two_stage_work(wl)["cand"] / two_stage_work(wl.with_(T=m["T_cap"]))["cand"])


# ------------------------------------------------------- algorithmic work
def two_stage_work(wl):
    """Data-independent algorithmic counts of the two-stage prefill."""
    T, H, d, B, keep, k = wl.T, wl.H, wl.d, wl.block_size, wl.keep_blocks, wl.k
    t = list(range(T))
    blocks_scored = sum(p // B for p in t)                       # blocks [0, cur) per query
    cand = sum(min(p + 1, (keep - 1) * B + p % B + 1) for p in t)  # visible keys of the kept blocks
    pairs = sum(min(k, p + 1) for p in t)                        # selected keys attended
    return {
        "stage1_flops": 2.0 * H * d * blocks_scored,
        "stage2_flops": 2.0 * H * d * cand,
        "cand": cand,
        "attn_pairs": pairs,
        "attn_bytes": pairs * 2 * wl.dh * 2,                     # gathered K+V rows (bf16)
        "attn_flops": 4.0 * wl.Hq * wl.dh * pairs,
        "topk_bytes": cand * 4 + T * k * 4,                      # candidate scores read + index rows written
    }


def flat_work(wl, streaming: bool):
    """Algorithmic counts of the flat prefill (every visible key scored)."""
    T, H, d, k = wl.T, wl.H, wl.d, wl.k
    scores = T * (T + 1) // 2                                    # sum over t of (t + 1)
    pairs = sum(min(k, p + 1) for p in range(T))
    return {
        "indexer_flops": 2.0 * H * d * scores,
        "attn_pairs": pairs,
        "attn_bytes": pairs * 2 * wl.dh * 2,
        "attn_flops": 4.0 * wl.Hq * wl.dh * pairs,
        # table path: the score table is read once by the selector (+ index rows written)
        "topk_bytes": 0 if streaming else scores * 4 + T * k * 4,
    }


def decode_work(wd):
    B, L, d = wd.batch, wd.L, wd.d
    return {
        "indexer_bytes": B * L * (d + 4) + B * L * 4,            # FP8 keys + scales read, row scores written
        "indexer_flops": 2.0 * wd.H * d * B * L,
        "topk_bytes": B * L * 4,
        "attn_bytes": B * min(wd.k, L) * 2 * wd.dh * 2,          # gathered K+V rows from HBM
    }


def lsa_work(wl):
    """Algorithmic counts of the LSA flat prefill over T tokens."""
    T, nc, m = wl.T, wl.n_cluster, wl.n_buckets
    nb = T // nc
    vis = [min(nb, p // nc) * m for p in range(T)]             # buckets each query scores
    return {
        "scores": sum(vis),
        "score_bytes": sum(vis) * 4,                             # S written once (read again by the top-p)
        "score_flops": 2.0 * wl.d * sum(vis),
    }


# ------------------------------------------------------------- CPU oracle
def timing_rows(T: int, n: int, seed: int = 0):
    """n evenly spaced query rows, t_i = floor((i + f) T / n), with the
    offset f in [0, 1) drawn from the seed: every stratum of [0, T) once, so
    the mean cost per row estimates the mean over all rows."""
    import numpy as np
    f = (0.5 + seed * 0.6180339887498949) % 1.0
    return np.minimum(T - 1, ((np.arange(n) + f) * T / n).astype(np.int64))


def oracle_two_stage_sample(host, wl, n_rows: int, seed: int = 0):
    """Times the oracle on pooling (all blocks) + n_rows evenly spaced rows of
    the two-stage prefill; returns (tokens/s extrapolated to T rows, info).
    info["cores"] is the process CPU time over the wall time: the host cores
    the oracle kept busy (its row loop is serial; numpy's BLAS threads the
    products)."""
    import oracle
    from oracle.two_stage import pool_block_keys
    rows = timing_rows(wl.T, n_rows, seed)
    c0, t0 = time.process_time(), time.perf_counter()
    blocks = pool_block_keys(host["k_idx"].numpy(), host["k_scale"].numpy(), wl.block_size)
    t1 = time.perf_counter()
    oracle.prefill_rows(host, rows, wl.k, mode="two_stage", keep=wl.keep_blocks, blocks=blocks)
    c2, t2 = time.process_time(), time.perf_counter()
    per_row = (t2 - t1) / len(rows)
    full_s = (t1 - t0) + per_row * wl.T
    return wl.T / full_s, {"pool_s": t1 - t0, "rows": len(rows), "rows_s": t2 - t1, "extrapolated_s": full_s,
                           "measured_s": t2 - t0, "cores": round((c2 - c0) / max(t2 - t0, 1e-9), 2)}


def oracle_decode_sample(hostd, wd, n_seq: int):
    import oracle
    t0 = time.perf_counter()
    oracle.decode_rows(hostd, range(n_seq), wd.k)
    dt = time.perf_counter() - t0
    return dt / n_seq * wd.batch * 1e6, dt        # µs per decode step of the full batch


def oracle_lsa_sample(k_host, q_host, attn_host, wl, n_rows: int, seed: int):
    """Times the LSA oracle: the bucket cache of every cluster block, then
    n_rows stratified query rows (search + attention); tokens/s extrapolated
    to T rows."""
    import numpy as np
    import oracle
    from oracle import lsa
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(wl.T, n_rows, replace=False))
    t0 = time.perf_counter()
    cent, off, keys = lsa.build_buckets(k_host, wl.n_pool, wl.n_cluster, wl.n_buckets, wl.max_bucket_keys)
    t1 = time.perf_counter()
    nb = wl.T // wl.n_cluster
    qn = lsa.normalized_queries(q_host[rows])
    Q, K, V = attn_host
    for r, qv in zip(rows, qn):
        J = lsa.search_row(qv, int(r), cent, off, keys, nb, wl.n_cluster, wl.n_buckets, wl.p, wl.k, wl.n_sink,
                           wl.n_window)
        oracle.sparse_attention_row(Q[r], K, V, J)
    t2 = time.perf_counter()
    full_s = (t1 - t0) + (t2 - t1) / len(rows) * wl.T
    return wl.T / full_s, {"build_s": t1 - t0, "rows": len(rows), "rows_s": t2 - t1, "extrapolated_s": full_s}


def lsa_host_inputs(wl, seed):
    from workloads import LsaInputs
    inp = LsaInputs(wl, "cpu", seed=seed)
    Q, K, V = inp.attention_operands()
    return (inp.k_idx.float().numpy(), inp.q_idx.float().numpy(),
            (Q.double().numpy(), K.double().numpy(), V.double().numpy()))


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max(i.get("num_threads", 1) for i in info if i.get("user_api") == "blas")
    except Exception:
        return os.cpu_count()


# --------------------------------------------------------------- arms
def run_reference_lsa(args):
    """The LSA oracle as the reference arm (rank 0, host cores)."""
    from workloads import LSA_WORKLOADS
    wl = LSA_WORKLOADS[args.workload]
    k_host, q_host, attn_host = lsa_host_inputs(wl, args.seed)
    for i in range(args.warmup):
        oracle_lsa_sample(k_host, q_host, attn_host, wl, args.ref_rows, seed=100 + i)
    vals, infos = [], []
    for i in range(args.steps):
        v, info = oracle_lsa_sample(k_host, q_host, attn_host, wl, args.ref_rows, seed=200 + i)
        vals.append(v)
        infos.append(info)
    value = statistics.mean(vals)
    sample = (f"per step: the bucket cache of all {wl.T // wl.n_cluster} cluster blocks + {args.ref_rows} "
              f"query rows (search, attention), extrapolated to {wl.T} rows")
    line = {
        "impl": "reference", "metric": LSA_METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(statistics.mean(x["extrapolated_s"] for x in infos) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 clustering, f64 scores",
        "data": "synthetic", "config": {"workload": wl.name, "T": wl.T, "k": wl.k, "p": wl.p, "seed": args.seed},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference(args):
    """The oracle as the reference arm: rank 0 only, on host cores."""
    import torch
    from workloads import WORKLOADS, PrefillInputs, DecodeInputs, LSA_WORKLOADS
    if args.workload in LSA_WORKLOADS:
        return run_reference_lsa(args)
    wl = WORKLOADS[args.workload]
    if args.T:
        wl = wl.with_(T=args.T)
    wd = WORKLOADS["decode_b64_l128k"]
    inp = PrefillInputs(wl, "cpu", seed=args.seed)
    host = inp.to_host()
    dinp = DecodeInputs(wd.with_(batch=2), "cpu", seed=args.seed)
    hostd = dinp.to_host()
    for i in range(args.warmup):
        oracle_two_stage_sample(host, wl, args.ref_rows, seed=100 + i)
    vals, infos = [], []
    for i in range(args.steps):
        v, info = oracle_two_stage_sample(host, wl, args.ref_rows, seed=200 + i)
        vals.append(v)
        infos.append(info)
    dec_us, _ = oracle_decode_sample(hostd, wd.with_(batch=2), 1)
    dec_us = dec_us / 2 * wd.batch
    value = statistics.mean(vals)
    measured_s = statistics.mean(x["measured_s"] for x in infos)
    sec_per_step = statistics.mean(x["extrapolated_s"] for x in infos)
    cores = round(statistics.mean(x["cores"] for x in infos), 2)
    sample = (f"per step: mean-pooling of all {wl.T // wl.block_size} blocks + {args.ref_rows} evenly spaced "
              f"query rows (both indexer stages, top-k, attention); value = {wl.T} rows over the extrapolated "
              f"time of all rows; cores = process CPU time / wall time")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        # the measured wall time of one step (its sample); the full workload's
        # time is an extrapolation and is reported apart
        "ms_per_step": round(measured_s * 1e3, 3),
        "extrapolated_full_step_ms": round(sec_per_step * 1e3, 3),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "k": wl.k, "mode": "two_stage", "block": wl.block_size,
                   "keep_blocks": wl.keep_blocks, "seed": args.seed, "rows_per_step": args.ref_rows},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "threads": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "decode": {"us_per_step": round(dec_us, 1), "us_per_token": round(dec_us / wd.batch, 2),
                   "sample": "1 sequence of 131072 keys, scaled to the 64-sequence step"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_native_lsa(args, rank, world, local_rank):
    """The LSA flat prefill: bucket cache of every cluster block, the index
    rows of every query, attention over them."""
    import torch
    import torch.distributed as dist
    import indexer_selected_top_b200 as sa
    from workloads import LSA_WORKLOADS, LsaInputs
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = LSA_WORKLOADS[args.workload]
    if args.T:
        wl = wl.with_(T=args.T)
    inp = LsaInputs(wl, dev, seed=rank_seed(args.seed, rank))
    Q, K, V = inp.attention_operands()
    prm = sa.lsa_params(n_pool=wl.n_pool, n_cluster=wl.n_cluster, n_buckets=wl.n_buckets,
                        max_bucket_keys=wl.max_bucket_keys)
    timer = sa.StageTimer(sa.LsaPrefill.STAGES)
    run = sa.LsaPrefill(inp.k_idx, inp.q_idx, Q, K, V, prm, wl.p, wl.k, wl.n_sink, wl.n_window, timer=timer)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush.fill_(1)
        run()
    torch.cuda.synchronize()
    if run.stage_status[:, 0].any():
        raise RuntimeError(f"LSA prefill status {run.stage_status.cpu().tolist()}")
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    tot, stage_ms = 0.0, {n: 0.0 for n in timer.names}
    for _ in range(args.steps):
        flush.fill_(1)                                   # evict L2, outside the timed events
        run()
        torch.cuda.synchronize()
        for n, v in timer.ms().items():
            stage_ms[n] += v
        tot += timer.events[0].elapsed_time(timer.events[-1])
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    K_ = args.steps
    tot = reduce_max([tot], device=dev)[0]
    peaks, peak_src = load_peaks()
    work = lsa_work(wl)
    # attention work: the (query, key) pairs the served rows actually hold
    work["attn_pairs"] = int((run.J >= 0).sum().item())
    work["attn_flops"] = 4.0 * wl.Hq * wl.dh * work["attn_pairs"]
    avg = {n: v / K_ for n, v in stage_ms.items()}
    stages = {n: {"ms": round(v, 4)} for n, v in avg.items()}
    # search: the score rows S are written once and read once by the top-p (HBM)
    s_search = max(avg["search"], 1e-9) * 1e-3
    stages["search"].update({"bound": "hbm", "achieved": round(2 * work["score_bytes"] / s_search / 1e9, 2),
                             "peak": peaks["hbm_gbs"], "unit": "GB/s"})
    s_attn = max(avg["attention"], 1e-9) * 1e-3
    stages["attention"].update({"bound": "tensor", "achieved": round(work["attn_flops"] / s_attn / 1e12, 2),
                                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"})
    for v in stages.values():
        if "achieved" in v:
            v["frac"] = round(v["achieved"] / v["peak"], 4)
    dom = max((n for n in stages if "achieved" in stages[n]), key=lambda n: stages[n]["ms"])
    roof = dict(stages[dom])
    roof.pop("ms")
    roof.update({"kernel": dom, "traffic": None,
                 "peak_source": f"{peak_src}: " + ("bf16 burst" if roof["unit"] == "TFLOP/s" else "HBM copy")})
    # ---------------- LSA decode step: 64 sequences, one new query each ----------------
    decode = None
    if not args.no_decode:
        B, L = args.lsa_decode_batch, wl.T
        nbl = L // wl.n_cluster
        cent = torch.zeros((B, nbl * wl.n_buckets, wl.d), dtype=torch.bfloat16, device=dev)
        boff = torch.zeros((B, nbl * wl.n_buckets), dtype=torch.int32, device=dev)
        bkeys = torch.zeros((B, nbl * wl.n_cluster), dtype=torch.int32, device=dev)
        qd = torch.empty((B, wl.d), dtype=torch.bfloat16, device=dev)
        for b in range(B):                                 # every sequence its own index keys and cache
            sb = LsaInputs(wl, dev, seed=rank_seed(args.seed, rank) + 10_000 + b)
            sa.lsa_build_buckets(sb.k_idx, prm, n_blocks=nbl, out=(cent[b], boff[b], bkeys[b]))
            qd[b] = sb.q_idx[L - 1]
            del sb
        g = torch.Generator(device=dev)
        g.manual_seed(rank_seed(args.seed, rank) + 20_000)
        std = 1.0 / math.sqrt(wl.dh)
        Kd = (torch.randn((B, L, wl.dh), generator=g, device=dev) * std).to(torch.bfloat16)
        Vd = (torch.randn((B, L, wl.dh), generator=g, device=dev) * std).to(torch.bfloat16)
        Qd = (torch.randn((B, wl.Hq, wl.dh), generator=g, device=dev) * std).to(torch.bfloat16)
        nbt = torch.full((B,), nbl, dtype=torch.int32, device=dev)
        lens = torch.full((B,), L, dtype=torch.int32, device=dev)
        ldec = sa.LsaDecode(qd, prm, (cent, boff, bkeys), nbt, lens, wl.p, wl.k, wl.n_sink, wl.n_window)
        out_d = torch.empty_like(Qd)
        lse_d = torch.empty((B, wl.Hq), dtype=torch.float32, device=dev)

        def dstep():
            J = ldec()
            sa.sparse_attn(Qd, Kd, Vd, J, out=out_d, lse=lse_d)

        for _ in range(args.warmup):
            flush.fill_(1)
            dstep()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        sel_ms = att_ms = 0.0
        for _ in range(K_):
            flush.fill_(1)
            ev[0].record(stream)
            J = ldec()
            ev[1].record(stream)
            sa.sparse_attn(Qd, Kd, Vd, J, out=out_d, lse=lse_d)
            ev[2].record(stream)
            torch.cuda.synchronize()
            sel_ms += ev[0].elapsed_time(ev[1])
            att_ms += ev[1].elapsed_time(ev[2])
        sel_ms, att_ms = reduce_max([sel_ms / K_, att_ms / K_], device=dev)
        cent_bytes = B * nbl * wl.n_buckets * (wl.d * 2 + 4)      # centroids read + row scores written
        us = (sel_ms + att_ms) * 1e3
        decode = {"us_per_step": round(us, 1), "us_per_token": round(us / B, 3), "batch": B, "L": L,
                  "select_us": round(sel_ms * 1e3, 1), "attention_us": round(att_ms * 1e3, 1),
                  "scan_hbm_bytes": cent_bytes,
                  "select_hbm_frac": round(cent_bytes / (sel_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
        # the selection replayed from a CUDA graph (no per-kernel launch cost), after the L2 flush
        g = ldec.graph()
        for _ in range(args.warmup):
            flush.fill_(1)
            g.replay()
        gt = 0.0
        for _ in range(K_):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            gt += a.elapsed_time(b)
        decode["graph_select_us"] = round(reduce_max([gt / K_ * 1e3], device=dev)[0], 1)
        del g, Kd, Vd

    e2e = None
    if not args.skip_e2e:
        srcs = (inp.k_idx, inp.q_idx, Q, K, V)
        hbuf = [t.cpu().pin_memory() for t in srcs]
        hout = torch.empty(run.out.shape, dtype=run.out.dtype).pin_memory()
        hlse = torch.empty(run.lse.shape, dtype=run.lse.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in hbuf)
        d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()
        ne = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            for d_, h_ in zip(srcs, hbuf):
                d_.copy_(h_, non_blocking=True)
            run()
            hout.copy_(run.out, non_blocking=True)
            hlse.copy_(run.lse, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(ne):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        t_e2e = reduce_max([a.elapsed_time(b) / ne], device=dev)[0]
        e2e = {"value": round(weak_scaling_value(world, 1, wl.T, t_e2e), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": ne}
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        k_host, q_host, attn_host = (inp.k_idx.float().cpu().numpy(), inp.q_idx.float().cpu().numpy(),
                                     (Q.double().cpu().numpy(), K.double().cpu().numpy(), V.double().cpu().numpy()))
        v, info = oracle_lsa_sample(k_host, q_host, attn_host, wl, args.lsa_cpu_rows, seed=7)
        cpu = {"value": round(v, 3), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"bucket cache of all {wl.T // wl.n_cluster} cluster blocks ({info['build_s']:.1f} s) + "
                         f"{info['rows']} query rows ({info['rows_s']:.1f} s: search, attention), extrapolated "
                         f"to {wl.T} rows"}
    chunks = -(-wl.T // 8192)
    # clustering; per 8192-query chunk: unit queries, scores, lengths, top-p, expansion; attention: per
    # 16384-query chunk local union, local pass, signatures, sort, long-range union, long-range pass, merge
    # (one launch on the per-query kernel)
    attn_launches = 7 * -(-wl.T // 16384) if run.attn.supported else 1
    launches = 1 + 5 * chunks + attn_launches
    line = {
        "metric": LSA_METRIC,
        "value": round(weak_scaling_value(world, K_, wl.T, tot), 1),
        "unit": "tokens/s", "n_gpus": world, "steps": K_, "warmup": args.warmup,
        "ms_per_step": round(tot / K_, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 index (f32 clustering and accumulation), bf16 attention (f32 softmax)",
        "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "d_idx": wl.d,
                   "attention": "tensor-core local + long-range passes" if run.attn.supported else "per-query", "n_pool": wl.n_pool, "n_cluster": wl.n_cluster,
                   "buckets_per_block": wl.n_buckets, "max_bucket_keys": wl.max_bucket_keys, "p": wl.p,
                   "k": wl.k, "n_sink": wl.n_sink, "n_window": wl.n_window, "Hq": wl.Hq, "head_dim": wl.dh,
                   "parallelism": f"replicas x{world}", "l2": "flushed (512 MB write) before every step"},
        "roofline": roof, "stages": stages, "decode": decode, "cpu_baseline": cpu, "e2e": e2e,
        # per stage (cluster, search, attention): error, wait site, fallback rows, overflowed rows
        "status": run.stage_status.cpu().tolist(),
        "gpu_launches": launches * K_, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def _build_library():
    import importlib.util
    spec = importlib.util.spec_from_file_location("_sa_build", os.path.join(ROOT, "indexer_selected_top_b200",
                                                                            "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


def measure_fp8_peak(dev, n: int = 8192, reps: int = 10):
    """Dense FP8 e4m3 tensor throughput of this GPU, measured the way the bf16
    peak in MEASURED_PEAKS.json is: one n^3 product (torch._scaled_mm, cuBLAS,
    bf16 output), best of `reps` CUDA-event timings, 2 n^3 flops."""
    import torch
    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
    one = torch.tensor(1.0, device=dev)
    for _ in range(3):
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e1.record()
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del a, b
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def prefill_roofline(wl, stages_ms: dict, peaks: dict, fp8_peak: float, traffic_known: bool = True):
    """Per-stage roofline of a prefill (algorithmic work over the stage's
    device time, summed over chunks) and the dominant stage's entry."""
    streaming = wl.mode != "two_stage" and wl.T > 65536
    work = two_stage_work(wl) if wl.mode == "two_stage" else flat_work(wl, streaming)
    idx_peak = fp8_peak if wl.idx_dtype == "fp8" else peaks["bf16_tflops"]
    flop_stage = {"stage2_indexer": "stage2_flops", "stage1_indexer": "stage1_flops", "indexer": "indexer_flops"}
    stages = {}
    for n, ms in stages_ms.items():
        s = max(ms, 1e-9) * 1e-3
        if n in flop_stage:
            stages[n] = {"ms": round(ms, 4), "bound": "tensor", "achieved": work[flop_stage[n]] / s / 1e12,
                         "peak": idx_peak, "unit": "TFLOP/s"}
        elif n == "attention":
            # the grouped kernels read each union key once per group of queries
            # (from L2), so gathered bytes do not bound them: the algorithmic
            # work is the 4 Hq dh flops of every selected (query, key) pair
            stages[n] = {"ms": round(ms, 4), "bound": "tensor", "achieved": work["attn_flops"] / s / 1e12,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
        elif n == "topk" and work["topk_bytes"] > 0 and ms > 0:
            stages[n] = {"ms": round(ms, 4), "bound": "hbm", "achieved": work["topk_bytes"] / s / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        else:
            stages[n] = {"ms": round(ms, 4)}
    for v in stages.values():
        if "achieved" in v:
            v["achieved"] = round(v["achieved"], 2)
            v["peak"] = round(v["peak"], 1)
            v["frac"] = round(v["achieved"] / v["peak"], 4)
    dom = max((n for n in stages if "achieved" in stages[n]), key=lambda n: stages[n]["ms"])
    roof = dict(stages[dom])
    roof.pop("ms")
    roof["kernel"] = dom
    roof["traffic"] = measured_traffic(dom, wl) if traffic_known else None
    return stages, roof


def time_lsa_prefill(sa, wl, dev, seed: int, warmup: int, steps: int, flush, peaks):
    """The LSA flat prefill of `wl` (bucket cache of every cluster block, the
    index rows of every query, attention over them), timed on the device like
    time_prefill. Returns a dict for the JSON line (tokens/s, stage times,
    roofline of the dominant stage, status words)."""
    import torch
    from workloads import LsaInputs
    inp = LsaInputs(wl, dev, seed=seed)
    Q, K, V = inp.attention_operands()
    prm = sa.lsa_params(n_pool=wl.n_pool, n_cluster=wl.n_cluster, n_buckets=wl.n_buckets,
                        max_bucket_keys=wl.max_bucket_keys)
    timer = sa.StageTimer(sa.LsaPrefill.STAGES)
    run = sa.LsaPrefill(inp.k_idx, inp.q_idx, Q, K, V, prm, wl.p, wl.k, wl.n_sink, wl.n_window, timer=timer)
    for _ in range(warmup):
        flush.fill_(1)
        run()
    torch.cuda.synchronize()
    tot, stage_ms = 0.0, {n: 0.0 for n in timer.names}
    for _ in range(steps):
        flush.fill_(1)
        run()
        torch.cuda.synchronize()
        if run.stage_status[:, 0].any():
            raise RuntimeError(f"LSA prefill status {run.stage_status.cpu().tolist()}")
        for n, v in timer.ms().items():
            stage_ms[n] += v
        tot += timer.total_ms()
    work = lsa_work(wl)
    pairs = int((run.J >= 0).sum().item())
    avg = {n: v / steps for n, v in stage_ms.items()}
    stages = {n: {"ms": round(v, 4)} for n, v in avg.items()}
    stages["search"].update({"bound": "hbm", "achieved": round(2 * work["score_bytes"] / (avg["search"] * 1e-3) / 1e9,
                                                                2), "peak": peaks["hbm_gbs"], "unit": "GB/s"})
    stages["attention"].update({"bound": "tensor", "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                "achieved": round(4.0 * wl.Hq * wl.dh * pairs / (avg["attention"] * 1e-3) / 1e12, 2)})
    for v in stages.values():
        if "achieved" in v:
            v["frac"] = round(v["achieved"] / v["peak"], 4)
    dom = max((n for n in stages if "achieved" in stages[n]), key=lambda n: stages[n]["ms"])
    roof = dict(stages[dom])
    roof.pop("ms")
    roof.update({"kernel": dom, "traffic": None})
    ms = tot / steps
    return {"tokens_per_s": round(wl.T / (ms * 1e-3), 1), "ms_per_step": round(ms, 4), "T": wl.T, "p": wl.p,
            "k": wl.k, "n_sink": wl.n_sink, "n_window": wl.n_window, "warmup": warmup, "steps": steps,
            "attention": "tensor-core local + long-range passes" if run.attn.supported else "per-query",
            "stages": stages, "roofline": roof, "status": run.stage_status.cpu().tolist()}


def time_prefill(sa, wl, dev, seed: int, warmup: int, steps: int, flush, mode=None):
    """A prepared sa_prefill over one seeded input of `wl`, timed on the
    device (CUDA events, L2 flushed before every step outside the events).
    Returns (ms per step, stage ms per step summed over chunks, status words,
    prepared call, inputs)."""
    import torch
    from workloads import PrefillInputs
    inp = PrefillInputs(wl, dev, seed=seed)
    status = sa.new_status(dev)
    mode = mode or wl.mode
    # the library's default chunking; two-stage tables for all rows at once
    chunk = wl.T if mode == "two_stage" else 0
    pre = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, wl.k, mode=mode,
                     keep_blocks=wl.keep_blocks, chunk_rows=chunk, status=status, timed=True)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush.fill_(1)
        pre()
    torch.cuda.synchronize()
    tot, stage_ms = 0.0, {n: 0.0 for n in pre.timer.names}
    words = [0, 0, 0, 0]
    for _ in range(steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pre()
        e1.record(stream)
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
        for n, v in pre.timer.ms().items():
            stage_ms[n] += v
        w = status.cpu().tolist()
        if w[0] != 0:
            raise RuntimeError(f"{wl.name}: device status {w}")
        words = [max(a, b) for a, b in zip(words, w)]
    return tot / steps, {n: v / steps for n, v in stage_ms.items()}, words, pre, inp


def run_native(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from workloads import LSA_WORKLOADS
    if rank == 0:
        _build_library()
    if world > 1:
        dist.barrier()
    if args.workload in LSA_WORKLOADS:
        return run_native_lsa(args, rank, world, local_rank)
    import indexer_selected_top_b200 as sa
    from workloads import WORKLOADS, DecodeInputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    fp8_peak = measure_fp8_peak(dev)
    wl = WORKLOADS[args.workload]
    if args.T:
        wl = wl.with_(T=args.T)
    wd = WORKLOADS["decode_b64_l128k"]
    if args.decode_L:
        wd = wd.with_(L=args.decode_L)
    seed = rank_seed(args.seed, rank)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    # ---------------- the headline prefill, the decode step ----------------
    from workloads import PrefillInputs
    inp = PrefillInputs(wl, dev, seed=seed)
    pstatus = sa.new_status(dev)
    chunk = wl.T if wl.mode == "two_stage" else 0
    pre = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, wl.k, mode=wl.mode,
                     keep_blocks=wl.keep_blocks, chunk_rows=chunk, status=pstatus, timed=True)
    ptimer = pre.timer
    dec = dstatus = None
    if not args.no_decode:
        dinp = DecodeInputs(wd, dev, seed=seed)
        dtimer = sa.StageTimer(sa.DECODE_STAGES)
        dstatus = sa.new_status(dev)
        dec = sa.Decode(dinp.q_idx, dinp.q_scale, dinp.k_idx, dinp.k_scale, dinp.w, dinp.Q, dinp.K, dinp.V,
                        dinp.seq_lens, wd.k, timer=dtimer, status=dstatus)

    def step():
        flush.fill_(1)                                   # evict L2, outside the timed events
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        pre()
        e1.record(stream)
        if dec is not None:
            dec()
        e2.record(stream)
        return e0, e1, e2

    def check_status():
        for name, st in (("prefill", pstatus), ("decode", dstatus)):
            if st is not None and st[0].item() != 0:
                raise RuntimeError(f"{name}: device status {st.cpu().tolist()}")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    check_status()
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    recs = []
    stage_ms = {n: 0.0 for n in ptimer.names}
    dstage_ms = {n: 0.0 for n in sa.DECODE_STAGES}
    words = {"prefill": [0, 0, 0, 0], "decode": [0, 0, 0, 0]}
    for _ in range(args.steps):
        recs.append(step())
        torch.cuda.synchronize()                         # read this step's stage events and status words
        check_status()
        for n, v in ptimer.ms().items():
            stage_ms[n] += v
        if dec is not None:
            for n, v in dtimer.ms().items():
                dstage_ms[n] += v
        for name, st in (("prefill", pstatus), ("decode", dstatus)):
            if st is not None:
                words[name] = [max(a, b) for a, b in zip(words[name], st.cpu().tolist())]
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    pre_ms = sum(a.elapsed_time(b) for a, b, _ in recs)
    dec_ms = sum(b.elapsed_time(c) for _, b, c in recs)
    pre_ms, dec_ms, all_ms = reduce_max([pre_ms, dec_ms, pre_ms + dec_ms], device=dev)
    K = args.steps

    avg = {n: v / K for n, v in stage_ms.items()}
    stages, roof = prefill_roofline(wl, avg, peaks, fp8_peak)
    roof["peak_source"] = (f"FP8 e4m3: measured in this run (cuBLAS _scaled_mm 8192^3, best of 10); "
                           f"2 x the bf16 burst of MEASURED_PEAKS.json would be {2 * peaks['bf16_tflops']:.1f}"
                           if roof["unit"] == "TFLOP/s" and roof["peak"] == round(fp8_peak, 1)
                           else f"{peak_src}: " + ("bf16 burst" if roof["unit"] == "TFLOP/s" else "HBM copy"))

    decode = None
    if dec is not None:
        dw = decode_work(wd)
        davg = {n: v / K for n, v in dstage_ms.items()}
        us = dec_ms / K * 1e3
        decode = {"us_per_step": round(us, 1), "us_per_token": round(us / wd.batch, 3), "batch": wd.batch,
                  "L": wd.L, "k": wd.k, "stages_ms": {n: round(v, 4) for n, v in davg.items()},
                  "indexer_hbm_frac": round(dw["indexer_bytes"] / (davg["indexer"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                            4),
                  "gather_hbm_frac": round(dw["attn_bytes"] / (davg["attention"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                           4),
                  "step_hbm_frac": round((dw["indexer_bytes"] + dw["topk_bytes"] + dw["attn_bytes"]) /
                                         (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                  "status": words["decode"]}
        # the same step replayed from a CUDA graph (no per-kernel launch cost),
        # each replay after the L2 flush, timed on the device like the eager steps
        g = dec.graph()
        for _ in range(args.warmup):
            flush.fill_(1)
            g.replay()
        gt = 0.0
        for _ in range(K):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            gt += a.elapsed_time(b)
        check_status()
        gus = reduce_max([gt / K * 1e3], device=dev)[0]
        decode["graph_us_per_step"] = round(gus, 1)
        decode["graph_us_per_token"] = round(gus / wd.batch, 3)
        del g
        decode["gather_gbs"] = round(dw["attn_bytes"] / (davg["attention"] * 1e-3) / 1e9, 1)
        # graphs per context-length bucket: every sequence at the bucket's
        # length, the narrowest bucket's graph replayed after the L2 flush
        graphs = sa.DecodeGraphs(dec, wd.L)
        saved = dinp.seq_lens.clone()
        per_bucket = {}
        for b in graphs.buckets:
            if b < 16384:
                continue
            dinp.seq_lens.fill_(b)
            for _ in range(args.warmup):
                flush.fill_(1)
                graphs.replay(b)
            bt = 0.0
            for _ in range(K):
                flush.fill_(1)
                a, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                graphs.replay(b)
                e_.record()
                e_.synchronize()
                bt += a.elapsed_time(e_)
            check_status()
            per_bucket[str(b)] = round(reduce_max([bt / K * 1e3], device=dev)[0], 1)
        dinp.seq_lens.copy_(saved)
        decode["graph_us_per_bucket"] = per_bucket
        del graphs

    # ---------------- end to end through host buffers ----------------
    e2e = None
    if not args.skip_e2e:
        names = ("q_idx", "q_scale", "k_idx", "k_scale", "w", "Q", "K", "V")
        hbuf = {n: getattr(inp, n).cpu().pin_memory() for n in names}
        hout = torch.empty(pre.out.shape, dtype=pre.out.dtype).pin_memory()
        hlse = torch.empty(pre.lse.shape, dtype=pre.lse.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in hbuf.values())
        d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()
        ne = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            for n in names:
                getattr(inp, n).copy_(hbuf[n], non_blocking=True)
            pre()
            hout.copy_(pre.out, non_blocking=True)
            hlse.copy_(pre.lse, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(ne):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        check_status()
        t_serial = reduce_max([a.elapsed_time(b) / ne], device=dev)[0]

        # the same steps pipelined: two device input sets with a prepared call
        # each; a step's host-to-device copies (one stream) overlap the prefill
        # of the step before, and its result is read back (another stream)
        # while the next one runs. Every step still copies all its inputs in
        # and its outputs out inside the timed region.
        dsets = [{n: getattr(inp, n) for n in names},
                 {n: torch.empty_like(getattr(inp, n)) for n in names}]
        pres = [pre, sa.Prefill(*(dsets[1][n] for n in names), wl.k, mode=wl.mode, keep_blocks=wl.keep_blocks,
                                chunk_rows=chunk, status=pstatus)]
        houts = [(hout, hlse), (torch.empty_like(hout).pin_memory(), torch.empty_like(hlse).pin_memory())]
        copy_in, copy_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        free = [torch.cuda.Event() for _ in range(2)]       # the set's prefill is done (inputs free, outputs ready)
        landed = [torch.cuda.Event() for _ in range(2)]     # the set's inputs are on the device
        read = [torch.cuda.Event() for _ in range(2)]       # the set's outputs are on the host

        def piped_step(i, start=None):
            k_ = i % 2
            with torch.cuda.stream(copy_in):
                if start is not None:
                    copy_in.wait_event(start)
                if i >= 2:
                    copy_in.wait_event(free[k_])
                for n in names:
                    dsets[k_][n].copy_(hbuf[n], non_blocking=True)
                landed[k_].record(copy_in)
            stream.wait_event(landed[k_])
            if i >= 2:
                stream.wait_event(read[k_])
            pres[k_]()
            free[k_].record(stream)
            with torch.cuda.stream(copy_out):
                copy_out.wait_event(free[k_])
                houts[k_][0].copy_(pres[k_].out, non_blocking=True)
                houts[k_][1].copy_(pres[k_].lse, non_blocking=True)
                read[k_].record(copy_out)

        for i in range(2):
            piped_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(ne):
            piped_step(i + 2, start=a if i == 0 else None)
        stream.wait_stream(copy_in)
        stream.wait_stream(copy_out)
        b.record(stream)
        torch.cuda.synchronize()
        check_status()
        t_e2e = reduce_max([a.elapsed_time(b) / ne], device=dev)[0]
        del pres, dsets
        e2e = {"value": round(weak_scaling_value(world, 1, wl.T, t_e2e), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": ne,
               "pipelined": "inputs of step i + 1 copied in while step i runs; outputs read back while the next runs",
               "serial_value": round(weak_scaling_value(world, 1, wl.T, t_serial), 1)}

    # ---------------- CPU oracle baseline (rank 0, N = 1) ----------------
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        host = inp.to_host()
        v, info = oracle_two_stage_sample(host, wl, args.cpu_rows)
        cpu = {"value": round(v, 3), "unit": "tokens/s", "cores": info["cores"], "kind": "oracle",
               "threads": blas_threads(),
               "sample": f"mean-pooling of all {wl.T // wl.block_size} blocks ({info['pool_s']:.1f} s) + "
                         f"{info['rows']} evenly spaced rows ({info['rows_s']:.1f} s: both indexer stages, top-k, "
                         f"attention), extrapolated to {wl.T} rows; cores = process CPU time / wall time"}
    if wl.mode == "two_stage":
        # pool, stage 1, keep, query groups, group block unions, stage 2, top-k,
        # attention groups, group key unions, attention
        pre_launches = 10 * pre.chunks
    elif wl.T <= 65536:
        pre_launches = 3 * pre.chunks          # indexer (table), top-k, attention
    else:                                      # streaming: sample gathers once; per chunk sample scores,
        pre_launches = 2 + 6 * pre.chunks      # thresholds, scan, list select, compaction, attention
    launches_per_step = pre_launches + (4 if dec is not None else 0)
    headline_cfg = {"workload": wl.name, "T": wl.T, "H": wl.H, "d_idx": wl.d, "k": wl.k, "mode": wl.mode,
                    "block": wl.block_size, "keep_blocks": wl.keep_blocks, "Hq": wl.Hq, "head_dim": wl.dh,
                    "decode": None if dec is None else {"workload": wd.name, "batch": wd.batch, "L": wd.L},
                    "parallelism": f"replicas x{world}", "l2": "flushed (512 MB write) before every step",
                    "prefill_ms_per_step": round(pre_ms / K, 4), "status": words["prefill"]}
    del pre, inp
    if dec is not None:
        del dec, dinp
    torch.cuda.empty_cache()

    # ---------------- the other configurations, one line each ----------------
    configs = {}
    if not args.headline_only:
        for name, mode, w_c, k_c in (("tiny_t512", None, 3, 20), ("prefill_t16k", None, 3, 5),
                                     ("two_stage_t64k", "flat", 2, 3), ("prefill_t1m", None, 1, 1)):
            c = WORKLOADS[name]
            if mode:
                c = c.with_(mode=mode)
            ms, sms, st, pc, ci = time_prefill(sa, c, dev, seed, w_c, k_c, flush)
            ms = reduce_max([ms], device=dev)[0]
            cst, croof = prefill_roofline(c, sms, peaks, fp8_peak, traffic_known=False)
            configs[name + ("_flat" if mode else "")] = {
                "tokens_per_s": round(weak_scaling_value(world, 1, c.T, ms), 1), "ms_per_step": round(ms, 4),
                "T": c.T, "k": c.k, "mode": c.mode, "idx_dtype": c.idx_dtype,
                "path": ("two-stage" if c.mode == "two_stage" else
                         "flat, score table" if c.T <= 65536 else "flat, streaming threshold (no table)"),
                "chunks": pc.chunks, "warmup": w_c, "steps": k_c, "stages": cst, "roofline": croof,
                "status": st}
            del pc, ci
            torch.cuda.empty_cache()
        # the LSA flat semantic search of the same length (clustering, bucket search, attention)
        from workloads import LSA_WORKLOADS
        lsa_line = time_lsa_prefill(sa, LSA_WORKLOADS["lsa_t64k"], dev, seed, 3, 5, flush, peaks)
        lsa_line["tokens_per_s"] = round(weak_scaling_value(world, 1, lsa_line["T"],
                                                            reduce_max([lsa_line["ms_per_step"]], device=dev)[0]), 1)
        configs["lsa_t64k"] = lsa_line
        torch.cuda.empty_cache()

    line = {
        "metric": METRIC,
        "value": round(weak_scaling_value(world, K, wl.T, pre_ms), 1),
        "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(all_ms / K, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8-e4m3 indexer (f32 accumulate), bf16 attention (f32 softmax)",
        "data": "synthetic",
        "config": headline_cfg,
        "roofline": roof,
        "stages": stages,
        "decode": decode,
        "configs": configs,
        "peaks": {"fp8_tflops_measured": round(fp8_peak, 1), "bf16_tflops": peaks["bf16_tflops"],
                  "hbm_gbs": peaks["hbm_gbs"], "source": peak_src},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--workload", default="two_stage_t64k",
                    help="two_stage_t64k (headline), another prefill workload, or lsa_t64k / lsa_t8k")
    ap.add_argument("--T", type=int, default=0, help="override the prefill length (profiling runs)")
    ap.add_argument("--decode-L", type=int, default=0, help="override the decode cache length (profiling runs)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the other configurations (16K, 1M, 64K flat, tiny) on the JSON line")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=4096, help="rows of the oracle baseline (about 4 ms each)")
    ap.add_argument("--ref-rows", type=int, default=12)
    ap.add_argument("--lsa-cpu-rows", type=int, default=2048, help="query rows of the LSA oracle baseline")
    ap.add_argument("--lsa-decode-batch", type=int, default=64, help="sequences of the LSA decode step")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_native(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
