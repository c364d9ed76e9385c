"""Seeded synthetic inputs for learned top-k sparse attention.

This module only draws random numbers and lays them out in the input formats
of the sparse-attention library (FP8 e4m3 bytes with one fp32 scale per row,
or bf16). It holds none of the method's arithmetic: no scoring, no selection,
no attention. Both the oracle (CPU) and the CUDA path consume exactly the
tensors it returns; the oracle receives a host copy of the same bytes.

Workloads follow the shapes and value distributions of the five synthetic
configurations of the sparse-attention hot path (tiny causal prefill, 16K
prefill, 64 x 128K decode, 64K two-stage prefill, 1M prefill). They stand in
for the long-context evaluation data of the pages (RULER, PaperTrail), which
are not used here.

Planted keys ("relevant keys per query block"): queries form blocks of
``plant_block`` rows; block b draws a direction y_b ~ N(0, I_d). Each of its
index-query rows is sqrt(1 - rho^2) z + rho y_b with z ~ N(0, I) (marginally
still N(0, 1) per element), and ``n_plant`` keys at distinct positions drawn
uniformly in [0, block_end) are set to 0.8 sqrt(d) y_b/|y_b| + 0.2 N(0, I).

Topic keys (two-stage workload): 16 centroids c ~ N(0, I_d); keys come in
contiguous runs of 2048 tokens whose topic is uniform per run, k = c + 0.3 n;
query t picks a topic uniformly among those present in keys [0, t] and each of
its heads is c + 0.3 n.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill" or "decode"
    T: int                    # query rows (prefill) / unused for decode
    H: int                    # indexer heads
    d: int                    # index dimension d_idx
    idx_dtype: str            # "bf16" or "fp8"
    k: int                    # top-k budget
    Hq: int                   # attention query heads (one shared KV head)
    dh: int                   # attention head dim
    mode: str = "flat"        # "flat" or "two_stage"
    plant_block: int = 0      # queries per planted block (0 = none)
    n_plant: int = 0          # planted keys per block
    rho: float = 0.5
    batch: int = 0            # decode sequences
    L: int = 0                # decode cache length
    block_size: int = 64      # two-stage key block
    keep_blocks: int = 64     # two-stage kept blocks per query
    topics: int = 0           # two-stage topic clusters
    topic_run: int = 2048
    topic_sigma: float = 0.3
    attn_std: float = 0.0     # std of Q/K/V (0 = 1/sqrt(dh))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # Tiny causal prefill: bf16 indexer, H=4, d_idx=32, k=64, 8 heads x 64.
    "tiny_t512": Workload("tiny_t512", "prefill", T=512, H=4, d=32, idx_dtype="bf16",
                          k=64, Hq=8, dh=64, plant_block=64, n_plant=8),
    # 16K prefill: FP8 indexer, H=64, d_idx=128, k=2048, MQA 16 x 128.
    "prefill_t16k": Workload("prefill_t16k", "prefill", T=16384, H=64, d=128, idx_dtype="fp8",
                             k=2048, Hq=16, dh=128, plant_block=256, n_plant=32),
    # Decode: 64 sequences x 131072 cached keys.
    "decode_b64_l128k": Workload("decode_b64_l128k", "decode", T=1, H=64, d=128, idx_dtype="fp8",
                                 k=2048, Hq=16, dh=128, plant_block=1, n_plant=32,
                                 batch=64, L=131072),
    # Two-stage hierarchical prefill at 64K (the headline prefill workload).
    "two_stage_t64k": Workload("two_stage_t64k", "prefill", T=65536, H=64, d=128, idx_dtype="fp8",
                               k=2048, Hq=16, dh=128, mode="two_stage", topics=16),
    # 1M-token prefill, selection on the fly (no score table).
    "prefill_t1m": Workload("prefill_t1m", "prefill", T=1 << 20, H=64, d=128, idx_dtype="fp8",
                            k=2048, Hq=16, dh=128, plant_block=1024, n_plant=32),
}


# ----------------------------------------------------------------------------
# seeding: one independent stream per (seed, tensor, chunk)
# ----------------------------------------------------------------------------
_STREAMS = {"q": 1, "k": 2, "w": 3, "Q": 4, "K": 5, "V": 6, "dir": 7, "plant": 8,
            "pnoise": 9, "topic": 10, "centroid": 11, "qtopic": 12, "runs": 13}


def _mix(*vals: int) -> int:
    """splitmix64 over the arguments: a 63-bit seed for torch.Generator."""
    x = 0x9E3779B97F4A7C15
    for v in vals:
        x = (x ^ (v & 0xFFFFFFFFFFFFFFFF)) & 0xFFFFFFFFFFFFFFFF
        x = (x + 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
        z = x
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
        x = z ^ (z >> 31)
    return x & 0x7FFFFFFFFFFFFFFF


def _gen(device, seed: int, stream: str, chunk: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_mix(seed, _STREAMS[stream], chunk))
    return g


def _np_rng(seed: int, stream: str, chunk: int = 0) -> np.random.Generator:
    return np.random.default_rng(_mix(seed, _STREAMS[stream], chunk))


def quantize_rows_e4m3(x: torch.Tensor):
    """Per-row FP8 e4m3 encoding of the inputs: scale = amax/448 (1 for an
    all-zero row), bytes = e4m3(x / scale) after clamping to +-448 (torch's
    cast does not saturate). Returns (uint8 bytes, fp32 scale)."""
    x = x.float()
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (x / scale.unsqueeze(-1)).clamp(-E4M3_MAX, E4M3_MAX)
    return y.to(torch.float8_e4m3fn).view(torch.uint8), scale.contiguous()


def _randn(shape, gen, device):
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)


def _plant_positions(seed: int, n_blocks: int, plant_block: int, n_plant: int, n_keys: int,
                     T: int):
    """Distinct planted positions: block b draws n_plant positions uniformly in
    [0, min(block_end, n_keys)) not already planted by an earlier block."""
    rng = _np_rng(seed, "plant")
    taken = np.zeros(n_keys, dtype=bool)
    out = []
    for b in range(n_blocks):
        end = min((b + 1) * plant_block, n_keys) if plant_block > 0 else n_keys
        pos = []
        tries = 0
        while len(pos) < n_plant and tries < 100 * n_plant:
            s = int(rng.integers(0, end))
            tries += 1
            if not taken[s]:
                taken[s] = True
                pos.append(s)
        out.append(np.array(sorted(pos), dtype=np.int64))
    return out


class PrefillInputs:
    """Tensors of one prefill workload on one device (all row-major, contiguous).

    q_idx  [T, H, d]  uint8 (fp8 e4m3) or bf16      q_scale [T, H] fp32 (fp8 only)
    k_idx  [T, d]     uint8 or bf16                  k_scale [T]    fp32 (fp8 only)
    w      [T, H]     fp32, U(0, 1)
    Q      [T, Hq, dh] bf16; K, V [T, dh] bf16
    """

    def __init__(self, wl: Workload, device="cpu", seed: int = 0, chunk_rows: int = 32768):
        self.wl, self.device, self.seed = wl, torch.device(device), seed
        self.chunk_rows = chunk_rows
        T, H, d = wl.T, wl.H, wl.d
        dev = self.device
        self.n_k = T
        self.planted = None
        self.block_dir = None
        self.query_topic = None
        # --- index keys (fp32 before encoding) ---
        if wl.topics:
            self._make_topics()
        elif wl.plant_block:
            n_blocks = (T + wl.plant_block - 1) // wl.plant_block
            self.block_dir = _randn((n_blocks, d), _gen(dev, seed, "dir"), dev)
            self.planted = _plant_positions(seed, n_blocks, wl.plant_block, wl.n_plant, T, T)
        self.k_f32 = self._keys_f32()
        if wl.idx_dtype == "fp8":
            self.k_idx, self.k_scale = quantize_rows_e4m3(self.k_f32)
        else:
            self.k_idx, self.k_scale = self.k_f32.to(torch.bfloat16), None
        # --- index queries, chunked so the fp32 rows never all exist at once ---
        if wl.idx_dtype == "fp8":
            self.q_idx = torch.empty((T, H, d), dtype=torch.uint8, device=dev)
            self.q_scale = torch.empty((T, H), dtype=torch.float32, device=dev)
        else:
            self.q_idx = torch.empty((T, H, d), dtype=torch.bfloat16, device=dev)
            self.q_scale = None
        for c0 in range(0, T, chunk_rows):
            qf = self.q_f32_rows(c0, min(T, c0 + chunk_rows))
            if wl.idx_dtype == "fp8":
                b, s = quantize_rows_e4m3(qf)
                self.q_idx[c0:c0 + qf.shape[0]] = b
                self.q_scale[c0:c0 + qf.shape[0]] = s
            else:
                self.q_idx[c0:c0 + qf.shape[0]] = qf.to(torch.bfloat16)
            del qf
        self.w = torch.rand((T, H), generator=_gen(dev, seed, "w"), device=dev)
        # --- attention operands ---
        std = wl.attn_std or 1.0 / math.sqrt(wl.dh)
        self.Q = torch.empty((T, wl.Hq, wl.dh), dtype=torch.bfloat16, device=dev)
        for c0 in range(0, T, chunk_rows):
            n = min(T, c0 + chunk_rows) - c0
            self.Q[c0:c0 + n] = (_randn((n, wl.Hq, wl.dh), _gen(dev, seed, "Q", c0 // chunk_rows), dev)
                                 * std).to(torch.bfloat16)
        self.K = (_randn((T, wl.dh), _gen(dev, seed, "K"), dev) * std).to(torch.bfloat16)
        self.V = (_randn((T, wl.dh), _gen(dev, seed, "V"), dev) * std).to(torch.bfloat16)

    # ----- keys -----
    def _make_topics(self):
        wl, dev, seed = self.wl, self.device, self.seed
        T, d = wl.T, wl.d
        self.centroids = _randn((wl.topics, d), _gen(dev, seed, "centroid"), dev)
        n_runs = (T + wl.topic_run - 1) // wl.topic_run
        rng = _np_rng(seed, "topic")
        self.run_topic = rng.integers(0, wl.topics, size=n_runs)
        # query t: uniform among the topics present in runs 0..t // run
        rngq = _np_rng(seed, "qtopic")
        present = np.zeros(wl.topics, dtype=bool)
        qt = np.empty(T, dtype=np.int64)
        u = rngq.random(T)
        for r in range(n_runs):
            present[self.run_topic[r]] = True
            ids = np.flatnonzero(present)
            lo, hi = r * wl.topic_run, min(T, (r + 1) * wl.topic_run)
            qt[lo:hi] = ids[np.minimum((u[lo:hi] * len(ids)).astype(np.int64), len(ids) - 1)]
        self.query_topic = qt

    def _keys_f32(self):
        wl, dev, seed = self.wl, self.device, self.seed
        T, d = wl.T, wl.d
        noise = _randn((T, d), _gen(dev, seed, "k"), dev)
        if wl.topics:
            run_of_key = torch.arange(T, device=dev) // wl.topic_run
            topic = torch.as_tensor(self.run_topic, device=dev)[run_of_key]
            return self.centroids[topic] + wl.topic_sigma * noise
        if self.planted is not None:
            pn = _randn((T, d), _gen(dev, seed, "pnoise"), dev)
            unit = self.block_dir / self.block_dir.norm(dim=1, keepdim=True)
            for b, pos in enumerate(self.planted):
                if len(pos) == 0:
                    continue
                p = torch.as_tensor(pos, device=dev)
                noise[p] = 0.8 * math.sqrt(d) * unit[b] + 0.2 * pn[p]
        return noise

    def q_f32_rows(self, r0: int, r1: int) -> torch.Tensor:
        """Pre-encoding fp32 index queries of rows [r0, r1) (re-drawn from the
        same per-chunk streams; r0 must be a multiple of chunk_rows or r1 stay
        within one chunk)."""
        wl, dev, seed = self.wl, self.device, self.seed
        H, d, cr = wl.H, wl.d, self.chunk_rows
        c = r0 // cr
        if r1 > (c + 1) * cr:
            raise ValueError("q_f32_rows spans chunks")
        n_chunk = min(wl.T, (c + 1) * cr) - c * cr
        z = _randn((n_chunk, H, d), _gen(dev, seed, "q", c), dev)[r0 - c * cr:r1 - c * cr]
        rows = torch.arange(r0, r1, device=dev)
        if wl.topics:
            cen = self.centroids[torch.as_tensor(self.query_topic[r0:r1], device=dev)]
            return cen.unsqueeze(1) + wl.topic_sigma * z
        if self.block_dir is not None:
            y = self.block_dir[rows // wl.plant_block]
            rho = wl.rho
            return math.sqrt(1 - rho * rho) * z + rho * y.unsqueeze(1)
        return z

    def planted_for_row(self, t: int):
        if self.planted is None:
            return np.zeros(0, dtype=np.int64)
        pos = self.planted[t // self.wl.plant_block]
        return pos[pos <= t]

    def to_host(self) -> dict:
        """Host copies of every input (the oracle's view of the same bytes)."""
        out = {}
        for name in ("q_idx", "q_scale", "k_idx", "k_scale", "w", "Q", "K", "V"):
            v = getattr(self, name)
            out[name] = None if v is None else v.cpu()
        return out


class DecodeInputs:
    """One decode step for ``batch`` sequences, each with one new query over a
    cache of L keys (its own key is the cache's last row).

    q_idx [B, H, d] uint8, q_scale [B, H], w [B, H]
    k_idx [B, L, d] uint8, k_scale [B, L]
    Q [B, Hq, dh] bf16; K, V [B, L, dh] bf16; seq_lens [B] int32 (= L)
    """

    def __init__(self, wl: Workload, device="cpu", seed: int = 0):
        self.wl, self.device, self.seed = wl, torch.device(device), seed
        B, L, H, d = wl.batch, wl.L, wl.H, wl.d
        dev = self.device
        self.block_dir = _randn((B, d), _gen(dev, seed, "dir"), dev)
        unit = self.block_dir / self.block_dir.norm(dim=1, keepdim=True)
        rng = _np_rng(seed, "plant")
        self.planted = [np.sort(rng.choice(L, size=min(wl.n_plant, L), replace=False)) for _ in range(B)]
        k_idx = torch.empty((B, L, d), dtype=torch.uint8, device=dev)
        k_scale = torch.empty((B, L), dtype=torch.float32, device=dev)
        for b in range(B):
            kf = _randn((L, d), _gen(dev, seed, "k", b), dev)
            if len(self.planted[b]):
                p = torch.as_tensor(self.planted[b], device=dev)
                pn = _randn((len(self.planted[b]), d), _gen(dev, seed, "pnoise", b), dev)
                kf[p] = 0.8 * math.sqrt(d) * unit[b] + 0.2 * pn
            k_idx[b], k_scale[b] = quantize_rows_e4m3(kf)
            del kf
        self.k_idx, self.k_scale = k_idx, k_scale
        z = _randn((B, H, d), _gen(dev, seed, "q"), dev)
        rho = wl.rho
        qf = math.sqrt(1 - rho * rho) * z + rho * self.block_dir.unsqueeze(1)
        self.q_idx, self.q_scale = quantize_rows_e4m3(qf)
        self.w = torch.rand((B, H), generator=_gen(dev, seed, "w"), device=dev)
        std = wl.attn_std or 1.0 / math.sqrt(wl.dh)
        self.Q = (_randn((B, wl.Hq, wl.dh), _gen(dev, seed, "Q"), dev) * std).to(torch.bfloat16)
        self.K = torch.empty((B, L, wl.dh), dtype=torch.bfloat16, device=dev)
        self.V = torch.empty((B, L, wl.dh), dtype=torch.bfloat16, device=dev)
        for b in range(B):
            self.K[b] = (_randn((L, wl.dh), _gen(dev, seed, "K", b), dev) * std).to(torch.bfloat16)
            self.V[b] = (_randn((L, wl.dh), _gen(dev, seed, "V", b), dev) * std).to(torch.bfloat16)
        self.seq_lens = torch.full((B,), L, dtype=torch.int32, device=dev)

    def to_host(self) -> dict:
        out = {}
        for name in ("q_idx", "q_scale", "k_idx", "k_scale", "w", "Q", "K", "V", "seq_lens"):
            out[name] = getattr(self, name).cpu()
        return out


def sample_rows(T: int, n: int, seed: int, k: int, extra=(), block: Optional[int] = None):
    """Seeded, stratified query rows for sampled checks: always t in
    {0, 1, k-1, k, k+1, T-1} (and block edges if given), the rest spread over
    [0, T) in equal strata."""
    must = {0, 1, k - 1, k, k + 1, T - 1}
    for e in extra:
        must.add(e)
    must = sorted(x for x in must if 0 <= x < T)
    rng = np.random.default_rng(_mix(seed, 99))
    rest = max(0, n - len(must))
    edges = np.linspace(0, T, rest + 1).astype(np.int64)
    picks = [int(rng.integers(edges[i], max(edges[i] + 1, edges[i + 1]))) for i in range(rest)]
    rows = sorted(set(must) | set(min(T - 1, p) for p in picks))
    return np.array(rows, dtype=np.int64)


# ----------------------------------------------------------------------------
# LSA semantic-search workloads
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class LsaWorkload:
    """Index keys and queries of the LSA flat semantic search (one bf16 head
    of d_idx = 64), with the clustering and search parameters.

    Keys follow topics that change every few tokens: ``topics`` centroids c ~
    N(0, I_d); the sequence is cut into runs of geometric length (mean
    ``run_mean``), each run takes a uniform topic, and its keys are c +
    sigma N(0, I). The query at position t takes the topic of a uniformly drawn
    position in [0, t] and is c + sigma N(0, I). Values are rounded to bf16;
    normalisation is the method's own step, not the generator's."""
    name: str
    T: int
    d: int = 64
    n_pool: int = 4
    n_cluster: int = 512
    n_buckets: int = 64
    max_bucket_keys: int = 32
    p: int = 512
    k: int = 2048
    n_sink: int = 4
    n_window: int = 512
    topics: int = 256
    run_mean: int = 16
    sigma: float = 0.5
    Hq: int = 16
    dh: int = 128

    def with_(self, **kw) -> "LsaWorkload":
        return dataclasses.replace(self, **kw)


LSA_WORKLOADS = {
    # 8K tokens: 16 cluster blocks, 1,024 buckets; small enough for the oracle
    "lsa_t8k": LsaWorkload("lsa_t8k", T=8192, p=128, k=512, topics=64),
    # 64K tokens: 128 cluster blocks of 512 keys, 8,192 buckets of about 8 keys,
    # p = 512 buckets for k = 2048 long-range keys, 4 sinks, a 512-key window
    "lsa_t64k": LsaWorkload("lsa_t64k", T=65536),
}


class LsaInputs:
    """k_idx [T, d] and q_idx [T, d] bf16 index keys / queries; Q [T, Hq, dh],
    K, V [T, dh] bf16 attention operands (drawn on first use)."""

    def __init__(self, wl: LsaWorkload, device="cpu", seed: int = 0):
        self.wl, self.device, self.seed = wl, torch.device(device), seed
        T, d, dev = wl.T, wl.d, self.device
        rng = _np_rng(seed, "runs")
        topic = np.empty(T, dtype=np.int64)
        t = 0
        while t < T:
            n = int(rng.geometric(1.0 / wl.run_mean))
            topic[t:t + n] = rng.integers(0, wl.topics)
            t += n
        src = np.minimum((_np_rng(seed, "qtopic").random(T) * (np.arange(T) + 1)).astype(np.int64), np.arange(T))
        self.key_topic = topic
        self.query_topic = topic[src]
        cen = _randn((wl.topics, d), _gen(dev, seed, "centroid"), dev)
        kt = torch.as_tensor(topic, device=dev)
        qt = torch.as_tensor(self.query_topic, device=dev)
        self.k_idx = (cen[kt] + wl.sigma * _randn((T, d), _gen(dev, seed, "k"), dev)).to(torch.bfloat16)
        self.q_idx = (cen[qt] + wl.sigma * _randn((T, d), _gen(dev, seed, "q"), dev)).to(torch.bfloat16)
        self._attn = None

    def attention_operands(self):
        if self._attn is None:
            wl, dev, seed = self.wl, self.device, self.seed
            std = 1.0 / math.sqrt(wl.dh)
            Q = (_randn((wl.T, wl.Hq, wl.dh), _gen(dev, seed, "Q"), dev) * std).to(torch.bfloat16)
            K = (_randn((wl.T, wl.dh), _gen(dev, seed, "K"), dev) * std).to(torch.bfloat16)
            V = (_randn((wl.T, wl.dh), _gen(dev, seed, "V"), dev) * std).to(torch.bfloat16)
            self._attn = (Q, K, V)
        return self._attn
