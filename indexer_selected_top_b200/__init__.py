"""Python binding of libsa (include/sa.h): argument marshalling only.

Every step of the sparse-attention path runs in the CUDA library; this module
passes torch tensors' device pointers and the current CUDA stream through the
C ABI and turns status codes into exceptions. There is no fallback: if the
library is missing, importing the binding fails.

    import indexer_selected_top_b200 as sa
    idx = sa.topk(scores, k=64)                 # exact top-k of each row
    out, lse = sa.prefill(inp, k=2048, mode="two_stage")
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# SA_LIB may name another build of the same library (e.g. a tuning variant)
LIB_PATH = os.environ.get("SA_LIB") or os.path.join(_HERE, "libsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libsa.so not built ({LIB_PATH}); run python indexer_selected_top_b200/build.py")
_lib = ctypes.CDLL(LIB_PATH)

# ----------------------------------------------------------------- constants
SA_OK, SA_ERR_INVALID_ARGUMENT, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE_TOO_SMALL, SA_ERR_CUDA, SA_ERR_TIMEOUT, \
    SA_ERR_INTERNAL = range(7)
SA_BF16, SA_FP8_E4M3, SA_F32 = 0, 1, 2
SA_MODE_FLAT, SA_MODE_TWO_STAGE = 0, 1
SA_OP_INDEX_SCORES, SA_OP_TOPK, SA_OP_SPARSE_ATTN, SA_OP_PREFILL, SA_OP_DECODE = range(5)
SA_HOOK_NONE, SA_HOOK_THETA_POS_INF, SA_HOOK_THETA_NEG_INF, SA_HOOK_STALL_WAIT, SA_HOOK_ATTN_UNGROUPED, \
    SA_HOOK_THETA_RUNNING = range(6)

EXPORTS = ("sa_status_string", "sa_index_scores", "sa_topk", "sa_sparse_attn", "sa_prefill", "sa_decode",
           "sa_workspace_size", "sa_sparse_attn_decode_noalloc", "sa_quantize_rows_e4m3",
           "sa_expand_sinks_window", "sa_lsa_build_buckets", "sa_lsa_search", "sa_lsa_search_workspace_size", "sa_lsa_decode",
           "sa_lsa_decode_workspace_size", "sa_lsa_attention", "sa_lsa_attention_workspace_size",
           "sa_debug_errors", "sa_prefill_chunk_rows")


class IndexerIn(ctypes.Structure):
    _fields_ = [("n_q", ctypes.c_int32), ("n_k", ctypes.c_int32), ("q_pos0", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("d_idx", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("q", ctypes.c_void_p), ("q_scale", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("w", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("seq_lens", ctypes.c_void_p)]


class AttnIn(ctypes.Structure):
    _fields_ = [("n_q", ctypes.c_int32), ("n_k", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("softmax_scale", ctypes.c_float), ("q", ctypes.c_void_p),
                ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p), ("batch", ctypes.c_int32)]


class PrefillOpts(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int32), ("mode", ctypes.c_int), ("block_size", ctypes.c_int32),
                ("keep_blocks", ctypes.c_int32), ("chunk_rows", ctypes.c_int32), ("status", ctypes.c_void_p),
                ("test_hook", ctypes.c_int32), ("stage_events", ctypes.c_void_p), ("n_stage_events", ctypes.c_int32),
                ("flat_path", ctypes.c_int32)]


SA_FLAT_AUTO, SA_FLAT_TABLE, SA_FLAT_STREAM = 0, 1, 2
FLAT_PATHS = {"auto": SA_FLAT_AUTO, "table": SA_FLAT_TABLE, "stream": SA_FLAT_STREAM}


class DecodeOpts(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int32), ("status", ctypes.c_void_p), ("test_hook", ctypes.c_int32),
                ("stage_events", ctypes.c_void_p), ("n_stage_events", ctypes.c_int32), ("max_len", ctypes.c_int32)]


class LsaParams(ctypes.Structure):
    _fields_ = [("d_idx", ctypes.c_int32), ("n_pool", ctypes.c_int32), ("n_cluster", ctypes.c_int32),
                ("n_buckets", ctypes.c_int32), ("max_bucket_keys", ctypes.c_int32)]


class LsaSearchOpts(ctypes.Structure):
    _fields_ = [("p", ctypes.c_int32), ("k", ctypes.c_int32), ("n_sink", ctypes.c_int32),
                ("n_window", ctypes.c_int32), ("status", ctypes.c_void_p), ("regime", ctypes.c_int32),
                ("test_hook", ctypes.c_int32)]


SA_LSA_AUTO, SA_LSA_TABLE, SA_LSA_STREAM = 0, 1, 2
LSA_REGIMES = {"auto": SA_LSA_AUTO, "table": SA_LSA_TABLE, "stream": SA_LSA_STREAM}


PREFILL_STAGES = {"flat": ("indexer", "topk", "attention"),
                  "two_stage": ("pool", "stage1_indexer", "block_keep", "stage2_indexer", "topk", "attention")}
DECODE_STAGES = ("indexer", "topk", "attention")


class StageTimer:
    """torch.cuda.Events handed to the library: chunk c's stage i runs between
    events c * (n + 1) + i and c * (n + 1) + i + 1 (n stages). ms() sums each
    stage over the chunks (a prepared Prefill sizes its timer for all of its
    chunks)."""

    def __init__(self, names, chunks: int = 1):
        self.names = names
        self.chunks = max(1, chunks)
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range((len(names) + 1) * self.chunks)]
        for e in self.events:          # torch creates the CUDA event on first record
            e.record()
        self._arr = (ctypes.c_void_p * len(self.events))(*[e.cuda_event for e in self.events])

    @property
    def ptr(self):
        return ctypes.cast(self._arr, ctypes.c_void_p)

    def ms(self) -> dict:
        n = len(self.names) + 1
        return {name: sum(self.events[c * n + i].elapsed_time(self.events[c * n + i + 1])
                          for c in range(self.chunks)) for i, name in enumerate(self.names)}

    def total_ms(self) -> float:
        """First event to last: the whole call, every chunk."""
        return self.events[0].elapsed_time(self.events[-1])


_P = ctypes.c_void_p
_lib.sa_status_string.restype = ctypes.c_char_p
_lib.sa_status_string.argtypes = [ctypes.c_int]
_lib.sa_index_scores.argtypes = [ctypes.POINTER(IndexerIn), _P, ctypes.c_int64, _P, ctypes.c_size_t, _P]
_lib.sa_topk.argtypes = [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P, _P,
                         ctypes.c_size_t, _P]
_lib.sa_sparse_attn.argtypes = [ctypes.POINTER(AttnIn), _P, ctypes.c_int32, _P, _P, _P, ctypes.c_size_t, _P]
_lib.sa_prefill.argtypes = [ctypes.POINTER(IndexerIn), ctypes.POINTER(AttnIn), ctypes.POINTER(PrefillOpts), _P, _P,
                            _P, _P, ctypes.c_size_t, _P]
_lib.sa_decode.argtypes = [ctypes.POINTER(IndexerIn), ctypes.POINTER(AttnIn), ctypes.POINTER(DecodeOpts), _P, _P,
                           _P, _P, ctypes.c_size_t, _P]
_lib.sa_quantize_rows_e4m3.argtypes = [_P, ctypes.c_int, ctypes.c_int64, ctypes.c_int32, _P, _P, _P]
_lib.sa_expand_sinks_window.argtypes = [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int32, _P, _P]
_lib.sa_lsa_build_buckets.argtypes = [ctypes.POINTER(LsaParams), _P, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_int32, _P, _P, _P, _P, _P]
_lib.sa_lsa_search.argtypes = [ctypes.POINTER(LsaParams), ctypes.POINTER(LsaSearchOpts), _P, ctypes.c_int32,
                               ctypes.c_int32, _P, _P, _P, ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]
_lib.sa_lsa_search_workspace_size.argtypes = [ctypes.POINTER(LsaParams), ctypes.POINTER(LsaSearchOpts),
                                              ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                              ctypes.POINTER(ctypes.c_size_t)]
_lib.sa_lsa_decode.argtypes = [ctypes.POINTER(LsaParams), ctypes.POINTER(LsaSearchOpts), _P, ctypes.c_int32, _P,
                               _P, _P, ctypes.c_int32, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.sa_lsa_decode_workspace_size.argtypes = [ctypes.POINTER(LsaParams), ctypes.POINTER(LsaSearchOpts),
                                              ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
_lib.sa_lsa_attention.argtypes = [ctypes.POINTER(AttnIn), _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                  ctypes.c_int32, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.sa_lsa_attention_workspace_size.argtypes = [ctypes.POINTER(AttnIn), ctypes.c_int32, ctypes.c_int32,
                                                 ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
_lib.sa_debug_errors.argtypes = [_P, ctypes.c_int32]
_lib.sa_workspace_size.argtypes = [ctypes.c_int, ctypes.POINTER(IndexerIn), ctypes.POINTER(AttnIn), _P,
                                   ctypes.POINTER(ctypes.c_size_t)]
_lib.sa_sparse_attn_decode_noalloc.argtypes = [ctypes.POINTER(AttnIn), _P, ctypes.c_int32, _P, _P, _P]
_lib.sa_prefill_chunk_rows.argtypes = [ctypes.POINTER(IndexerIn), ctypes.POINTER(PrefillOpts),
                                       ctypes.POINTER(ctypes.c_int32)]
for _f in ("sa_index_scores", "sa_topk", "sa_sparse_attn", "sa_prefill", "sa_decode", "sa_workspace_size",
           "sa_sparse_attn_decode_noalloc", "sa_quantize_rows_e4m3", "sa_expand_sinks_window",
           "sa_lsa_build_buckets", "sa_lsa_search", "sa_lsa_search_workspace_size", "sa_lsa_decode",
           "sa_lsa_decode_workspace_size", "sa_lsa_attention", "sa_lsa_attention_workspace_size",
           "sa_debug_errors", "sa_prefill_chunk_rows"):
    getattr(_lib, _f).restype = ctypes.c_int


class SaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_lib.sa_status_string(code).decode()}")


def _check(code: int, where: str):
    if code != SA_OK:
        raise SaError(code, where)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def status_string(code: int) -> str:
    return _lib.sa_status_string(code).decode()


# ------------------------------------------------------------- descriptors
def indexer_in(q, q_scale, k, k_scale, w, q_pos0=0, seq_lens=None) -> IndexerIn:
    """q [n_q, H, d] (uint8 e4m3 bytes or bf16), k [n_k, d] (decode: q [B, H, d],
    k [B, L, d] with seq_lens [B] int32 or None)."""
    decode = k.dim() == 3
    dt = SA_FP8_E4M3 if q.dtype == torch.uint8 else SA_BF16
    return IndexerIn(n_q=q.shape[0], n_k=k.shape[-2], q_pos0=q_pos0, n_heads=q.shape[1], d_idx=q.shape[2], dtype=dt,
                     q=_ptr(q), q_scale=_ptr(q_scale), k=_ptr(k), k_scale=_ptr(k_scale), w=_ptr(w),
                     batch=k.shape[0] if decode else 0, seq_lens=_ptr(seq_lens))


def attn_in(Q, K, V, softmax_scale=0.0) -> AttnIn:
    """Q [n_q, Hq, dh] bf16, K/V [n_k, dh] (decode: [B, L, dh]) bf16."""
    decode = K.dim() == 3
    return AttnIn(n_q=Q.shape[0], n_k=K.shape[-2], n_q_heads=Q.shape[1], head_dim=Q.shape[2],
                  softmax_scale=softmax_scale, q=_ptr(Q), k_cache=_ptr(K), v_cache=_ptr(V),
                  batch=K.shape[0] if decode else 0)


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 256) + 256, dtype=torch.uint8, device=device)


def _aligned(ws: torch.Tensor) -> int:
    p = ws.data_ptr()
    return (p + 255) & ~255


def workspace_size(op: int, ind=None, att=None, opts=None) -> int:
    n = ctypes.c_size_t(0)
    o = None
    if isinstance(opts, int):
        o = ctypes.cast(ctypes.pointer(ctypes.c_int32(opts)), ctypes.c_void_p)
    elif opts is not None:
        o = ctypes.cast(ctypes.pointer(opts), ctypes.c_void_p)
    _check(_lib.sa_workspace_size(op, ctypes.byref(ind) if ind is not None else None,
                                  ctypes.byref(att) if att is not None else None, o, ctypes.byref(n)),
           "sa_workspace_size")
    return n.value


# ------------------------------------------------------------------- calls
def index_scores(q, q_scale, k, k_scale, w, q_pos0=0, out=None, stream=None):
    """Causal score table [n_q, n_k] fp32 (-inf where invisible)."""
    ind = indexer_in(q, q_scale, k, k_scale, w, q_pos0)
    if out is None:
        out = torch.empty((q.shape[0], k.shape[0]), dtype=torch.float32, device=q.device)
    _check(_lib.sa_index_scores(ctypes.byref(ind), _ptr(out), out.stride(0), None, 0, _stream(stream)),
           "sa_index_scores")
    return out


def topk(scores, k: int, q_pos0: int = 0, n_k=None, out=None, stream=None):
    """Exact top-k of each row over columns s <= q_pos0 + row (unspecified
    order within a row, -1 padded)."""
    n_q = scores.shape[0]
    n_k = scores.shape[1] if n_k is None else n_k
    if out is None:
        out = torch.empty((n_q, k), dtype=torch.int32, device=scores.device)
    _check(_lib.sa_topk(_ptr(scores), n_q, n_k, scores.stride(0), q_pos0, k, _ptr(out), None, 0, _stream(stream)),
           "sa_topk")
    return out


def sparse_attn(Q, K, V, idx, softmax_scale=0.0, out=None, lse=None, stream=None, want_lse=True):
    att = attn_in(Q, K, V, softmax_scale)
    k = idx.shape[1]
    if out is None:
        out = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty(Q.shape[:2], dtype=torch.float32, device=Q.device)
    nws = workspace_size(SA_OP_SPARSE_ATTN, att=att, opts=k)
    ws = _workspace(nws, Q.device)
    _check(_lib.sa_sparse_attn(ctypes.byref(att), _ptr(idx), k, _ptr(out), _ptr(lse), _aligned(ws), nws,
                               _stream(stream)), "sa_sparse_attn")
    return out, lse


def sparse_attn_decode_noalloc(Q, K, V, idx, softmax_scale=0.0, out=None, lse=None, stream=None):
    """Decode attention (K/V [B, L, dh]) that takes no workspace: for callers
    that cannot allocate device memory around the call (see sa.h)."""
    att = attn_in(Q, K, V, softmax_scale)
    if out is None:
        out = torch.empty_like(Q)
    if lse is None:
        lse = torch.empty(Q.shape[:2], dtype=torch.float32, device=Q.device)
    _check(_lib.sa_sparse_attn_decode_noalloc(ctypes.byref(att), _ptr(idx), idx.shape[1], _ptr(out), _ptr(lse),
                                              _stream(stream)), "sa_sparse_attn_decode_noalloc")
    return out, lse


class Prefill:
    """A prepared sa_prefill call: descriptors and workspace built once, so a
    timed loop runs only the library call."""

    def __init__(self, q, q_scale, k, k_scale, w, Q, K, V, k_top: int, mode: str = "flat", block_size=64,
                 keep_blocks=64, chunk_rows=0, q_pos0=0, softmax_scale=0.0, want_idx=True, want_lse=True,
                 status=None, test_hook=0, timer: "StageTimer" = None, flat_path: str = "auto",
                 timed: bool = False):
        """timed=True: the call records its stages on a StageTimer of its
        own (self.timer), sized for every chunk; or pass `timer`."""
        self.ind = indexer_in(q, q_scale, k, k_scale, w, q_pos0)
        self.att = attn_in(Q, K, V, softmax_scale)
        self.opts = PrefillOpts(k=k_top, mode=SA_MODE_TWO_STAGE if mode == "two_stage" else SA_MODE_FLAT,
                                block_size=block_size, keep_blocks=keep_blocks, chunk_rows=chunk_rows,
                                status=_ptr(status), test_hook=test_hook, flat_path=FLAT_PATHS[flat_path])
        rows = ctypes.c_int32(0)
        _check(_lib.sa_prefill_chunk_rows(ctypes.byref(self.ind), ctypes.byref(self.opts), ctypes.byref(rows)),
               "sa_prefill_chunk_rows")
        self.chunk_rows = rows.value
        self.chunks = -(-q.shape[0] // max(rows.value, 1))
        if timed and timer is None:
            timer = StageTimer(PREFILL_STAGES[mode], self.chunks)
        if timer is not None:
            self.opts.stage_events = timer.ptr
            self.opts.n_stage_events = len(timer.events)
        self.timer = timer
        self.nws = workspace_size(SA_OP_PREFILL, self.ind, self.att, self.opts)
        self.ws = _workspace(self.nws, Q.device)
        self.idx = torch.empty((Q.shape[0], k_top), dtype=torch.int32, device=Q.device) if want_idx else None
        self.out = torch.empty_like(Q)
        self.lse = torch.empty(Q.shape[:2], dtype=torch.float32, device=Q.device) if want_lse else None
        self._keep = (q, q_scale, k, k_scale, w, Q, K, V, status)

    def __call__(self, stream=None):
        _check(_lib.sa_prefill(ctypes.byref(self.ind), ctypes.byref(self.att), ctypes.byref(self.opts),
                               _ptr(self.idx), _ptr(self.out), _ptr(self.lse), _aligned(self.ws), self.nws,
                               _stream(stream)), "sa_prefill")
        return self.out, self.lse, self.idx


def prefill(q, q_scale, k, k_scale, w, Q, K, V, k_top: int, mode: str = "flat", **kw):
    return Prefill(q, q_scale, k, k_scale, w, Q, K, V, k_top, mode, **kw)()


class Decode:
    """A prepared sa_decode call (one decode step of a batch of sequences)."""

    def __init__(self, q, q_scale, k, k_scale, w, Q, K, V, seq_lens, k_top: int, softmax_scale=0.0,
                 want_idx=True, want_lse=True, status=None, test_hook=0, timer: "StageTimer" = None,
                 max_len: int = 0):
        """max_len: 0, or the longest context the calls serve (sa_decode_opts.max_len)."""
        self.ind = indexer_in(q, q_scale, k, k_scale, w, 0, seq_lens)
        self.att = attn_in(Q, K, V, softmax_scale)
        self.opts = DecodeOpts(k=k_top, status=_ptr(status), test_hook=test_hook,
                               stage_events=timer.ptr if timer else None,
                               n_stage_events=len(timer.events) if timer else 0, max_len=max_len)
        self.timer = timer
        self.nws = workspace_size(SA_OP_DECODE, self.ind, self.att, self.opts)
        self.ws = _workspace(self.nws, Q.device)
        self.idx = torch.empty((Q.shape[0], k_top), dtype=torch.int32, device=Q.device) if want_idx else None
        self.out = torch.empty_like(Q)
        self.lse = torch.empty(Q.shape[:2], dtype=torch.float32, device=Q.device) if want_lse else None
        self._keep = (q, q_scale, k, k_scale, w, Q, K, V, seq_lens, status)

    def __call__(self, stream=None):
        _check(_lib.sa_decode(ctypes.byref(self.ind), ctypes.byref(self.att), ctypes.byref(self.opts),
                              _ptr(self.idx), _ptr(self.out), _ptr(self.lse), _aligned(self.ws), self.nws,
                              _stream(stream)), "sa_decode")
        return self.out, self.lse, self.idx

    def graph(self, max_len: int = None) -> "torch.cuda.CUDAGraph":
        """This decode step captured as a CUDA graph. The step launches no
        host synchronisation and no allocation, so every replay reruns it on the
        same buffers (write the next token's inputs into them between replays).
        max_len (default: the call's own) bounds the contexts the graph serves.
        The stage timer, if any, is not recorded by the graph."""
        ml = self.opts.max_len if max_len is None else max_len
        opts, self.opts = self.opts, DecodeOpts(k=self.opts.k, status=self.opts.status,
                                                test_hook=self.opts.test_hook, stage_events=None, n_stage_events=0,
                                                max_len=ml)
        try:
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                self(s)                       # one eager run: first-launch setup stays out of the graph
            torch.cuda.current_stream().wait_stream(s)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                self(s)
        finally:
            self.opts = opts
        return g


def context_buckets(capacity: int, smallest: int = 4096):
    """Context-length bounds of the decode graphs: ceil(1.125 * 2^e) rounded
    up to whole 128-key tiles for every e whose bound is at least `smallest`
    and below `capacity`, then `capacity` (the pages capture their decode
    graphs for context ranges of this form, LSA appendix F.1 "CUDA graphs")."""
    out, e = [], 0
    while True:
        b = -(-(9 << e) // 8)
        b = -(-b // 128) * 128
        if b >= capacity:
            break
        if b >= smallest:
            out.append(b)
        e += 1
    return out + [capacity]


class DecodeGraphs:
    """One CUDA graph of a prepared Decode per context-length bucket
    (context_buckets). replay(longest) replays the graph of the narrowest
    bucket that holds the batch's longest sequence, so a step over short
    contexts launches grids sized for them. Graphs are captured on first use
    (after one eager run of that bucket); inputs are read from the Decode's
    tensors at every replay."""

    def __init__(self, dec: Decode, capacity: int, smallest: int = 4096):
        self.dec = dec
        self.buckets = context_buckets(capacity, smallest)
        self.graphs = {}

    def bucket(self, longest: int) -> int:
        for b in self.buckets:
            if longest <= b:
                return b
        raise ValueError(f"context {longest} beyond the capacity {self.buckets[-1]}")

    def replay(self, longest: int) -> int:
        b = self.bucket(longest)
        g = self.graphs.get(b)
        if g is None:
            g = self.graphs[b] = self.dec.graph(max_len=b)
        g.replay()
        return b


def decode(q, q_scale, k, k_scale, w, Q, K, V, seq_lens, k_top: int, **kw):
    return Decode(q, q_scale, k, k_scale, w, Q, K, V, seq_lens, k_top, **kw)()


def quantize_rows_e4m3(x: torch.Tensor):
    """Per-row FP8 e4m3 encoding on the device (sa_quantize_rows_e4m3):
    returns (uint8 bytes shaped like x, fp32 scale per row)."""
    if x.dtype not in (torch.float32, torch.bfloat16) or not x.is_cuda or x.dim() < 1:
        raise ValueError("x: a CUDA float32 or bfloat16 tensor")
    x = x.contiguous()
    d = x.shape[-1]
    n = x.numel() // max(d, 1)
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _check(_lib.sa_quantize_rows_e4m3(_ptr(x), SA_F32 if x.dtype == torch.float32 else SA_BF16, n, d, _ptr(out),
                                      _ptr(scale), _stream()), "sa_quantize_rows_e4m3")
    return out, scale


def expand_sinks_window(idx: torch.Tensor, q_pos0: int, n_sink: int, n_window: int) -> torch.Tensor:
    """Served index rows (sa_expand_sinks_window): per row the sinks, the local
    window and the selected keys neither covers, -1 padded to
    n_sink + n_window + k columns."""
    if idx.dtype != torch.int32 or not idx.is_cuda or idx.dim() != 2:
        raise ValueError("idx: a CUDA int32 tensor [n_q, k]")
    idx = idx.contiguous()
    n_q, k = idx.shape
    out = torch.empty((n_q, n_sink + n_window + k), dtype=torch.int32, device=idx.device)
    _check(_lib.sa_expand_sinks_window(_ptr(idx), n_q, k, q_pos0, n_sink, n_window, _ptr(out), _stream()),
           "sa_expand_sinks_window")
    return out


# ------------------------------------------------- LSA flat semantic search
def lsa_params(n_pool: int = 4, n_cluster: int = 512, n_buckets: int = 64, max_bucket_keys: int = 32,
               d_idx: int = 64) -> LsaParams:
    """Clustering parameters of the bucket cache (sa_lsa_params)."""
    return LsaParams(d_idx=d_idx, n_pool=n_pool, n_cluster=n_cluster, n_buckets=n_buckets,
                     max_bucket_keys=max_bucket_keys)


def lsa_build_buckets(k_idx: torch.Tensor, prm: LsaParams, n_blocks: int = None, block0: int = 0, out=None,
                      status: torch.Tensor = None):
    """Bucket cache of cluster blocks [block0, block0 + n_blocks) of the bf16
    index keys k_idx [n_k, d_idx] (sa_lsa_build_buckets). Returns (centroids
    bf16 [nb * m, d], bucket_off int32 [nb * m], bucket_keys int32
    [nb * n_cluster]) with nb = block0 + n_blocks; `out` may pass those three
    tensors to add blocks to an existing cache."""
    if k_idx.dtype != torch.bfloat16 or not k_idx.is_cuda or k_idx.dim() != 2:
        raise ValueError("k_idx: a CUDA bfloat16 tensor [n_k, d_idx]")
    k_idx = k_idx.contiguous()
    if n_blocks is None:
        n_blocks = k_idx.shape[0] // prm.n_cluster - block0
    nb = block0 + n_blocks
    if out is None:
        dev = k_idx.device
        out = (torch.zeros((nb * prm.n_buckets, k_idx.shape[1]), dtype=torch.bfloat16, device=dev),
               torch.zeros(nb * prm.n_buckets, dtype=torch.int32, device=dev),
               torch.zeros(nb * prm.n_cluster, dtype=torch.int32, device=dev))
    cent, off, keys = out
    _check(_lib.sa_lsa_build_buckets(ctypes.byref(prm), _ptr(k_idx), k_idx.shape[0], block0, n_blocks, _ptr(cent),
                                     _ptr(off), _ptr(keys), _ptr(status), _stream()), "sa_lsa_build_buckets")
    return cent, off, keys


def lsa_search(q_idx: torch.Tensor, prm: LsaParams, buckets, n_blocks: int, q_pos0: int, p: int, k: int,
               n_sink: int = 0, n_window: int = 0, status: torch.Tensor = None, regime: str = "auto",
               test_hook: int = 0) -> torch.Tensor:
    """Index rows J [n_q, n_sink + n_window + k] int32 of the bf16 index
    queries q_idx [n_q, d_idx] at positions q_pos0 + i over a bucket cache
    from lsa_build_buckets holding n_blocks cluster blocks (sa_lsa_search).
    regime: "auto", "table" (bucket scores written) or "stream" (threshold
    scan, no score matrix)."""
    if q_idx.dtype != torch.bfloat16 or not q_idx.is_cuda or q_idx.dim() != 2:
        raise ValueError("q_idx: a CUDA bfloat16 tensor [n_q, d_idx]")
    q_idx = q_idx.contiguous()
    cent, off, keys = buckets
    o = LsaSearchOpts(p=p, k=k, n_sink=n_sink, n_window=n_window, status=_ptr(status), regime=LSA_REGIMES[regime],
                      test_hook=test_hook)
    n_q = q_idx.shape[0]
    nbytes = ctypes.c_size_t(0)
    _check(_lib.sa_lsa_search_workspace_size(ctypes.byref(prm), ctypes.byref(o), n_q, q_pos0, n_blocks,
                                             ctypes.byref(nbytes)), "sa_lsa_search_workspace_size")
    ws = _workspace(nbytes.value, q_idx.device)
    J = torch.empty((n_q, n_sink + n_window + k), dtype=torch.int32, device=q_idx.device)
    _check(_lib.sa_lsa_search(ctypes.byref(prm), ctypes.byref(o), _ptr(q_idx), n_q, q_pos0, _ptr(cent), _ptr(off),
                              _ptr(keys), n_blocks, _ptr(J), _aligned(ws), nbytes.value, _stream()),
           "sa_lsa_search")
    return J


class LsaPrefill:
    """A prepared LSA flat prefill of one sequence: the bucket cache of its
    complete cluster blocks (sa_lsa_build_buckets), the index rows of every
    query (sa_lsa_search) and attention over them (sa_lsa_attention, or
    sa_sparse_attn for shapes it does not take). Buffers
    and workspaces are allocated once; stage i of a call runs between the
    timer's events i and i + 1 (stages: cluster, search, attention). Each
    stage reports to its own row of `stage_status` ([3, 4] int32 on the
    device, sa_device_status words), which every call rewrites."""

    STAGES = ("cluster", "search", "attention")

    def __init__(self, k_idx, q_idx, Q, K, V, prm: LsaParams, p: int, k: int, n_sink: int = 4,
                 n_window: int = 512, softmax_scale: float = 0.0, timer: "StageTimer" = None,
                 regime: str = "auto"):
        dev = Q.device
        self.stage_status = torch.zeros((3, 4), dtype=torch.int32, device=dev)
        status = self.stage_status[1]
        self.k_idx, self.q_idx = k_idx.contiguous(), q_idx.contiguous()
        self.prm = prm
        T = self.k_idx.shape[0]
        self.n_blocks = T // prm.n_cluster
        nb = self.n_blocks
        self.cache = (torch.zeros((nb * prm.n_buckets, self.k_idx.shape[1]), dtype=torch.bfloat16, device=dev),
                      torch.zeros(nb * prm.n_buckets, dtype=torch.int32, device=dev),
                      torch.zeros(nb * prm.n_cluster, dtype=torch.int32, device=dev))
        self.opts = LsaSearchOpts(p=p, k=k, n_sink=n_sink, n_window=n_window, status=_ptr(status),
                                  regime=LSA_REGIMES[regime], test_hook=0)
        n = ctypes.c_size_t(0)
        _check(_lib.sa_lsa_search_workspace_size(ctypes.byref(prm), ctypes.byref(self.opts), self.q_idx.shape[0],
                                                 0, nb, ctypes.byref(n)), "sa_lsa_search_workspace_size")
        self.nws = n.value
        self.ws = _workspace(self.nws, dev)
        self.J = torch.empty((self.q_idx.shape[0], n_sink + n_window + k), dtype=torch.int32, device=dev)
        self.attn = LsaAttention(Q, K, V, self.J, 0, n_sink, n_window, softmax_scale, self.stage_status[2])
        self.out, self.lse = self.attn.out, self.attn.lse
        self.timer = timer
        self._keep = (Q, K, V)

    def __call__(self, stream=None):
        st = _stream(stream)
        ev = self.timer.events if self.timer else None
        ts = (torch.cuda.current_stream() if stream is None else stream) if ev else None
        cent, off, keys = self.cache
        if ev:
            ev[0].record(ts)
        _check(_lib.sa_lsa_build_buckets(ctypes.byref(self.prm), _ptr(self.k_idx), self.k_idx.shape[0], 0,
                                         self.n_blocks, _ptr(cent), _ptr(off), _ptr(keys),
                                         _ptr(self.stage_status[0]), st), "sa_lsa_build_buckets")
        if ev:
            ev[1].record(ts)
        _check(_lib.sa_lsa_search(ctypes.byref(self.prm), ctypes.byref(self.opts), _ptr(self.q_idx),
                                  self.q_idx.shape[0], 0, _ptr(cent), _ptr(off), _ptr(keys), self.n_blocks,
                                  _ptr(self.J), _aligned(self.ws), self.nws, st), "sa_lsa_search")
        if ev:
            ev[2].record(ts)
        self.attn(stream)
        if ev:
            ev[3].record(ts)
        return self.out, self.lse


class LsaDecode:
    """A prepared LSA decode step (sa_lsa_decode) for `batch` sequences with
    per-sequence bucket caches: centroids [batch, max_blocks * m, 64] bf16,
    bucket_off [batch, max_blocks * m] and bucket_keys [batch, max_blocks *
    n_cluster] int32 (each slab as lsa_build_buckets writes it for that
    sequence), n_blocks and seq_lens [batch] int32 on the device. Inputs are
    read from the tensors given here at every call, so a captured graph
    (graph()) replays over whatever they hold."""

    def __init__(self, q_idx, prm: LsaParams, caches, n_blocks, seq_lens, p: int, k: int, n_sink: int = 4,
                 n_window: int = 512, status=None):
        self.q_idx, self.prm = q_idx, prm
        self.cent, self.off, self.keys = caches
        self.batch = q_idx.shape[0]
        self.max_blocks = self.off.shape[1] // prm.n_buckets
        self.n_blocks, self.seq_lens = n_blocks, seq_lens
        self.opts = LsaSearchOpts(p=p, k=k, n_sink=n_sink, n_window=n_window, status=_ptr(status))
        n = ctypes.c_size_t(0)
        _check(_lib.sa_lsa_decode_workspace_size(ctypes.byref(prm), ctypes.byref(self.opts), self.batch,
                                                 self.max_blocks, ctypes.byref(n)), "sa_lsa_decode_workspace_size")
        self.nws = n.value
        self.ws = _workspace(self.nws, q_idx.device)
        self.J = torch.empty((self.batch, n_sink + n_window + k), dtype=torch.int32, device=q_idx.device)
        self.status = status

    def __call__(self, stream=None):
        _check(_lib.sa_lsa_decode(ctypes.byref(self.prm), ctypes.byref(self.opts), _ptr(self.q_idx), self.batch,
                                  _ptr(self.cent), _ptr(self.off), _ptr(self.keys), self.max_blocks,
                                  _ptr(self.n_blocks), _ptr(self.seq_lens), _ptr(self.J), _aligned(self.ws),
                                  self.nws, _stream(stream)), "sa_lsa_decode")
        return self.J

    def graph(self) -> "torch.cuda.CUDAGraph":
        """The step captured as a CUDA graph, after one eager run (first-launch
        setup stays out of the graph); every replay reruns it on the same
        buffers."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self(s)
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            self(s)
        return g


class LsaAttention:
    """A prepared sa_lsa_attention call over index rows J [n_q, width] from
    lsa_search (same q_pos0, n_sink, n_window): the sinks and windows of
    consecutive queries and the long-range keys of queries grouped by overlap,
    on the tensor cores, merged by log-sum-exp. `supported` is False for shapes
    the tensor-core kernel does not take; calls then run sa_sparse_attn (the
    per-query kernel) over the same rows."""

    def __init__(self, Q, K, V, J, q_pos0: int = 0, n_sink: int = 4, n_window: int = 512,
                 softmax_scale: float = 0.0, status=None):
        self.att = attn_in(Q, K, V, softmax_scale)
        self.J, self.q_pos0, self.n_sink, self.n_window = J, q_pos0, n_sink, n_window
        self.width = J.shape[1]
        n = ctypes.c_size_t(0)
        code = _lib.sa_lsa_attention_workspace_size(ctypes.byref(self.att), self.width, q_pos0, n_sink, n_window,
                                                    ctypes.byref(n))
        self.supported = code == SA_OK
        if code not in (SA_OK, SA_ERR_UNSUPPORTED):
            _check(code, "sa_lsa_attention_workspace_size")
        if not self.supported:
            n.value = workspace_size(SA_OP_SPARSE_ATTN, att=self.att, opts=self.width)
        self.nws = n.value
        self.ws = _workspace(self.nws, Q.device)
        self.out = torch.empty_like(Q)
        self.lse = torch.empty(Q.shape[:2], dtype=torch.float32, device=Q.device)
        self.status = status
        self._keep = (Q, K, V)

    def __call__(self, stream=None):
        if self.supported:
            _check(_lib.sa_lsa_attention(ctypes.byref(self.att), _ptr(self.J), self.width, self.q_pos0,
                                         self.n_sink, self.n_window, _ptr(self.out), _ptr(self.lse),
                                         _ptr(self.status), _aligned(self.ws), self.nws, _stream(stream)),
                   "sa_lsa_attention")
        else:
            _check(_lib.sa_sparse_attn(ctypes.byref(self.att), _ptr(self.J), self.width, _ptr(self.out),
                                       _ptr(self.lse), _aligned(self.ws), self.nws, _stream(stream)),
                   "sa_sparse_attn")
        return self.out, self.lse


def lsa_attention(Q, K, V, J, q_pos0: int = 0, n_sink: int = 4, n_window: int = 512, softmax_scale: float = 0.0,
                  status=None):
    """Attention over LSA index rows (sa_lsa_attention; the per-query kernel
    for shapes it does not take). Returns (out, lse)."""
    return LsaAttention(Q, K, V, J, q_pos0, n_sink, n_window, softmax_scale, status)()


DEBUG_SITES = {1: "attention index beyond the cache", 2: "two-stage group union beyond its list",
               3: "LSA bucket the query cannot see", 4: "LSA long-range key outside [0, position]",
               5: "LSA long-range union beyond its list", 6: "LSA bucket list entry outside its block"}


def debug_errors(reset: bool = True):
    """The debug build's record of failed invariant checks (sa_debug_errors):
    None when nothing failed, else (site name, value, count). Raises SaError
    with SA_ERR_UNSUPPORTED on a release build."""
    out = (ctypes.c_uint32 * 4)()
    _check(_lib.sa_debug_errors(ctypes.cast(out, ctypes.c_void_p), 1 if reset else 0), "sa_debug_errors")
    if out[0] == 0:
        return None
    return DEBUG_SITES.get(out[0], str(out[0])), out[1], out[2]


def new_status(device) -> torch.Tensor:
    """A zeroed device sa_device_status (4 x uint32, as int32)."""
    return torch.zeros(4, dtype=torch.int32, device=device)
