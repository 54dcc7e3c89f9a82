"""Plain fp64 CPU oracle of RTPurbo's head-wise sparse attention layer.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import or run this module; the library's product path
never does.  It shares no code with the CUDA kernels.  Its only common input
with them is the seeded generator in `synth/`, which holds none of the layer's
arithmetic.

What it computes (sources are the scraped pages on "Full Attention Strikes
Back: Transferring Full Attention into Sparse within Hundred Training Steps",
arXiv 2605.16928):

* Head split: only a small subset of heads needs full long context
  (abstract, observation (1); Daily Paper Cast episode page and the OpenAlex
  record).  Retrieval heads keep the full KV cache; local heads attend to
  attention sinks plus a sliding window (atlas.scime.ai summary, "Approach").
* Retrieval heads pick tokens with a 16-dimensional indexer (abstract,
  observation (2)) built on a pre-RoPE low-dimensional projection
  (atlas.scime.ai summary, "Approach" and the one-line summary above
  "Problem"):  q~ = W_q q_pre,  k~ = W_k k_pre,  score = q~ . k~ / 4
  (1/sqrt(16)).  The pages' dimension ablation also runs other widths
  (atlas "Surprising findings": dimension 4); at width d the score is
  q~ . k~ / sqrt(d) (the reading that keeps d = 16 as above).
* The token budget is query-dependent: a top-p threshold rather than a fixed
  top-k (abstract, observation (3); atlas "Approach": "query-adaptive top-p
  threshold").  Reading used here: P = softmax of the scores over every
  cached token the query may see; keep the shortest prefix of the tokens
  ordered by (P descending, index ascending) whose cumulative P reaches p
  (>= p); p >= 1 keeps everything.  Sinks and window are always added to the
  kept set (union after the top-p choice).
* Static top-k (the pages' ablation baseline, atlas "Key results" and
  "Baselines"): when the layer asks for a fixed k, the k highest scores (ties
  to the lower index) replace the top-p set.
* Attention itself is exact softmax attention with RoPE (rotate-half, angle
  pos * base^(-2k/D)) and scale 1/sqrt(D), over only the kept rows.

Precision: everything is fp64.  The caches are modelled with the storage
precision the layer stores them in (bf16, or fp32 for fp32 layers): stored
keys are round(RoPE(k_pre)), stored indexer keys are round(W_k k_pre), with
round-to-nearest-even applied to the exact fp64 value.  Queries, indexer
queries, scores and probabilities are never rounded.

Parity pins live in tests/test_oracle_*.py: closed forms, brute-force subset
enumeration for the top-p rule, a textbook dense attention for the p = 1 /
window >= context reductions, and RoPE's relative-position identity.
"""

from __future__ import annotations

import math
from typing import Dict, Iterable, Optional, Sequence

import numpy as np

IDX_DIM = 16
INDEXER_SCALE = 0.25  # 1 / sqrt(16), the pages' width

_BF16_DROP = 45  # fp64 has 52 explicit mantissa bits, bf16 keeps 7


def _as_f64(x) -> np.ndarray:
    """Upcast numpy arrays or torch tensors (any float dtype, incl. bf16) to fp64."""
    if hasattr(x, "detach"):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def round_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 (ties to even), returned as fp64.

    Normal range: drop 45 mantissa bits with round-to-nearest-even on the bit
    pattern.  Below 2^-126 (bf16 subnormals) the spacing is 2^-133.
    """
    a = np.array(x, dtype=np.float64, copy=True)
    if not np.all(np.isfinite(a)):
        raise ValueError("round_bf16: non-finite input")
    tiny = np.abs(a) < 2.0 ** -126
    bits = a.view(np.uint64)
    one = np.uint64(1)
    drop = np.uint64(_BF16_DROP)
    lsb = (bits >> drop) & one
    bias = np.uint64((1 << (_BF16_DROP - 1)) - 1) + lsb
    mask = ~np.uint64((1 << _BF16_DROP) - 1)
    out = ((bits + bias) & mask).view(np.float64)
    if np.any(tiny):
        out = np.where(tiny, np.round(a * 2.0 ** 133) * 2.0 ** -133, out)
    return out


def round_storage(x, dtype: str) -> np.ndarray:
    """Round to the cache's storage precision ("bf16" or "fp32")."""
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "fp32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


def rope_inv_freq(head_dim: int, base: float) -> np.ndarray:
    """inv_freq_k = base^(-2k/D), k = 0 .. D/2-1."""
    k = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * k / head_dim)


def rope(x, pos, base: float) -> np.ndarray:
    """Rotate-half rotary embedding of x[..., D] at positions pos (broadcast over x[..., 0]).

    Pair (x_k, x_{k+D/2}) is rotated by angle pos * inv_freq_k:
      y_k       = x_k cos - x_{k+D/2} sin
      y_{k+D/2} = x_{k+D/2} cos + x_k sin
    """
    x = _as_f64(x)
    D = x.shape[-1]
    h = D // 2
    theta = np.asarray(pos, dtype=np.float64)[..., None] * rope_inv_freq(D, base)
    c, s = np.cos(theta), np.sin(theta)
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def indexer_project(x_pre, w) -> np.ndarray:
    """d-dim pre-RoPE projection:  w [d, D] applied to x_pre [..., D]."""
    return _as_f64(x_pre) @ _as_f64(w).T


def indexer_scores(q_idx, k_idx) -> np.ndarray:
    """score_j = q~ . k~_j / sqrt(d)  for k_idx [n, d], q_idx [d] (d = 16: / 4)."""
    q = _as_f64(q_idx)
    d = q.shape[-1]
    scale = INDEXER_SCALE if d == IDX_DIM else 1.0 / math.sqrt(d)
    return (_as_f64(k_idx) @ q) * scale


def top_p_set(scores, p: float) -> np.ndarray:
    """Smallest set whose softmax mass reaches p; ties to the lower index.

    Returns the kept token indices, ascending.
    """
    s = _as_f64(scores)
    n = s.shape[0]
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    if p >= 1.0:
        return np.arange(n, dtype=np.int64)
    w = np.exp(s - s.max())
    P = w / w.sum()
    order = np.lexsort((np.arange(n), -P))  # P descending, then index ascending
    cum = np.cumsum(P[order])
    k = min(int(np.searchsorted(cum, p, side="left")) + 1, n)
    return np.sort(order[:k]).astype(np.int64)


def top_k_set(scores, k: int) -> np.ndarray:
    """Static top-k, the pages' fixed-budget baseline (atlas.scime.ai summary,
    "Baselines: static top-k"): the k highest scores, ties to the lower index;
    every token when k >= n.  Returns the kept token indices, ascending."""
    s = _as_f64(scores)
    n = s.shape[0]
    order = np.lexsort((np.arange(n), -s))  # score descending, then index ascending
    return np.sort(order[:min(int(k), n)]).astype(np.int64)


def sink_window_set(i: int, n_sink: int, window: int) -> np.ndarray:
    """Sinks [0, S) and the window of the last W positions ending at i, both within [0, i]."""
    sinks = np.arange(min(n_sink, i + 1), dtype=np.int64)
    win = np.arange(max(0, i - window + 1), i + 1, dtype=np.int64)
    return np.union1d(sinks, win)


def attend(q, K, V) -> np.ndarray:
    """Exact softmax attention of one query over rows K, V (scale 1/sqrt(D))."""
    q, K, V = _as_f64(q), _as_f64(K), _as_f64(V)
    z = (K @ q) / math.sqrt(q.shape[-1])
    e = np.exp(z - z.max())
    return (e @ V) / e.sum()


class OracleCache:
    """The layer's cache as the oracle sees it.

    Holds the pre-RoPE keys and the values as given (bf16 / fp32 containers,
    converted to fp64 on read) and the stored d-dim indexer keys (fp64, rounded
    to the storage precision) for the retrieval KV heads.  A stored key row is
    round(RoPE(k_pre, pos)), produced when read.
    """

    def __init__(self, shape, max_ctx: int, k_store=None, v_store=None):
        self.shape = shape
        self.max_ctx = int(max_ctx)
        B, Hkv, D = shape.batch, shape.n_kv_heads, shape.head_dim
        self.k_pre = k_store  # [B, Lmax, Hkv, D]
        self.v = v_store
        d = int(getattr(shape, "idx_dim", IDX_DIM))
        self.kidx = np.full((B, shape.n_retrieval, self.max_ctx, d), np.nan)
        self.length = np.zeros(B, dtype=np.int64)

    # -- append ---------------------------------------------------------
    def append(self, k_pre, v, start_pos: Sequence[int], T: int, w_k, block: int = 1 << 15):
        """Append T tokens per sequence at positions start_pos[b] + t.

        k_pre, v: [B, T, Hkv, D].  The pre-RoPE keys and values are recorded
        as given and, for every retrieval KV head r, k~ = round(W_k^(r) k_pre)
        is stored.
        """
        sh = self.shape
        if self.k_pre is None:
            import torch  # container only
            dt = torch.bfloat16 if sh.dtype == "bf16" else torch.float32
            self.k_pre = torch.zeros((sh.batch, self.max_ctx, sh.n_kv_heads, sh.head_dim), dtype=dt)
            self.v = torch.zeros_like(self.k_pre)
        for b in range(sh.batch):
            s0 = int(start_pos[b])
            if s0 + T > self.max_ctx:
                raise ValueError("append past max_ctx")
            if self.k_pre is not k_pre:
                self.k_pre[b, s0:s0 + T] = k_pre[b, :T]
                self.v[b, s0:s0 + T] = v[b, :T]
            for r, h in enumerate(sh.retrieval):
                for t0 in range(0, T, block):
                    t1 = min(T, t0 + block)
                    ki = indexer_project(k_pre[b, t0:t1, h], w_k[r])
                    self.kidx[b, r, s0 + t0:s0 + t1] = round_storage(ki, sh.dtype)
            self.length[b] = max(self.length[b], s0 + T)

    def append_in_place(self, k_pre, v, seq_len, w_k):
        """Adopt k_pre/v [B, Lmax, Hkv, D] as the whole context (rows [0, seq_len[b]))."""
        self.k_pre, self.v = k_pre, v
        sh = self.shape
        for b in range(sh.batch):
            L = int(seq_len[b])
            for r, h in enumerate(sh.retrieval):
                for t0 in range(0, L, 1 << 15):
                    t1 = min(L, t0 + (1 << 15))
                    ki = indexer_project(k_pre[b, t0:t1, h], w_k[r])
                    self.kidx[b, r, t0:t1] = round_storage(ki, sh.dtype)
            self.length[b] = L

    # -- reads ----------------------------------------------------------
    def keys(self, b: int, h: int, rows) -> np.ndarray:
        """Stored (RoPE'd, rounded) key rows."""
        rows = np.asarray(rows, dtype=np.int64)
        kp = _as_f64(self.k_pre[b, rows, h])
        return round_storage(rope(kp, rows, self.shape.rope_base), self.shape.dtype)

    def values(self, b: int, h: int, rows) -> np.ndarray:
        rows = np.asarray(rows, dtype=np.int64)
        return _as_f64(self.v[b, rows, h])

    def indexer_keys(self, b: int, r: int, n: int) -> np.ndarray:
        return self.kidx[b, r, :n]


def _row(cache: OracleCache, b: int, hq: int, i: int, q_pre_row, w_q, p: float,
         rows_override: Optional[Dict] = None):
    """One query (sequence b, q head hq, position i) over context [0, i]."""
    sh = cache.shape
    G = sh.group
    h = hq // G
    q = rope(_as_f64(q_pre_row), i, sh.rope_base)
    sw = sink_window_set(i, sh.n_sink, sh.window)
    topp = None
    if h in sh.retrieval:
        r = sh.retrieval.index(h)
        q_idx = indexer_project(q_pre_row, w_q[r])
        s = indexer_scores(q_idx, cache.indexer_keys(b, r, i + 1))
        k_fixed = int(getattr(sh, "top_k", 0) or 0)
        topp = top_k_set(s, k_fixed) if k_fixed > 0 else top_p_set(s, p)
        rows = np.union1d(topp, sw)
    else:
        rows = sw
    if rows_override is not None and (b, hq) in rows_override:
        rows = np.asarray(rows_override[(b, hq)], dtype=np.int64)
    o = attend(q, cache.keys(b, h, rows), cache.values(b, h, rows))
    return o, topp, rows


def decode(cache: OracleCache, q_pre, seq_len, w_q, top_p: Optional[float] = None,
           rows_override: Optional[Dict] = None, heads: Optional[Iterable[int]] = None):
    """One decode step: query of sequence b sits at position seq_len[b] - 1
    (the token just appended) and sees [0, seq_len[b]).

    Returns out [B, Hq, D] (fp64), topp {(b, hq): kept indices} for retrieval
    heads and final {(b, hq): attended rows}.  `rows_override` replaces the
    attended row set of given (b, hq) (used to evaluate attention on another
    selection).
    """
    sh = cache.shape
    p = sh.top_p if top_p is None else top_p
    B, Hq, D = sh.batch, sh.n_q_heads, sh.head_dim
    out = np.zeros((B, Hq, D))
    topp, final = {}, {}
    hs = range(Hq) if heads is None else heads
    for b in range(B):
        i = int(seq_len[b]) - 1
        for hq in hs:
            o, t, rows = _row(cache, b, hq, i, q_pre[b, hq], w_q, p, rows_override)
            out[b, hq] = o
            final[(b, hq)] = rows
            if t is not None:
                topp[(b, hq)] = t
    return out, topp, final


def recall_of_rows(cache: OracleCache, b: int, hq: int, i: int, q_pre_row, rows) -> float:
    """Attention mass recall of an attended row set (atlas.scime.ai summary,
    "Experimental setup", metrics): the share of the full causal attention's
    softmax mass, over every position in [0, i], that `rows` carry."""
    sh = cache.shape
    h = hq // sh.group
    q = rope(_as_f64(q_pre_row), i, sh.rope_base)
    allr = np.arange(i + 1, dtype=np.int64)
    z = (cache.keys(b, h, allr) @ q) / math.sqrt(q.shape[-1])
    e = np.exp(z - z.max())
    return float(e[np.asarray(rows, dtype=np.int64)].sum() / e.sum())


def decode_recall(cache: OracleCache, q_pre, seq_len, final: Dict) -> Dict:
    """Recall of each retrieval query head's attended rows of a decode step
    (`final` as returned by decode: {(b, hq): rows})."""
    sh = cache.shape
    out = {}
    for (b, hq), rows in final.items():
        if hq // sh.group in sh.retrieval:
            out[(b, hq)] = recall_of_rows(cache, b, hq, int(seq_len[b]) - 1, q_pre[b, hq], rows)
    return out


def prefill(cache: OracleCache, q_pre, start_pos, w_q, rows: Optional[Sequence[int]] = None,
            top_p: Optional[float] = None, heads: Optional[Iterable[int]] = None,
            rows_override: Optional[Dict] = None):
    """Causal prefill chunk: query row t of sequence b sits at position
    start_pos[b] + t and sees [0, start_pos[b] + t].

    q_pre [B, T, Hq, D].  Returns out {(b, t): [Hq, D]}, topp {(b, t, hq): kept
    indices} for retrieval heads, over the requested rows (default: all).
    `rows_override` {(b, t, hq): rows} replaces the attended rows of a query.
    """
    sh = cache.shape
    p = sh.top_p if top_p is None else top_p
    T = q_pre.shape[1]
    rows = range(T) if rows is None else rows
    hs = list(range(sh.n_q_heads)) if heads is None else list(heads)
    out, topp = {}, {}
    for b in range(sh.batch):
        for t in rows:
            i = int(start_pos[b]) + int(t)
            o_bt = np.zeros((sh.n_q_heads, sh.head_dim))
            for hq in hs:
                ov = None
                if rows_override is not None and (b, int(t), hq) in rows_override:
                    ov = {(b, hq): rows_override[(b, int(t), hq)]}
                o, tp, _ = _row(cache, b, hq, i, q_pre[b, t, hq], w_q, p, ov)
                o_bt[hq] = o
                if tp is not None:
                    topp[(b, int(t), hq)] = tp
            out[(b, int(t))] = o_bt
    return out, topp
