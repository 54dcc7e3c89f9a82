"""Seeded synthetic inputs shaped like the layer-speed workloads of RTPurbo.

"Full Attention Strikes Back" (atlas.scime.ai summary, "Key results") measures
attention-layer prefill at 32K..1M tokens and decode at 1M tokens, but ships no
data.  The workloads below stand in for those: N(0,1) pre-RoPE queries, keys
and values, N(0, 1/D) indexer projections, and planted "needle" keys whose
16-d indexer key is aligned with a query's indexer direction and scaled by 4,
so that retrieval heads have something real to retrieve.

Everything here is input construction.  The needle planting solves a small
least-squares problem (minimum-norm correction of a key through the indexer
projection); it computes no score, softmax, selection, RoPE or attention.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np
import torch

IDX_DIM = 16


@dataclasses.dataclass(frozen=True)
class LayerShape:
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_sink: int
    window: int
    top_p: float
    retrieval: tuple
    dtype: str = "bf16"          # storage / IO dtype: "bf16" or "fp32"
    rope_base: float = 10000.0
    idx_dim: int = IDX_DIM
    top_k: int = 0               # > 0: static top-k selection instead of top-p

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_retrieval(self) -> int:
        return len(self.retrieval)

    @property
    def retrieval_mask(self) -> int:
        m = 0
        for h in self.retrieval:
            m |= 1 << h
        return m

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw) -> "LayerShape":
        return dataclasses.replace(self, **kw)


_QWEN8B = dict(n_q_heads=32, n_kv_heads=8, head_dim=128, retrieval=(0, 5), dtype="bf16")

# name -> workload description.  Sizes follow the pages' layer-speed settings
# (32K prefill chunk, 128K..1M decode) with a Qwen3-8B-shaped attention layer.
WORKLOADS: Dict[str, dict] = {
    "tiny_decode_2k_fp32": dict(
        kind="decode", seed=0, ctx=2048, needles=8,
        shape=LayerShape(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=64, n_sink=4, window=128,
                         top_p=0.9, retrieval=(0,), dtype="fp32")),
    "decode_128k_bf16": dict(
        kind="decode", seed=1, ctx=131072, needles=64,
        shape=LayerShape(batch=1, n_sink=64, window=2048, top_p=0.95, **_QWEN8B)),
    "ragged_decode_b8_8k_32k_bf16": dict(
        kind="decode", seed=2, ctx=(8192, 32768), needles=64,
        shape=LayerShape(batch=8, n_sink=64, window=2048, top_p=0.95, **_QWEN8B)),
    "prefill_32k_bf16": dict(
        kind="prefill", seed=3, ctx=32768, needles=256,
        shape=LayerShape(batch=1, n_sink=64, window=2048, top_p=0.95, **_QWEN8B)),
    "decode_1m_bf16": dict(
        kind="decode", seed=4, ctx=1048576, needles=1024,
        shape=LayerShape(batch=1, n_sink=64, window=4096, top_p=0.95, **_QWEN8B)),
}


def workload(name: str, **overrides) -> dict:
    """Return a copy of WORKLOADS[name]; `shape_*` keys override LayerShape fields."""
    w = dict(WORKLOADS[name])
    shape_kw = {k[6:]: v for k, v in overrides.items() if k.startswith("shape_")}
    other = {k: v for k, v in overrides.items() if not k.startswith("shape_")}
    if shape_kw:
        w["shape"] = w["shape"].replace(**shape_kw)
    w.update(other)
    w["name"] = name
    return w


def _randn(gen: torch.Generator, shape, dtype, block_rows: int = 1 << 16) -> torch.Tensor:
    """N(0,1) draws rounded (RNE) to `dtype`; drawn in fp32 blocks along dim 1."""
    out = torch.empty(shape, dtype=dtype)
    if len(shape) >= 2 and shape[1] > block_rows:
        for s in range(0, shape[1], block_rows):
            e = min(shape[1], s + block_rows)
            sub = list(shape)
            sub[1] = e - s
            out[:, s:e] = torch.randn(sub, generator=gen, dtype=torch.float32).to(dtype)
    else:
        out.copy_(torch.randn(shape, generator=gen, dtype=torch.float32).to(dtype))
    return out


def _projections(gen: torch.Generator, shape: LayerShape):
    D, R = shape.head_dim, shape.n_retrieval
    std = 1.0 / np.sqrt(D)
    w_q = (torch.randn((R, shape.idx_dim, D), generator=gen, dtype=torch.float32) * std).contiguous()
    w_k = (torch.randn((R, shape.idx_dim, D), generator=gen, dtype=torch.float32) * std).contiguous()
    return w_q, w_k


def _needle_positions(gen: torch.Generator, lo: int, hi: int, n: int) -> np.ndarray:
    """n distinct positions drawn uniformly from [lo, hi), sorted."""
    span = hi - lo
    n = min(n, max(span, 0))
    if n <= 0:
        return np.zeros(0, dtype=np.int64)
    perm = torch.randperm(span, generator=gen)[:n].numpy().astype(np.int64)
    return np.sort(perm + lo)


def _plant(k_row: torch.Tensor, w_k: np.ndarray, w_k_pinv: np.ndarray, direction: np.ndarray,
           dtype) -> torch.Tensor:
    """Return k_row moved (minimum-norm) so that its indexer key points along
    `direction` with 4x its original indexer-key norm."""
    k = k_row.double().numpy()
    ki = w_k @ k
    target = 4.0 * np.linalg.norm(ki) * direction / np.linalg.norm(direction)
    k_new = k + w_k_pinv @ (target - ki)
    return torch.from_numpy(k_new).to(torch.float32).to(dtype)


def make_decode_inputs(w: dict, max_ctx: Optional[int] = None) -> dict:
    """Inputs for one decode step over a cache of seq_len[b] tokens.

    Returns k_pre, v [B, Lmax, Hkv, D] (the whole context, the last valid row
    of each sequence being the token appended by the decode step), q_pre
    [B, Hq, D] (the decode query), seq_len [B] int32, w_q, w_k [R, 16, D] fp32
    and the planted needle positions.
    """
    shape: LayerShape = w["shape"]
    gen = torch.Generator().manual_seed(int(w["seed"]))
    B, Hq, Hkv, D, G = shape.batch, shape.n_q_heads, shape.n_kv_heads, shape.head_dim, shape.group
    ctx = w["ctx"]
    if isinstance(ctx, tuple):
        lens = torch.randint(ctx[0], ctx[1] + 1, (B,), generator=gen).numpy().astype(np.int32)
    else:
        lens = np.full((B,), int(ctx), dtype=np.int32)
    Lmax = int(max_ctx) if max_ctx is not None else int(lens.max())
    assert Lmax >= int(lens.max())
    dt = shape.torch_dtype
    w_q, w_k = _projections(gen, shape)
    q_pre = _randn(gen, (B, Hq, D), dt)
    k_pre = _randn(gen, (B, Lmax, Hkv, D), dt)
    v = _randn(gen, (B, Lmax, Hkv, D), dt)
    needles: List[List[np.ndarray]] = []
    for b in range(B):
        L = int(lens[b])
        per_r = []
        for r, h in enumerate(shape.retrieval):
            wk = w_k[r].double().numpy()
            wk_pinv = np.linalg.pinv(wk)
            wq = w_q[r].double().numpy()
            # eligible: outside the sinks and outside the window of the decode query
            pos = _needle_positions(gen, shape.n_sink, max(shape.n_sink, L - shape.window), w["needles"])
            for n, j in enumerate(pos):
                g = n % G
                direction = wq @ q_pre[b, h * G + g].double().numpy()
                k_pre[b, j, h] = _plant(k_pre[b, j, h], wk, wk_pinv, direction, dt)
            per_r.append(pos)
        needles.append(per_r)
    return dict(shape=shape, seq_len=lens, max_ctx=Lmax, q_pre=q_pre, k_pre=k_pre, v=v,
                w_q=w_q, w_k=w_k, needles=needles, name=w.get("name", ""))


def make_prefill_inputs(w: dict, T: Optional[int] = None, start_pos: int = 0,
                        max_ctx: Optional[int] = None) -> dict:
    """Inputs for one causal prefill chunk of T tokens per sequence at positions
    [start_pos, start_pos + T).  Rows [0, start_pos) of k_pre/v are the earlier
    context (already in the cache); rows [start_pos, start_pos+T) are the chunk.

    Needles get an indexer key along a fixed seeded unit direction per
    retrieval head, since every query row of a chunk differs.
    """
    shape: LayerShape = w["shape"]
    gen = torch.Generator().manual_seed(int(w["seed"]))
    B, Hq, Hkv, D = shape.batch, shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    T = int(T if T is not None else w["ctx"])
    L = start_pos + T
    Lmax = int(max_ctx) if max_ctx is not None else L
    assert Lmax >= L
    dt = shape.torch_dtype
    w_q, w_k = _projections(gen, shape)
    q_pre = _randn(gen, (B, T, Hq, D), dt)
    k_pre = _randn(gen, (B, Lmax, Hkv, D), dt)
    v = _randn(gen, (B, Lmax, Hkv, D), dt)
    dirs = torch.randn((shape.n_retrieval, shape.idx_dim), generator=gen, dtype=torch.float64).numpy()
    needles = []
    for b in range(B):
        per_r = []
        for r, h in enumerate(shape.retrieval):
            wk = w_k[r].double().numpy()
            wk_pinv = np.linalg.pinv(wk)
            pos = _needle_positions(gen, shape.n_sink, max(shape.n_sink, L - 1), w["needles"])
            for j in pos:
                k_pre[b, j, h] = _plant(k_pre[b, j, h], wk, wk_pinv, dirs[r], dt)
            per_r.append(pos)
        needles.append(per_r)
    return dict(shape=shape, T=T, start_pos=np.full((B,), start_pos, dtype=np.int32), max_ctx=Lmax,
                q_pre=q_pre, k_pre=k_pre, v=v, w_q=w_q, w_k=w_k, needles=needles,
                name=w.get("name", ""))
