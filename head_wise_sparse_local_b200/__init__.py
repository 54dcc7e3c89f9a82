"""B200 (sm_100a) head-wise sparse attention layer: Python binding of librtp.

The functions below keep the C names of include/rtp.h and only marshal
arguments (torch tensors -> device pointers, the current CUDA stream); every
step of the layer runs in the library's CUDA kernels.  There is no CPU
fallback: importing this package loads librtp.so or raises.

`Layer` is a convenience holder for one layer's configuration, cache and
scratch memory, all allocated with torch (PyTorch supplies memory and streams).
"""

from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import torch

from . import _abi
from ._abi import (EXPORTS, RTP_BF16, RTP_DEV_POSITION, RTP_DEV_SEQ_LEN, RTP_DEV_TIMEOUT, RTP_FP32,
                   RTP_NOALLOC_SCRATCH_BYTES, STAGES, RtpError, rtp_cache, rtp_layer_cfg)

_lib = _abi.load()

__all__ = ["Layer", "RtpError", "rtp_layer_cfg", "rtp_cache", "rtp_cache_bytes",
           "rtp_decode_workspace_bytes", "rtp_prefill_workspace_bytes", "rtp_append_kv",
           "rtp_decode_attn", "rtp_decode_attn_noalloc", "rtp_decode_recall", "rtp_prefill_attn",
           "rtp_trace_stage",
           "rtp_debug_wait_expiry",
           "rtp_last_error", "RTP_NOALLOC_SCRATCH_BYTES",
           "rtp_version", "make_cfg", "STAGES",
           "library_path", "EXPORTS", "RTP_BF16", "RTP_FP32", "RTP_DEV_SEQ_LEN",
           "RTP_DEV_POSITION", "RTP_DEV_TIMEOUT"]


def library_path() -> str:
    return _abi.LIB_PATH


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        if not x.is_cuda:
            raise ValueError("expected a CUDA tensor")
        if not x.is_contiguous():
            raise ValueError("expected a contiguous tensor")
        return x.data_ptr()
    raise TypeError(f"cannot pass {type(x)} as a device pointer")


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def make_cfg(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int, max_ctx: int,
             n_sink: int, window: int, top_p: float, retrieval: Sequence[int],
             dtype: str = "bf16", rope_base: float = 10000.0, idx_dim: int = 16,
             local_cap: int = 0, top_k: int = 0) -> rtp_layer_cfg:
    mask = 0
    for h in retrieval:
        mask |= 1 << int(h)
    return rtp_layer_cfg(batch, n_q_heads, n_kv_heads, head_dim, idx_dim, max_ctx, n_sink, window,
                         top_p, rope_base, mask, RTP_BF16 if dtype == "bf16" else RTP_FP32,
                         int(local_cap), int(top_k))


def rtp_version() -> str:
    return _lib.rtp_version().decode()


def rtp_last_error() -> str:
    return _lib.rtp_last_error().decode()


def rtp_trace_stage(stage, start_event=None, stop_event=None) -> None:
    """Arm CUDA events (torch.cuda.Event with timing) around the next launch of a stage."""
    sid = STAGES[stage] if isinstance(stage, str) else int(stage)
    handles = []
    for ev in (start_event, stop_event):
        if ev is None:
            handles.append(None)
            continue
        if not ev.cuda_event:  # torch creates its events lazily, at the first record
            ev.record()
        handles.append(ev.cuda_event)
    _abi.check(_lib.rtp_trace_stage(sid, handles[0], handles[1]))


def rtp_debug_wait_expiry(polls: int) -> None:
    """Arm the next rtp_decode_attn call on this thread to let its bounded waits expire."""
    _abi.check(_lib.rtp_debug_wait_expiry(int(polls)))


def rtp_cache_bytes(cfg: rtp_layer_cfg):
    k, v, ki = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _abi.check(_lib.rtp_cache_bytes(ctypes.byref(cfg), ctypes.byref(k), ctypes.byref(v), ctypes.byref(ki)))
    return k.value, v.value, ki.value


def rtp_decode_workspace_bytes(cfg: rtp_layer_cfg) -> int:
    n = ctypes.c_size_t()
    _abi.check(_lib.rtp_decode_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def rtp_prefill_workspace_bytes(cfg: rtp_layer_cfg, T: int) -> int:
    n = ctypes.c_size_t()
    _abi.check(_lib.rtp_prefill_workspace_bytes(ctypes.byref(cfg), int(T), ctypes.byref(n)))
    return n.value


def rtp_append_kv(cfg, cache, k_pre, v_in, start_pos, T, w_k, stream=None) -> None:
    _abi.check(_lib.rtp_append_kv(ctypes.byref(cfg), ctypes.byref(cache), _ptr(k_pre), _ptr(v_in),
                                  _ptr(start_pos), int(T), _ptr(w_k), _stream(stream)))


def rtp_decode_attn(cfg, cache, q_pre, seq_len, max_seq_len, w_q, out, sel_bitmask=None,
                    sel_count=None, workspace=None, workspace_bytes=0, stream=None) -> None:
    _abi.check(_lib.rtp_decode_attn(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q_pre),
                                    _ptr(seq_len), int(max_seq_len), _ptr(w_q), _ptr(out),
                                    _ptr(sel_bitmask), _ptr(sel_count), _ptr(workspace),
                                    int(workspace_bytes), _stream(stream)))


def rtp_decode_attn_noalloc(cfg, cache, q_pre, seq_len, max_seq_len, w_q, out, sel_bitmask=None,
                            sel_count=None, stream=None) -> None:
    """rtp_decode_attn with the library's fixed device scratch instead of a workspace."""
    _abi.check(_lib.rtp_decode_attn_noalloc(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q_pre),
                                            _ptr(seq_len), int(max_seq_len), _ptr(w_q), _ptr(out),
                                            _ptr(sel_bitmask), _ptr(sel_count), _stream(stream)))


def rtp_decode_recall(cfg, cache, q_pre, seq_len, max_seq_len, sel_bitmask, recall, workspace=None,
                      workspace_bytes=0, stream=None) -> None:
    _abi.check(_lib.rtp_decode_recall(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q_pre),
                                      _ptr(seq_len), int(max_seq_len), _ptr(sel_bitmask), _ptr(recall),
                                      _ptr(workspace), int(workspace_bytes), _stream(stream)))


def rtp_prefill_attn(cfg, cache, q_pre, start_pos, T, w_q, out, sel_bitmask=None, sel_tau=None,
                     sel_jcut=None, sel_count=None, workspace=None, workspace_bytes=0,
                     stream=None) -> None:
    _abi.check(_lib.rtp_prefill_attn(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q_pre),
                                     _ptr(start_pos), int(T), _ptr(w_q), _ptr(out),
                                     _ptr(sel_bitmask), _ptr(sel_tau), _ptr(sel_jcut),
                                     _ptr(sel_count), _ptr(workspace), int(workspace_bytes),
                                     _stream(stream)))


class Layer:
    """One layer's configuration plus its device cache and scratch (torch-allocated).

    local_cap > 0 selects ring mode: local heads keep only their sinks and a
    ring of local_cap window rows.  k and v are then flat [B, rows, D] buffers
    (head_rows() gives each head's slice); otherwise [B, Hkv, max_ctx, D]."""

    def __init__(self, shape, max_ctx: int, device="cuda", prefill_T: int = 0, local_cap: int = 0):
        self.shape = shape
        self.cfg = make_cfg(shape.batch, shape.n_q_heads, shape.n_kv_heads, shape.head_dim, max_ctx,
                            shape.n_sink, shape.window, shape.top_p, shape.retrieval, shape.dtype,
                            shape.rope_base, shape.idx_dim, local_cap, getattr(shape, "top_k", 0))
        self.max_ctx = max_ctx
        dt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
        B, Hkv, D, R = shape.batch, shape.n_kv_heads, shape.head_dim, shape.n_retrieval
        es = 2 if shape.dtype == "bf16" else 4
        k_bytes, _, _ = rtp_cache_bytes(self.cfg)
        rows = k_bytes // (B * D * es)
        self.ring = rows != Hkv * max_ctx
        if self.ring:
            self.k = torch.empty((B, rows, D), dtype=dt, device=device)
        else:
            self.k = torch.empty((B, Hkv, max_ctx, D), dtype=dt, device=device)
        self.v = torch.empty_like(self.k)
        # indexer keys [B, R, Lk, d] (Lk = max_ctx, or max_ctx rounded up to even
        # for 8-byte bf16 d = 4 rows); kidx views the first max_ctx rows of each block
        d = shape.idx_dim
        _, _, ki_bytes = rtp_cache_bytes(self.cfg)
        Lk = ki_bytes // (B * max(R, 1) * d * es) if R > 0 else max_ctx
        self.kidx_full = torch.empty((B, max(R, 1), Lk, d), dtype=dt, device=device)
        self.kidx = self.kidx_full[:, :, :max_ctx]
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.cache = rtp_cache(self.k.data_ptr(), self.v.data_ptr(), self.kidx_full.data_ptr(),
                               self.status.data_ptr())
        self.ws_decode_bytes = rtp_decode_workspace_bytes(self.cfg)
        self.ws_decode = torch.empty(self.ws_decode_bytes, dtype=torch.uint8, device=device)
        self.ws_prefill = None
        self.ws_prefill_bytes = 0
        if prefill_T:
            self.reserve_prefill(prefill_T)

    def reserve_prefill(self, T: int) -> None:
        n = rtp_prefill_workspace_bytes(self.cfg, T)
        if n > self.ws_prefill_bytes:
            self.ws_prefill_bytes = n
            self.ws_prefill = torch.empty(n, dtype=torch.uint8, device=self.k.device)

    def append(self, k_pre, v_in, start_pos, w_k, stream=None) -> None:
        rtp_append_kv(self.cfg, self.cache, k_pre, v_in, start_pos, k_pre.shape[1], w_k, stream)

    def decode(self, q_pre, seq_len, w_q, out, max_seq_len: int = 0, sel_bitmask=None,
               sel_count=None, stream=None) -> None:
        rtp_decode_attn(self.cfg, self.cache, q_pre, seq_len, max_seq_len, w_q, out, sel_bitmask,
                        sel_count, self.ws_decode, self.ws_decode_bytes, stream)

    def recall(self, q_pre, seq_len, sel_bitmask, recall, max_seq_len: int = 0, stream=None) -> None:
        rtp_decode_recall(self.cfg, self.cache, q_pre, seq_len, max_seq_len, sel_bitmask, recall,
                          self.ws_decode, self.ws_decode_bytes, stream)

    def prefill(self, q_pre, start_pos, w_q, out, sel_bitmask=None, sel_tau=None, sel_jcut=None,
                sel_count=None, stream=None) -> None:
        T = q_pre.shape[1]
        self.reserve_prefill(T)
        rtp_prefill_attn(self.cfg, self.cache, q_pre, start_pos, T, w_q, out, sel_bitmask, sel_tau,
                         sel_jcut, sel_count, self.ws_prefill, self.ws_prefill_bytes, stream)

    def device_status(self) -> int:
        return int(self.status.item())
