"""ctypes view of include/rtp.h.  Loads the in-tree librtp.so or fails loudly."""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librtp.so")

RTP_OK = 0
RTP_ERR_INVALID = 1
RTP_ERR_SHAPE = 2
RTP_ERR_DTYPE = 3
RTP_ERR_WORKSPACE = 4
RTP_ERR_CUDA = 5
RTP_DEV_SEQ_LEN = 0x1
RTP_DEV_POSITION = 0x2
RTP_DEV_TIMEOUT = 0x4
RTP_BF16 = 0
RTP_FP32 = 1
RTP_NOALLOC_SCRATCH_BYTES = 32 << 20

STATUS_NAMES = {0: "RTP_OK", 1: "RTP_ERR_INVALID", 2: "RTP_ERR_SHAPE", 3: "RTP_ERR_DTYPE",
                4: "RTP_ERR_WORKSPACE", 5: "RTP_ERR_CUDA"}

# Every entry point declared in include/rtp.h.
EXPORTS = ("rtp_cache_bytes", "rtp_decode_workspace_bytes", "rtp_prefill_workspace_bytes",
           "rtp_append_kv", "rtp_decode_attn", "rtp_decode_attn_noalloc", "rtp_decode_recall",
           "rtp_prefill_attn",
           "rtp_trace_stage", "rtp_debug_wait_expiry",
           "rtp_last_error", "rtp_version")

STAGES = {"append": 0, "decode_score": 1, "decode_select": 2, "decode_local": 3,
          "prefill_index": 4, "prefill_attn": 5}


class rtp_layer_cfg(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("idx_dim", ctypes.c_int), ("max_ctx", ctypes.c_int),
                ("n_sink", ctypes.c_int), ("window", ctypes.c_int), ("top_p", ctypes.c_float),
                ("rope_base", ctypes.c_float), ("retrieval_mask", ctypes.c_uint64),
                ("dtype", ctypes.c_int), ("local_cap", ctypes.c_int), ("top_k", ctypes.c_int)]


class rtp_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("kidx", ctypes.c_void_p),
                ("status", ctypes.c_void_p)]


class RtpError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load librtp.so once.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python head_wise_sparse_local_b200/build.py`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    cfgp, cachep = P(rtp_layer_cfg), P(rtp_cache)
    lib.rtp_cache_bytes.argtypes = [cfgp, P(sz), P(sz), P(sz)]
    lib.rtp_decode_workspace_bytes.argtypes = [cfgp, P(sz)]
    lib.rtp_prefill_workspace_bytes.argtypes = [cfgp, i32, P(sz)]
    lib.rtp_append_kv.argtypes = [cfgp, cachep, vp, vp, vp, i32, vp, vp]
    lib.rtp_decode_attn.argtypes = [cfgp, cachep, vp, vp, i32, vp, vp, vp, vp, vp, sz, vp]
    lib.rtp_prefill_attn.argtypes = [cfgp, cachep, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.rtp_trace_stage.argtypes = [i32, vp, vp]
    lib.rtp_debug_wait_expiry.argtypes = [i32]
    lib.rtp_decode_attn_noalloc.argtypes = [cfgp, cachep, vp, vp, i32, vp, vp, vp, vp, vp]
    lib.rtp_decode_recall.argtypes = [cfgp, cachep, vp, vp, i32, vp, vp, vp, sz, vp]
    for name in EXPORTS:
        getattr(lib, name).restype = ctypes.c_char_p if name in ("rtp_last_error", "rtp_version") \
            else ctypes.c_int
    _lib = lib
    return lib


def check(code: int) -> None:
    if code != RTP_OK:
        raise RtpError(code, load().rtp_last_error().decode())
