"""rtp_decode_attn_noalloc: the decode step for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc: plug-ins inside a host
framework that owns the GPU memory pool, latency-critical paths that cannot
take cudaMalloc's implicit synchronisation, and C callers that hold only their
inputs and outputs.  For them the library runs the same decode step with its
scratch in a fixed device array it owns, instead of a caller workspace.

These tests check, through the C ABI, that this variant returns what
rtp_decode_attn returns for the same inputs on two calls in a row (the second
with different inputs, so leftovers of the first call in the shared array must
not leak into it), and that configurations whose scratch would not fit are
refused before any device work.  This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

import head_wise_sparse_local_b200 as rtp
from parity import TOL
from synth import make_decode_inputs, workload


def test_noalloc_refuses_configs_that_do_not_fit():
    # 1M context needs far more than the fixed array; refused on the host, no GPU work.
    cfg = rtp.make_cfg(1, 32, 8, 128, 1 << 20, 64, 4096, 0.95, (0, 5))
    assert rtp.rtp_decode_workspace_bytes(cfg) > rtp.RTP_NOALLOC_SCRATCH_BYTES
    fake = 1 << 20
    cache = rtp.rtp_cache(fake, fake, fake, fake)
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_decode_attn_noalloc(cfg, cache, fake, fake, 0, fake, fake, stream=0)
    assert e.value.code == 4
    assert "scratch" in str(e.value)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    dev = torch.device("cuda")
    inp = make_decode_inputs(workload("decode_128k_bf16"))
    sh = inp["shape"]
    L = int(inp["seq_len"][0])
    layer = rtp.Layer(sh, inp["max_ctx"], device=dev)
    assert layer.ws_decode_bytes <= rtp.RTP_NOALLOC_SCRATCH_BYTES
    w_q, w_k = inp["w_q"].to(dev), inp["w_k"].to(dev)
    layer.append(inp["k_pre"].to(dev), inp["v"].to(dev), torch.zeros(1, dtype=torch.int32, device=dev), w_k)
    seq = torch.from_numpy(inp["seq_len"]).to(dev)
    NR = sh.n_retrieval * sh.group
    words = (inp["max_ctx"] + 31) // 32
    g = torch.Generator().manual_seed(99)
    queries = [inp["q_pre"], torch.randn(inp["q_pre"].shape, generator=g).to(torch.bfloat16)]
    atol, rtol = TOL["bf16"]
    for q_host in queries:
        q = q_host.to(dev)
        ref = torch.empty((1, sh.n_q_heads, sh.head_dim), dtype=torch.bfloat16, device=dev)
        bm_ref = torch.zeros((1, NR, words), dtype=torch.int32, device=dev)
        layer.decode(q, seq, w_q, ref, max_seq_len=L, sel_bitmask=bm_ref)
        got = torch.empty_like(ref)
        bm = torch.zeros_like(bm_ref)
        cnt = torch.zeros((1, NR), dtype=torch.int32, device=dev)
        rtp.rtp_decode_attn_noalloc(layer.cfg, layer.cache, q, seq, L, w_q, got, bm, cnt)
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        r, o = ref.double().cpu().numpy(), got.double().cpu().numpy()
        assert np.all(np.abs(o - r) <= atol + rtol * np.abs(r)), float(np.abs(o - r).max())
        assert torch.equal(bm, bm_ref)
        assert int(cnt.min()) >= 1
