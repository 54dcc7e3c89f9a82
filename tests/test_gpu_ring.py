"""GPU parity of the memory-sparse cache (ring mode, cfg.local_cap > 0): local
heads keep only their sinks and a ring of window rows, retrieval heads the
whole context, as the abstract of "Full Attention Strikes Back" describes
(the full KV cache is kept only for retrieval heads; atlas.scime.ai summary,
"Experimental setup": memory sparsity).  The layer must compute exactly what
it computes with the full cache: decode steps and prefill chunks are checked
against the fp64 oracle, which knows nothing of the ring, including rings that
wrapped many times, the smallest ring a prefill chunk allows, and decode steps
that continue after a prefill chunk."""

import numpy as np
import pytest
import torch

import head_wise_sparse_local_b200 as rtp
import oracle
from parity import TOL, append_context, check_decode_parity, check_prefill_parity
from synth import LayerShape, make_decode_inputs, make_prefill_inputs, workload

pytestmark = pytest.mark.gpu


def test_ring_cache_bytes_and_layout():
    cfg_full = rtp.make_cfg(1, 32, 8, 128, 1 << 20, 64, 4096, 0.95, (0, 5))
    cfg_ring = rtp.make_cfg(1, 32, 8, 128, 1 << 20, 64, 4096, 0.95, (0, 5), local_cap=4096)
    kf, _, _ = rtp.rtp_cache_bytes(cfg_full)
    kr, _, _ = rtp.rtp_cache_bytes(cfg_ring)
    assert kf == 8 * (1 << 20) * 128 * 2
    assert kr == (2 * (1 << 20) + 6 * (64 + 4096)) * 128 * 2
    assert kr / kf < 0.26


@pytest.mark.parametrize("cap_extra", [0, 37])
def test_ring_decode_wrapped(cap_extra):
    # 9000 tokens through a ring of W (+37): the window rows wrapped many times
    inp = make_decode_inputs(workload("decode_128k_bf16", ctx=9000, needles=16))
    sh = inp["shape"]
    st = check_decode_parity(inp, top_p=0.9, local_cap=sh.window + cap_extra)
    assert st["exact"] >= st["heads"] - 1


def test_ring_decode_ragged_batch_edges():
    # sequences shorter than the sinks, than the window, exactly sinks + ring, and longer
    w = workload("ragged_decode_b8_8k_32k_bf16", shape_batch=5, ctx=(1, 9000), needles=4,
                 shape_window=300, shape_n_sink=16)
    inp = make_decode_inputs(w, max_ctx=9100)
    inp["seq_len"] = np.array([1, 10, 250, 16 + 310, 9000], dtype=np.int32)
    check_decode_parity(inp, top_p=0.9, local_cap=310)


def test_ring_decode_fp32_small_window():
    sh = LayerShape(batch=2, n_q_heads=8, n_kv_heads=4, head_dim=64, n_sink=3, window=5,
                    top_p=0.7, retrieval=(1,), dtype="fp32")
    w = dict(kind="decode", seed=12, ctx=(700, 2000), needles=3, shape=sh)
    check_decode_parity(make_decode_inputs(w), local_cap=7)


def test_ring_decode_128k_full_size():
    inp = make_decode_inputs(workload("decode_128k_bf16"))
    st = check_decode_parity(inp, local_cap=inp["shape"].window)
    assert st["exact"] == st["heads"]


def test_ring_decode_1m_full_size():
    inp = make_decode_inputs(workload("decode_1m_bf16"))
    st = check_decode_parity(inp, local_cap=inp["shape"].window)
    assert st["exact"] >= st["heads"] - 1


def test_ring_prefill_smallest_ring_then_decode_steps():
    """A prefill chunk with the smallest ring it allows (T + W - 1), after a
    context, then decode steps that keep wrapping the ring."""
    T, W, S, start = 300, 100, 8, 250
    w = workload("prefill_32k_bf16", needles=10, shape_window=W, shape_n_sink=S, shape_top_p=0.85)
    inp = make_prefill_inputs(w, T=T, start_pos=start, max_ctx=start + T + 3)
    cap = T + W - 1
    st = check_prefill_parity(inp, local_cap=cap)
    assert st["exact"] >= st["heads"] - 2
    # decode steps at positions start+T .. start+T+2 on the same ring cache
    lay = st["g"]["layer"]
    sh = inp["shape"]
    dev = torch.device("cuda")
    w_q, w_k = inp["w_q"].to(dev), inp["w_k"].to(dev)
    oc = oracle.OracleCache(sh, inp["max_ctx"])
    oc.append_in_place(inp["k_pre"], inp["v"], np.array([start + T + 3]), inp["w_k"])
    g = torch.Generator().manual_seed(5)
    atol, rtol = TOL["bf16"]
    for step in range(3):
        pos = start + T + step
        k1 = inp["k_pre"][:, pos:pos + 1].contiguous().to(dev)
        v1 = inp["v"][:, pos:pos + 1].contiguous().to(dev)
        lay.append(k1, v1, torch.full((1,), pos, dtype=torch.int32, device=dev), w_k)
        q = torch.randn((1, sh.n_q_heads, sh.head_dim), generator=g).to(torch.bfloat16)
        out = torch.empty((1, sh.n_q_heads, sh.head_dim), dtype=torch.bfloat16, device=dev)
        NR = sh.n_retrieval * sh.group
        bm = torch.zeros((1, NR, (inp["max_ctx"] + 31) // 32), dtype=torch.int32, device=dev)
        seq = torch.full((1,), pos + 1, dtype=torch.int32, device=dev)
        lay.decode(q.to(dev), seq, w_q, out, max_seq_len=pos + 1, sel_bitmask=bm)
        torch.cuda.synchronize()
        assert lay.device_status() == 0
        ref, topp, _ = oracle.decode(oc, q, np.array([pos + 1]), inp["w_q"])
        bits = np.unpackbits(bm.cpu().numpy().view(np.uint32)[0].view(np.uint8).reshape(NR, -1),
                             axis=1, bitorder="little")[:, :pos + 1]
        override = {}
        for r, h in enumerate(sh.retrieval):
            for gg in range(sh.group):
                kept = np.nonzero(bits[r * sh.group + gg])[0]
                if not np.array_equal(kept, topp[(0, h * sh.group + gg)]):
                    override[(0, h * sh.group + gg)] = np.union1d(
                        kept, oracle.sink_window_set(pos, sh.n_sink, sh.window))
        if override:
            ref, _, _ = oracle.decode(oc, q, np.array([pos + 1]), inp["w_q"], rows_override=override)
        got = out.double().cpu().numpy()
        assert np.all(np.abs(got - ref) <= atol + rtol * np.abs(ref)), (step, float(np.abs(got - ref).max()))


def test_ring_prefill_chunk_too_long_is_refused():
    sh = workload("prefill_32k_bf16")["shape"]
    lay = rtp.Layer(sh, 4096, device="cuda", local_cap=sh.window + 10)
    q = torch.zeros((1, 64, sh.n_q_heads, sh.head_dim), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    start = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(rtp.RtpError) as e:
        lay.prefill(q, start, torch.zeros((2, 16, sh.head_dim), device="cuda"), out)
    assert e.value.code == 2
