"""GPU parity of the prefill path (rtp_append_kv + rtp_prefill_attn through
the C ABI) against the fp64 oracle: per-row top-p sets and outputs on chunks
that span several tiles with ragged tails, chunked prefill after a context,
p = 1, a ragged batch, agreement with decode steps at the same positions, and
sampled rows of the full 32K prefill workload."""

import numpy as np
import pytest
import torch

from parity import check_prefill_parity, run_gpu_decode, run_gpu_prefill
from synth import LayerShape, make_prefill_inputs, workload

pytestmark = pytest.mark.gpu


def _inp(T=700, start=0, needles=16, **shape_kw):
    kw = {"shape_" + k: v for k, v in shape_kw.items()}
    w = workload("prefill_32k_bf16", needles=needles, **kw)
    return make_prefill_inputs(w, T=T, start_pos=start)


def test_prefill_small_all_rows():
    inp = _inp(T=700, n_sink=16, window=128, top_p=0.9)
    st = check_prefill_parity(inp)
    assert st["exact"] >= st["heads"] - 2


def test_prefill_chunk_after_context():
    inp = _inp(T=450, start=333, n_sink=8, window=100, top_p=0.8)
    check_prefill_parity(inp)


def test_prefill_rows_longer_than_the_key_ring():
    # rows of 3000-3200 keys: 6-7 key tiles of 512, more than the tiles in flight
    inp = _inp(T=200, start=3000, n_sink=8, window=100, top_p=0.9, needles=12)
    st = check_prefill_parity(inp)
    assert st["exact"] >= st["heads"] - 2


def test_prefill_p1_is_dense_causal():
    inp = _inp(T=300, n_sink=4, window=50, top_p=1.0)
    st = check_prefill_parity(inp)
    assert st["exact"] == st["heads"]
    assert np.all(st["g"]["count"][0, 0] == np.arange(1, 301))


def test_prefill_ragged_batch_and_head_dim_64():
    sh = LayerShape(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=64, n_sink=4, window=40,
                    top_p=0.85, retrieval=(1,), dtype="bf16")
    w = dict(kind="prefill", seed=31, ctx=260, needles=6, shape=sh)
    inp = make_prefill_inputs(w, T=260, start_pos=0, max_ctx=600)
    inp["start_pos"] = np.array([0, 200], dtype=np.int32)
    check_prefill_parity(inp)


def test_prefill_rows_equal_decode_steps():
    """A prefill row's top-p set equals the decode step's at that position, bit
    for bit: both compute the indexer scores with the same tensor-core
    arithmetic (q~ as bf16 hi + lo parts accumulated into one fp32 value) and
    the same exact fixed-point selection, so nothing is left to tolerance."""
    inp = _inp(T=520, n_sink=16, window=64, top_p=0.9)
    g = run_gpu_prefill(inp)
    sh = inp["shape"]
    bm_p = g["bitmask"].cpu().numpy().view(np.uint32)
    for t in [0, 1, 63, 64, 255, 519]:
        dec = dict(shape=sh, seq_len=np.array([t + 1], dtype=np.int32), max_ctx=inp["max_ctx"],
                   q_pre=inp["q_pre"][:, t].contiguous(), k_pre=inp["k_pre"], v=inp["v"],
                   w_q=inp["w_q"], w_k=inp["w_k"])
        d = run_gpu_decode(dec)
        bm_d = d["bitmask"].cpu().numpy().view(np.uint32)
        for rg in range(sh.n_retrieval * sh.group):
            dset = np.nonzero(np.unpackbits(bm_d[0, rg].view(np.uint8), bitorder="little")[: t + 1])[0]
            pset = np.nonzero(np.unpackbits(bm_p[0, rg, t].view(np.uint8), bitorder="little")[: t + 1])[0]
            assert np.array_equal(pset, dset), (t, rg, len(pset), len(dset))
            assert int(g["count"][0, rg, t]) == int(d["count"][0, rg])


def test_prefill_32k_sampled_rows():
    inp = make_prefill_inputs(workload("prefill_32k_bf16"))
    rows = [0, 1, 64, 2047, 2048, 5000, 16383, 16384, 30000, 32767]
    st = check_prefill_parity(inp, rows=rows)
    assert st["exact"] >= st["heads"] - 2


def test_prefill_single_row_and_tiny_p():
    inp = _inp(T=1, start=0, n_sink=4, window=16, top_p=0.9)
    st = check_prefill_parity(inp)
    assert st["exact"] == st["heads"]
    inp = _inp(T=300, start=100, n_sink=4, window=16, top_p=1e-6)
    st = check_prefill_parity(inp)
    assert np.all(st["g"]["count"] == 1)


@pytest.mark.parametrize("p", [0.5, 0.77])
def test_prefill_all_scores_equal(p):
    """Every indexer key of the retrieval heads identical: each row's scores
    are all tied, so the selection resolves the cut by index alone (the tie
    passes); row t keeps its first ceil(p (t + 1)) tokens."""
    inp = _inp(T=300, n_sink=4, window=16, top_p=p, needles=0)
    sh = inp["shape"]
    for h in sh.retrieval:
        inp["k_pre"][0, :, h] = inp["k_pre"][0, 0, h]
    g = run_gpu_prefill(inp)
    assert g["status"] == 0
    bm = g["bitmask"].cpu().numpy().view(np.uint32)
    pf = float(np.float32(p))
    for t in [0, 1, 2, 31, 32, 100, 299]:
        want = int(np.ceil(pf * (t + 1)))
        for rg in range(sh.n_retrieval * sh.group):
            bits = np.unpackbits(bm[0, rg, t].view(np.uint8), bitorder="little")[: t + 1]
            assert np.array_equal(np.nonzero(bits)[0], np.arange(want)), (t, rg, int(bits.sum()), want)
            assert g["count"][0, rg, t] == want
    check_prefill_parity(inp, rows=[0, 5, 77, 299], g=g)


def test_prefill_tied_block_keeps_lowest_indices():
    """A block of identical indexer keys at a needle's key: for rows where the
    block holds the cut, the kept part of the block is its lowest indices."""
    inp = _inp(T=900, n_sink=4, window=32, top_p=0.6, needles=8)
    sh = inp["shape"]
    h = sh.retrieval[0]
    src = int(inp["needles"][0][0][0])
    inp["k_pre"][0, 300:600, h] = inp["k_pre"][0, src, h]
    g = run_gpu_prefill(inp)
    assert g["status"] == 0
    bm = g["bitmask"].cpu().numpy().view(np.uint32)
    n_cut = 0
    for t in range(600, 900, 7):
        for gg in range(sh.group):
            bits = np.unpackbits(bm[0, gg, t].view(np.uint8), bitorder="little")[: t + 1]
            kept = np.nonzero(bits[300:600])[0]
            if 0 < len(kept) < 300:
                n_cut += 1
                assert np.array_equal(kept, np.arange(len(kept))), (t, gg, kept[:8])
    check_prefill_parity(inp, rows=list(range(600, 900, 37)), g=g)
    assert n_cut > 0


def test_prefill_refuses_static_topk():
    """Static top-k is a decode-only variant: the prefill entry point refuses it
    on the host, before any device work."""
    import head_wise_sparse_local_b200 as rtp
    sh = workload("prefill_32k_bf16")["shape"].replace(top_k=100)
    lay = rtp.Layer(sh, 1024, device="cuda")
    q = torch.zeros((1, 64, sh.n_q_heads, sh.head_dim), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rtp.RtpError) as e:
        lay.prefill(q, torch.zeros(1, dtype=torch.int32, device="cuda"),
                    torch.zeros((2, 16, sh.head_dim), device="cuda"), torch.empty_like(q))
    assert e.value.code == 2 and "top-k" in str(e.value)


def test_prefill_row_blocks_equal_one_block():
    """A chunk whose per-row bitmask would pass the workspace budget runs in
    blocks of rows: at a 1M-token capacity a row's bitmask over 8 retrieval q
    heads is 1 MiB, so a 2304-row chunk without a caller bitmask runs as blocks
    of 1024, 1024 and 256 rows (selection, tile map and attention per block).
    Its outputs, counts, thresholds and cut indices equal the one-block run's
    (the caller's bitmask holds every row) bit for bit, and the one-block run
    matches the oracle on rows at the block edges."""
    from head_wise_sparse_local_b200 import Layer
    inp = _inp(T=2304, n_sink=16, window=256, top_p=0.9, needles=16)
    sh, T = inp["shape"], inp["T"]
    Lmax = 1 << 20
    dev = torch.device("cuda")
    lay = Layer(sh, Lmax, device=dev, prefill_T=T)
    zero = torch.zeros(sh.batch, dtype=torch.int32, device=dev)
    lay.append(inp["k_pre"][:, :T].contiguous().to(dev), inp["v"][:, :T].contiguous().to(dev), zero,
               inp["w_k"].to(dev))
    q, w_q = inp["q_pre"].to(dev), inp["w_q"].to(dev)
    NR = sh.n_retrieval * sh.group
    runs = []
    for with_bm in (True, False):
        out = torch.empty((sh.batch, T, sh.n_q_heads, sh.head_dim), dtype=sh.torch_dtype, device=dev)
        bm = torch.zeros((sh.batch, NR, T, Lmax // 32), dtype=torch.int32, device=dev) if with_bm else None
        cnt = torch.full((sh.batch, NR, T), -1, dtype=torch.int32, device=dev)
        tau = torch.zeros((sh.batch, NR, T), dtype=torch.float32, device=dev)
        jcut = torch.zeros((sh.batch, NR, T), dtype=torch.int32, device=dev)
        lay.prefill(q, zero, w_q, out, sel_bitmask=bm, sel_tau=tau, sel_jcut=jcut, sel_count=cnt)
        torch.cuda.synchronize()
        runs.append(dict(out=out, bitmask=bm, count=cnt.cpu().numpy(), tau=tau.cpu().numpy(),
                         jcut=jcut.cpu().numpy()))
        del bm
    assert lay.device_status() == 0
    one, blocks = runs
    assert torch.equal(one["out"], blocks["out"])
    assert np.array_equal(one["count"], blocks["count"])
    assert np.array_equal(one["tau"], blocks["tau"])
    assert np.array_equal(one["jcut"], blocks["jcut"])
    g = dict(out=one["out"].double().cpu().numpy(), bitmask=one["bitmask"], count=one["count"], status=0)
    st = check_prefill_parity(inp, rows=[0, 1, 1023, 1024, 1025, 2047, 2048, 2303], g=g)
    assert st["exact"] >= st["heads"] - 2
