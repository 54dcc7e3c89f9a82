"""GPU parity of the decode path (rtp_append_kv + rtp_decode_attn through the
C ABI) against the fp64 oracle: selection sets and outputs, at sizes that span
several tiles with ragged tails, the edge cases (one-token contexts, contexts
shorter than the sinks or the window, p = 1, exact ties), and the full-size
128K, ragged-batch and 1M decode workloads."""

import numpy as np
import pytest
import torch

import oracle
from parity import (TOL, bitmask_to_sets, check_decode_parity, kidx_bound, oracle_cache_from_inputs,
                    run_gpu_decode)
from synth import LayerShape, make_decode_inputs, workload

pytestmark = pytest.mark.gpu


def _small(name="decode_128k_bf16", **kw):
    return make_decode_inputs(workload(name, **kw))


def test_tiny_decode_fp32():
    inp = make_decode_inputs(workload("tiny_decode_2k_fp32"))
    st = check_decode_parity(inp)
    assert st["exact"] == st["heads"]


@pytest.mark.parametrize("p", [0.3, 0.9, 0.95, 0.999, 1.0])
def test_decode_bf16_several_tiles(p):
    # 5000 tokens: 5 score chunks, 2 histogram chunks, 3 selected-row tiles (ragged tails)
    inp = _small(ctx=5000, needles=16)
    st = check_decode_parity(inp, top_p=p)
    assert st["exact"] >= st["heads"] - 1


def test_decode_flat_scores_dense_selection():
    # no needles: scores ~ N(0, 1), top-p keeps ~Phi(Phi^-1(p) - 1) of the context
    inp = _small(ctx=20000, needles=0)
    st = check_decode_parity(inp, top_p=0.8)
    frac = st["counts"].mean() / 20000
    assert 0.3 < frac < 0.55, frac


def test_decode_ragged_edges():
    # seq lens below the sinks, between sinks and window, and beyond; plus L = 1
    w = workload("ragged_decode_b8_8k_32k_bf16", shape_batch=5, ctx=(1, 9000), needles=4)
    inp = make_decode_inputs(w, max_ctx=9100)
    inp["seq_len"] = np.array([1, 37, 2100, 2113, 9000], dtype=np.int32)
    check_decode_parity(inp, top_p=0.9)


def test_decode_small_window_and_no_sinks_fp32():
    sh = LayerShape(batch=2, n_q_heads=8, n_kv_heads=4, head_dim=64, n_sink=0, window=1,
                    top_p=0.7, retrieval=(1, 3), dtype="fp32")
    w = dict(kind="decode", seed=11, ctx=(300, 3000), needles=3, shape=sh)
    inp = make_decode_inputs(w)
    check_decode_parity(inp)


@pytest.mark.parametrize("G", [1, 2, 8])
def test_decode_group_sizes(G):
    sh = LayerShape(batch=1, n_q_heads=4 * G, n_kv_heads=4, head_dim=128, n_sink=16, window=256,
                    top_p=0.9, retrieval=(2,), dtype="bf16")
    w = dict(kind="decode", seed=20 + G, ctx=6000, needles=2 * G, shape=sh)
    check_decode_parity(make_decode_inputs(w))


def test_decode_exact_ties_resolved_by_index():
    inp = _small(ctx=5000, needles=8)
    sh = inp["shape"]
    h = sh.retrieval[0]
    src = int(inp["needles"][0][0][0])  # a needle aimed at q head h*G + 0
    inp["k_pre"][0, 100:400, h] = inp["k_pre"][0, src, h]
    for p in [0.2, 0.5, 0.9]:
        g = run_gpu_decode(inp, top_p=p)
        oc = oracle_cache_from_inputs(inp)
        oc.shape = sh.replace(top_p=p)
        _, topp_o, _ = oracle.decode(oc, inp["q_pre"], inp["seq_len"], inp["w_q"],
                                     heads=[h * sh.group])
        gset = bitmask_to_sets(g["bitmask"][0], [5000] * (sh.n_retrieval * sh.group))[0]
        o = topp_o[(0, h * sh.group)]
        assert np.array_equal(gset, o), (p, len(gset), len(o))
        tied = np.intersect1d(o, np.arange(100, 400))
        if 0 < len(tied) < 300:
            assert np.array_equal(tied, np.arange(100, 100 + len(tied)))  # lowest indices win


def test_decode_repeatable_bitwise():
    inp = _small(ctx=12000, needles=0)
    a = run_gpu_decode(inp, top_p=0.9)
    b = run_gpu_decode(inp, top_p=0.9)
    assert np.array_equal(a["out"], b["out"])
    assert torch.equal(a["bitmask"], b["bitmask"])


def test_decode_invalid_seq_len_sets_status_and_skips():
    inp = _small(ctx=3000, needles=2, shape_batch=2)
    inp["seq_len"] = np.array([3000, 0], dtype=np.int32)
    g = run_gpu_decode(inp, append_last_separately=False)
    assert g["status"] & 0x1
    sh1 = inp["shape"].replace(batch=1)
    oc = oracle.OracleCache(sh1, inp["max_ctx"])
    oc.append_in_place(inp["k_pre"][:1], inp["v"][:1], inp["seq_len"][:1], inp["w_k"])
    out_o, _, _ = oracle.decode(oc, inp["q_pre"][:1], inp["seq_len"][:1], inp["w_q"])
    atol, rtol = TOL["bf16"]
    assert np.all(np.abs(g["out"][0] - out_o[0]) <= atol + rtol * np.abs(out_o[0]))


def test_append_matches_oracle_cache():
    inp = _small(ctx=3000, needles=2)
    g = run_gpu_decode(inp)
    lay, sh = g["layer"], g["shape"]
    oc = oracle_cache_from_inputs(inp)
    rows = np.array([0, 1, 63, 64, 1000, 2999])
    for h in [0, 1, 5]:
        kg = lay.k[0, h, rows].double().cpu().numpy()
        ko = oc.keys(0, h, rows)
        ulp = np.abs(ko) * 2.0 ** -7 + 1e-30
        assert np.all(np.abs(kg - ko) <= ulp), h
        vg = lay.v[0, h, rows].double().cpu().numpy()
        assert np.array_equal(vg, oc.values(0, h, rows))
    for r in range(sh.n_retrieval):
        kig = lay.kidx[0, r, :3000].double().cpu().numpy()
        kio = oc.indexer_keys(0, r, 3000)
        assert np.all(np.abs(kig - kio) <= kidx_bound(inp, 0, r, np.arange(3000)))
        assert np.mean(kig == kio) > 0.999


def test_decode_128k_full_size():
    inp = make_decode_inputs(workload("decode_128k_bf16"))
    st = check_decode_parity(inp)
    assert st["exact"] == st["heads"]
    # needles dominate: each retrieval q head keeps only planted needle tokens
    assert st["counts"].max() <= 64


@pytest.mark.parametrize("p", [0.8, 0.95, 0.99])
def test_ragged_batch_full_size(p):
    inp = make_decode_inputs(workload("ragged_decode_b8_8k_32k_bf16"))
    check_decode_parity(inp, top_p=p)


def test_decode_1m_full_size():
    inp = make_decode_inputs(workload("decode_1m_bf16"))
    st = check_decode_parity(inp)
    assert st["exact"] >= st["heads"] - 1


@pytest.mark.parametrize("n_tied,p", [(300, 0.5), (2000, 0.3), (2000, 0.9)])
def test_decode_large_tie_blocks(n_tied, p):
    """Many identical indexer keys near the boundary: exercises the exact solve
    over small and large candidate sets (pairwise ranks / radix passes)."""
    inp = _small(ctx=12000, needles=8)
    sh = inp["shape"]
    h = sh.retrieval[1]
    src = int(inp["needles"][0][1][1])  # a needle aimed at q head h*G + 1
    inp["k_pre"][0, 200:200 + n_tied, h] = inp["k_pre"][0, src, h]
    g = run_gpu_decode(inp, top_p=p)
    oc = oracle_cache_from_inputs(inp)
    oc.shape = sh.replace(top_p=p)
    hq = h * sh.group + 1
    _, topp_o, _ = oracle.decode(oc, inp["q_pre"], inp["seq_len"], inp["w_q"], heads=[hq])
    gset = bitmask_to_sets(g["bitmask"][0], [12000] * (sh.n_retrieval * sh.group))[sh.group + 1]
    assert np.array_equal(gset, topp_o[(0, hq)]), (len(gset), len(topp_o[(0, hq)]))


@pytest.mark.parametrize("p", [0.5, 0.77])
def test_decode_all_scores_equal(p):
    """Every indexer key identical: one bucket holds all 20000 scores (more than
    the leader's candidate buffer), so the exact solve scans every score; the
    kept set is the first ceil(p * L) tokens."""
    inp = _small(ctx=20000, needles=0)
    sh = inp["shape"]
    for h in sh.retrieval:
        inp["k_pre"][0, :, h] = inp["k_pre"][0, 0, h]
    g = run_gpu_decode(inp, top_p=p)
    L = 20000
    want = int(np.ceil(p * L - 1e-9))
    sets = bitmask_to_sets(g["bitmask"][0], [L] * (sh.n_retrieval * sh.group))
    for s in sets:
        assert np.array_equal(s, np.arange(want)), (len(s), want)
    check_decode_parity(inp, top_p=p)


def test_decode_tiny_p_keeps_the_top_token():
    # p far below any single token's probability: the set is the top token
    inp = _small(ctx=3000, needles=8)
    st = check_decode_parity(inp, top_p=1e-6)
    assert np.all(st["counts"] == 1), st["counts"]


def test_decode_many_needles_second_tier():
    # every other token a needle: more than 4096 scores lie within 8 of the
    # maximum, so the selection collects a lower rung's scores in a second pass
    # (or falls back to the histogram); both must stay exact
    inp = _small(ctx=20000, needles=10000)
    st = check_decode_parity(inp, top_p=0.9)
    assert st["exact"] >= st["heads"] - 1


@pytest.mark.parametrize("case", ["needles_p03", "needles_p09", "needles_p0999", "flat", "ragged",
                                  "many_needles", "full_128k", "full_1m"])
def test_decode_without_bitmask_matches(case):
    """Without a bitmask to write, a selection settled over the top-rung items
    reads only those items in its tail. The kept counts must equal those of the
    call that writes the bitmask; so must the output, bitwise where each CTA's
    scores fit in shared memory (the kept rows are then attended in the same
    groups), within the bf16 tolerance at 1M (grouped per staged chunk there)."""
    p = None
    if case.startswith("needles"):
        inp = _small(ctx=5000, needles=16)
        p = {"needles_p03": 0.3, "needles_p09": 0.9, "needles_p0999": 0.999}[case]
    elif case == "flat":
        inp, p = _small(ctx=20000, needles=0), 0.8
    elif case == "ragged":
        w = workload("ragged_decode_b8_8k_32k_bf16", shape_batch=5, ctx=(1, 9000), needles=4)
        inp = make_decode_inputs(w, max_ctx=9100)
        inp["seq_len"] = np.array([1, 37, 2100, 2113, 9000], dtype=np.int32)
    elif case == "many_needles":
        inp, p = _small(ctx=20000, needles=10000), 0.9
    elif case == "full_128k":
        inp = make_decode_inputs(workload("decode_128k_bf16"))
    else:
        inp = make_decode_inputs(workload("decode_1m_bf16"))
    a = run_gpu_decode(inp, top_p=p)
    b = run_gpu_decode(inp, top_p=p, with_bitmask=False)
    assert a["status"] == 0 and b["status"] == 0
    assert np.array_equal(a["count"], b["count"])
    if case != "full_1m":
        assert np.array_equal(a["out"], b["out"])
    else:
        atol, rtol = TOL["bf16"]
        assert np.all(np.abs(a["out"] - b["out"]) <= atol + rtol * np.abs(a["out"]))


def test_decode_workspace_needs_no_initialisation():
    """Completion flags are cleared by their owners inside every call, so a
    workspace full of leftovers gives the same result as a zeroed one: every
    byte 0xFF, and the raised flags (value 1) a previous call leaves behind."""
    inp = _small(ctx=6000, needles=8)
    ref = run_gpu_decode(inp, top_p=0.9, ws_fill=0)
    got = run_gpu_decode(inp, top_p=0.9, ws_fill=0xFF)
    assert got["status"] == 0
    assert np.array_equal(got["out"], ref["out"])
    assert torch.equal(got["bitmask"], ref["bitmask"])
    # a second call on the same workspace, after a call with another query
    lay, sh = got["layer"], got["shape"]
    dev = torch.device("cuda")
    seq = torch.from_numpy(inp["seq_len"]).to(dev)
    w_q = inp["w_q"].to(dev)
    out = torch.empty((1, sh.n_q_heads, sh.head_dim), dtype=torch.bfloat16, device=dev)
    q_other = torch.randn(inp["q_pre"].shape, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    lay.decode(q_other.to(dev), seq, w_q, out, max_seq_len=6000)
    lay.decode(inp["q_pre"].to(dev), seq, w_q, out, max_seq_len=6000)
    torch.cuda.synchronize()
    assert lay.device_status() == 0
    assert np.array_equal(out.double().cpu().numpy(), ref["out"])


def test_bounded_wait_expiry_sets_timeout_and_returns():
    """The decode step's in-kernel waits are bounded: armed through the test
    hook, a call waits for flags that never reach the awaited value, gives up
    after a few thousand polls, sets RTP_DEV_TIMEOUT and returns; the GPU
    stays usable and the next call is correct again."""
    import head_wise_sparse_local_b200 as rtp
    inp = _small(ctx=3000, needles=4)
    g = run_gpu_decode(inp, top_p=0.9)
    lay = g["layer"]
    sh = g["shape"]
    dev = torch.device("cuda")
    q = inp["q_pre"].to(dev)
    seq = torch.from_numpy(inp["seq_len"]).to(dev)
    w_q = inp["w_q"].to(dev)
    out = torch.empty((1, sh.n_q_heads, sh.head_dim), dtype=torch.bfloat16, device=dev)
    rtp.rtp_debug_wait_expiry(2000)
    lay.decode(q, seq, w_q, out, max_seq_len=3000)
    torch.cuda.synchronize()
    assert lay.device_status() & rtp.RTP_DEV_TIMEOUT
    lay.status.zero_()
    lay.decode(q, seq, w_q, out, max_seq_len=3000)  # not armed any more
    torch.cuda.synchronize()
    assert lay.device_status() == 0
    assert np.array_equal(out.double().cpu().numpy(), g["out"])


@pytest.mark.parametrize("k", [1, 16, 300, 4999, 7000])
def test_decode_static_topk(k):
    """Static top-k (the pages' fixed-budget baseline): each retrieval q head
    keeps exactly min(k, L) tokens, the highest scores, ties to the lower index
    (k above the 16 needles of a head and above the context length included)."""
    inp = _small(ctx=5000, needles=16, shape_top_k=k)
    st = check_decode_parity(inp)
    assert st["exact"] >= st["heads"] - 1
    assert np.all(st["counts"] == min(k, 5000)), st["counts"]


def test_decode_static_topk_tie_block():
    """The k-th score sits inside a block of 300 identical keys: the lowest
    indices of the block are kept, bit for bit."""
    inp = _small(ctx=5000, needles=8, shape_top_k=150)
    sh = inp["shape"]
    h = sh.retrieval[0]
    src = int(inp["needles"][0][0][0])
    inp["k_pre"][0, 100:400, h] = inp["k_pre"][0, src, h]
    g = run_gpu_decode(inp)
    oc = oracle_cache_from_inputs(inp)
    _, topk_o, _ = oracle.decode(oc, inp["q_pre"], inp["seq_len"], inp["w_q"], heads=[h * sh.group])
    gset = bitmask_to_sets(g["bitmask"][0], [5000] * (sh.n_retrieval * sh.group))[0]
    assert np.array_equal(gset, topk_o[(0, h * sh.group)]), (len(gset), len(topk_o[(0, h * sh.group)]))


@pytest.mark.parametrize("k", [64, 4096])
def test_decode_static_topk_128k(k):
    inp = make_decode_inputs(workload("decode_128k_bf16", shape_top_k=k))
    st = check_decode_parity(inp)
    assert st["exact"] >= st["heads"] - 1
    assert np.all(st["counts"] == k)


def test_decode_static_topk_ragged():
    inp = make_decode_inputs(workload("ragged_decode_b8_8k_32k_bf16", shape_top_k=1000))
    st = check_decode_parity(inp)
    assert np.all(st["counts"] == 1000)
