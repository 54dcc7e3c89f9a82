"""Layer-level pins of the oracle.

(a) p = 1 with window >= context reduces to dense causal attention;
(b) local heads with window >= context reduce to dense attention;
both checked against torch's scaled_dot_product_attention in fp64 (a textbook
library routine).  Also: one-token context gives o = v_0; the indexer scale
1/4 through a hand-derived two-token case; needle dominance on the tiny decode
workload; prefill rows agree with decode steps; kept-set size monotone in p.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import OracleCache
from synth import LayerShape, make_decode_inputs, make_prefill_inputs, workload

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _shape(**kw):
    base = dict(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=32, n_sink=2, window=4,
                top_p=0.9, retrieval=(0,), dtype="fp32")
    base.update(kw)
    return LayerShape(**base)


def _rand_layer(shape, L, seed):
    g = torch.Generator().manual_seed(seed)
    dt = shape.torch_dtype
    B, Hq, Hkv, D, R = shape.batch, shape.n_q_heads, shape.n_kv_heads, shape.head_dim, shape.n_retrieval
    k = torch.randn((B, L, Hkv, D), generator=g).to(dt)
    v = torch.randn((B, L, Hkv, D), generator=g).to(dt)
    q = torch.randn((B, L, Hq, D), generator=g).to(dt)
    wq = torch.randn((R, 16, D), generator=g) / D ** 0.5
    wk = torch.randn((R, 16, D), generator=g) / D ** 0.5
    return q, k, v, wq, wk


def _dense_reference(shape, q, k, v, L):
    """Causal dense attention over the stored (RoPE'd, rounded) keys, via
    torch SDPA in fp64.  RoPE and rounding come from the separately pinned
    oracle helpers."""
    B, Hq, Hkv, D, G = shape.batch, shape.n_q_heads, shape.n_kv_heads, shape.head_dim, shape.group
    pos = np.arange(L)
    out = np.zeros((B, L, Hq, D))
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            qr = oracle.rope(q[b, :, hq].double().numpy(), pos, shape.rope_base)
            kr = oracle.round_storage(oracle.rope(k[b, :, h].double().numpy(), pos, shape.rope_base),
                                      shape.dtype)
            vv = v[b, :, h].double()
            o = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(qr)[None], torch.from_numpy(kr)[None], vv[None], is_causal=True)
            out[b, :, hq] = o[0].numpy()
    return out


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_reduction_a_dense_when_p1_and_wide_window(dtype):
    L = 23
    sh = _shape(top_p=1.0, window=L, n_sink=3, dtype=dtype, retrieval=(0, 1))
    q, k, v, wq, wk = _rand_layer(sh, L, 1)
    c = OracleCache(sh, L)
    c.append(k, v, [0, 0], L, wk)
    out, topp = oracle.prefill(c, q, [0, 0], wq)
    ref = _dense_reference(sh, q, k, v, L)
    for b in range(sh.batch):
        for t in range(L):
            assert np.allclose(out[(b, t)], ref[b, t], atol=1e-12, rtol=1e-12)
    # decode at every length agrees too
    for Lc in [1, 2, 7, L]:
        od, _, _ = oracle.decode(c, q[:, Lc - 1], [Lc, Lc], wq)
        assert np.allclose(od, ref[:, Lc - 1], atol=1e-12)


def test_reduction_b_local_dense_when_window_covers_context():
    L = 19
    sh = _shape(top_p=0.5, window=L + 5, n_sink=0, retrieval=(0,))
    q, k, v, wq, wk = _rand_layer(sh, L, 2)
    c = OracleCache(sh, L)
    c.append(k, v, [0, 0], L, wk)
    out, _ = oracle.prefill(c, q, [0, 0], wq)
    ref = _dense_reference(sh, q, k, v, L)
    G = sh.group
    for b in range(sh.batch):
        for t in range(L):
            # local KV head 1 -> q heads G..2G-1; retrieval heads also see the full window
            assert np.allclose(out[(b, t)][G:], ref[b, t][G:], atol=1e-12)
            assert np.allclose(out[(b, t)][:G], ref[b, t][:G], atol=1e-12)


def test_one_token_context_returns_v0():
    sh = _shape(batch=1, dtype="bf16")
    q, k, v, wq, wk = _rand_layer(sh, 1, 3)
    c = OracleCache(sh, 1)
    c.append(k, v, [0], 1, wk)
    out, topp, final = oracle.decode(c, q[:, 0], [1], wq)
    for hq in range(sh.n_q_heads):
        assert np.array_equal(out[0, hq], v[0, 0, hq // sh.group].double().numpy())
        assert list(final[(0, hq)]) == [0]


def test_indexer_scale_two_token_golden():
    d = json.load(open(os.path.join(GOLD, "indexer_two_token.json")))
    D, qc, kc = d["head_dim"], d["q_coord"], d["k_coord"]
    for case in d["cases"]:
        sh = LayerShape(batch=1, n_q_heads=1, n_kv_heads=1, head_dim=D, n_sink=0, window=1,
                        top_p=case["p"], retrieval=(0,), dtype="fp32")
        wq = torch.zeros((1, 16, D))
        wq[0, 0, qc] = 1.0
        wk = torch.zeros((1, 16, D))
        wk[0, 0, kc] = 1.0
        k = torch.zeros((1, 2, 1, D))
        for j in range(2):
            k[0, j, 0, kc] = d["k_values"][j]
            k[0, j, 0, qc] = d["k_junk"][j]
        v = torch.randn((1, 2, 1, D))
        q = torch.zeros((1, 1, D))
        q[0, 0, qc] = d["q_value"]
        q[0, 0, kc] = d["q_junk"]
        c = OracleCache(sh, 2)
        c.append(k, v, [0], 2, wk)
        # decode query at position 1 sees [0, 1]
        out, topp, final = oracle.decode(c, q, [2], wq)
        assert list(topp[(0, 0)]) == case["kept"], case


@pytest.mark.parametrize("width", [0, 1, 2, 3])
def test_indexer_width_golden(width):
    """Score scale 1/sqrt(d) at every width of the dimension ablation, with the
    projection into the last of the d indexer dims (hand-derived, tests/golden)."""
    d = json.load(open(os.path.join(GOLD, "indexer_widths.json")))
    D, qc, kc = d["head_dim"], d["q_coord"], d["k_coord"]
    w = d["widths"][width]
    n = w["idx_dim"]
    for case in d["cases"]:
        sh = LayerShape(batch=1, n_q_heads=1, n_kv_heads=1, head_dim=D, n_sink=0, window=1,
                        top_p=case["p"], retrieval=(0,), dtype="fp32", idx_dim=n)
        wq = torch.zeros((1, n, D))
        wq[0, n - 1, qc] = 1.0
        wk = torch.zeros((1, n, D))
        wk[0, n - 1, kc] = 1.0
        k = torch.zeros((1, 2, 1, D), dtype=torch.float64)
        for j in range(2):
            k[0, j, 0, kc] = w["k_values"][j]
            k[0, j, 0, qc] = d["k_junk"][j]
        v = torch.randn((1, 2, 1, D))
        q = torch.zeros((1, 1, D))
        q[0, 0, qc] = d["q_value"]
        q[0, 0, kc] = d["q_junk"]
        c = OracleCache(sh, 2)
        c.append(k, v, [0], 2, wk)
        _, topp, _ = oracle.decode(c, q, [2], wq)
        assert list(topp[(0, 0)]) == case["kept"], (n, case)


@pytest.mark.parametrize("path", ["append", "append_in_place", "prefill"])
def test_indexer_key_storage_rounding_golden(path):
    """The stored indexer key is rounded to the cache's storage type before it
    is scored: a bf16 layer ties two tokens that an fp32 layer separates by
    2^-11, which flips the kept set (hand-derived, tests/golden)."""
    d = json.load(open(os.path.join(GOLD, "indexer_bf16_rounding.json")))
    D = d["head_dim"]
    for case in d["cases"]:
        L = case["L"]
        sh = LayerShape(batch=1, n_q_heads=1, n_kv_heads=1, head_dim=D, n_sink=0, window=1,
                        top_p=case["p"], retrieval=(0,), dtype=case["dtype"])
        wq = torch.zeros((1, 16, D))
        wq[0, 0, 0] = 1.0
        wk = torch.zeros((1, 16, D))
        wk[0, 0] = torch.tensor(d["w_k_row0"], dtype=torch.float32)
        k = torch.zeros((1, L, 1, D), dtype=sh.torch_dtype)
        for j in range(L):
            k[0, j, 0, j] = 1.0
        v = torch.randn((1, L, 1, D)).to(sh.torch_dtype)
        q = torch.zeros((1, 1, D), dtype=sh.torch_dtype)
        q[0, 0, 0] = 1.0
        c = OracleCache(sh, L)
        if path == "append_in_place":
            c.append_in_place(k, v, [L], wk)
        else:
            c.append(k, v, [0], L, wk)
        stored = c.indexer_keys(0, 0, L)[:, 0]
        assert list(stored) == d["stored_" + case["dtype"]][:L], (case, stored)
        assert np.all(c.indexer_keys(0, 0, L)[:, 1:] == 0.0)
        if path == "prefill":
            _, topp = oracle.prefill(c, q[:, None].expand(1, L, 1, D).contiguous(), [0], wq, rows=[L - 1])
            kept = topp[(0, L - 1, 0)]
        else:
            _, topp, _ = oracle.decode(c, q, [L], wq)
            kept = topp[(0, 0)]
        assert list(kept) == case["kept"], (path, case)


def test_sink_window_golden():
    d = json.load(open(os.path.join(GOLD, "sink_window.json")))
    for c in d["cases"]:
        assert list(oracle.sink_window_set(c["i"], c["S"], c["W"])) == c["rows"], c


def test_local_head_attends_exactly_sink_and_window():
    """A local head's output equals SDPA over the hand-listed rows (the value
    rows carry one-hot markers so the attended set shows in the output)."""
    d = json.load(open(os.path.join(GOLD, "sink_window.json")))
    for c in d["cases"]:
        i, S, W = c["i"], c["S"], c["W"]
        L = i + 1
        D = 128
        sh = LayerShape(batch=1, n_q_heads=1, n_kv_heads=1, head_dim=D, n_sink=S, window=W,
                        top_p=0.5, retrieval=(), dtype="fp32")
        g = torch.Generator().manual_seed(i)
        k = torch.randn((1, L, 1, D), generator=g)
        v = torch.zeros((1, L, 1, D))
        for j in range(L):
            v[0, j, 0, j % D] = 1.0
        q = torch.randn((1, 1, D), generator=g)
        cache = OracleCache(sh, L)
        cache.append(k, v, [0], L, torch.zeros((0, 16, D)))
        out, _, final = oracle.decode(cache, q, [L], torch.zeros((0, 16, D)))
        assert list(final[(0, 0)]) == c["rows"]
        rows = c["rows"]
        qr = oracle.rope(q[0, 0].double().numpy(), i, sh.rope_base)
        kr = oracle.round_storage(oracle.rope(k[0, rows, 0].double().numpy(), np.array(rows),
                                              sh.rope_base), "fp32")
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr)[None, None], torch.from_numpy(kr)[None], v[0, rows, 0].double()[None])
        assert np.allclose(out[0, 0], ref[0, 0].numpy(), atol=1e-12)
        support = set(np.nonzero(out[0, 0] > 0)[0].tolist())
        assert support == {j % D for j in rows}


def test_tiny_decode_needles_dominate():
    w = workload("tiny_decode_2k_fp32")
    inp = make_decode_inputs(w)
    sh = inp["shape"]
    c = OracleCache(sh, inp["max_ctx"])
    c.append_in_place(inp["k_pre"], inp["v"], inp["seq_len"], inp["w_k"])
    out, topp, final = oracle.decode(c, inp["q_pre"], inp["seq_len"], inp["w_q"])
    G = sh.group
    for (b, hq), kept in topp.items():
        r = sh.retrieval.index(hq // G)
        needles = inp["needles"][b][r]
        mine = {int(j) for n, j in enumerate(needles) if n % G == hq % G}
        assert len(kept) >= 1 and set(kept.tolist()) <= mine, (hq, kept, mine)
    assert np.all(np.isfinite(out))


def test_prefill_rows_match_decode_steps():
    sh = _shape(batch=1, top_p=0.7, window=3, n_sink=1, retrieval=(1,), dtype="bf16")
    L = 17
    q, k, v, wq, wk = _rand_layer(sh, L, 5)
    c = OracleCache(sh, L)
    c.append(k, v, [0], L, wk)
    out, topp = oracle.prefill(c, q, [0], wq)
    for t in range(L):
        od, tp, _ = oracle.decode(c, q[:, t], [t + 1], wq)
        assert np.array_equal(od[0], out[(0, t)])
        for hq in range(sh.group, 2 * sh.group):
            assert list(tp[(0, hq)]) == list(topp[(0, t, hq)])


def test_prefill_chunk_after_context_matches_single_chunk():
    sh = _shape(batch=1, top_p=0.8, window=5, n_sink=2, retrieval=(0,), dtype="fp32")
    L = 20
    q, k, v, wq, wk = _rand_layer(sh, L, 6)
    c1 = OracleCache(sh, L)
    c1.append(k, v, [0], L, wk)
    o1, t1 = oracle.prefill(c1, q, [0], wq)
    c2 = OracleCache(sh, L)
    c2.append(k[:, :12], v[:, :12], [0], 12, wk)
    c2.append(k[:, 12:], v[:, 12:], [12], 8, wk)
    o2, t2 = oracle.prefill(c2, q[:, 12:], [12], wq)
    for t in range(8):
        assert np.array_equal(o1[(0, 12 + t)], o2[(0, t)])


def test_layer_kept_size_monotone_in_p():
    w = workload("tiny_decode_2k_fp32")
    inp = make_decode_inputs(w)
    sh = inp["shape"]
    c = OracleCache(sh, inp["max_ctx"])
    c.append_in_place(inp["k_pre"], inp["v"], inp["seq_len"], inp["w_k"])
    prev = None
    for p in [0.5, 0.9, 0.99, 0.999999, 1.0]:
        _, topp, _ = oracle.decode(c, inp["q_pre"], inp["seq_len"], inp["w_q"], top_p=p)
        sizes = {k: len(v) for k, v in topp.items()}
        if prev is not None:
            assert all(sizes[k] >= prev[k] for k in sizes)
        prev = sizes
    assert all(s == inp["seq_len"][0] for s in prev.values())


def test_synth_is_deterministic_and_needles_outside_sink_window():
    w = workload("ragged_decode_b8_8k_32k_bf16", shape_batch=2, ctx=(300, 600), needles=5)
    a = make_decode_inputs(w)
    b = make_decode_inputs(w)
    assert torch.equal(a["k_pre"], b["k_pre"]) and np.array_equal(a["seq_len"], b["seq_len"])
    sh = a["shape"]
    for bb in range(sh.batch):
        L = int(a["seq_len"][bb])
        for pos in a["needles"][bb]:
            assert np.all(pos >= sh.n_sink) and np.all(pos < L - sh.window)
    p = make_prefill_inputs(workload("prefill_32k_bf16", needles=4), T=64)
    assert p["q_pre"].shape == (1, 64, 32, 128)


def test_recall_golden_three_keys():
    d = json.load(open(os.path.join(GOLD, "recall_three_keys.json")))
    D = d["head_dim"]
    sh = LayerShape(batch=1, n_q_heads=1, n_kv_heads=1, head_dim=D, n_sink=0, window=1,
                    top_p=0.5, retrieval=(0,), dtype="fp32")
    k = torch.tensor(d["keys"], dtype=torch.float32)[None, :, None, :]
    c = OracleCache(sh, 3)
    c.append(k, torch.zeros_like(k), [0], 3, torch.zeros((1, 16, D)))
    q = torch.tensor(d["q"], dtype=torch.float32)
    for case in d["cases"]:
        got = oracle.recall_of_rows(c, 0, 0, 2, q, case["rows"])
        assert abs(got - case["recall"]) < 1e-6, (case, got)


def test_recall_is_one_for_the_dense_reduction():
    """p = 1 with a window covering the context attends every row: recall 1."""
    L = 40
    sh = _shape(batch=1, top_p=1.0, window=L, n_sink=2, retrieval=(0,), dtype="bf16")
    q, k, v, wq, wk = _rand_layer(sh, L, 9)
    c = OracleCache(sh, L)
    c.append(k, v, [0], L, wk)
    _, _, final = oracle.decode(c, q[:, L - 1], [L], wq)
    rec = oracle.decode_recall(c, q[:, L - 1], [L], final)
    assert rec and all(abs(x - 1.0) < 1e-12 for x in rec.values())
