"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and compare with the fp64 oracle under the layer's stated tolerances.

Selection: the kept index sets must match exactly, except for tokens whose
indexer probability lies within 1e-6 of the probability of the last token the
oracle admitted; and when the oracle's cumulative mass at its cut is itself
within 1e-6 of p, the two cuts may differ by one token.

Outputs: |gpu - oracle| <= atol + rtol * |oracle| with (2e-2, 1e-2) for bf16
and (1e-5, 1e-5) for fp32, against the oracle evaluated on the GPU's own kept
set (identical to the oracle's own set whenever the selections agree).

Every decode parity check also repeats the call without a bitmask (the call
the benchmark times, whose tail reads only the top-rung items when it can) and
holds its kept counts and its output to the same oracle reference.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle import OracleCache

SEL_EPS = 1e-6
TOL = {"bf16": (2e-2, 1e-2), "fp32": (1e-5, 1e-5)}


def bitmask_to_sets(mask: torch.Tensor, n_valid) -> list:
    """mask [NR, words] uint32 (as int32 tensor) -> list of index arrays."""
    m = mask.cpu().numpy().view(np.uint32)
    out = []
    for row, n in zip(m, n_valid):
        bits = np.unpackbits(row.view(np.uint8), bitorder="little")
        out.append(np.nonzero(bits[:n])[0])
    return out


def compare_selection(scores: np.ndarray, p: float, gpu_set: np.ndarray, oracle_set: np.ndarray):
    """Returns (exact, n_diff).  Raises AssertionError on a disallowed difference."""
    gs, os_ = set(gpu_set.tolist()), set(oracle_set.tolist())
    if gs == os_:
        return True, 0
    s = scores.astype(np.float64)
    P = np.exp(s - s.max())
    P /= P.sum()
    order = np.lexsort((np.arange(len(s)), -P))
    cum = np.cumsum(P[order])
    k = len(oracle_set)
    p_cut = P[order[k - 1]]
    cum_cut = cum[k - 1]
    boundary_cut = abs(cum_cut - p) <= SEL_EPS or (k >= 2 and abs(cum[k - 2] - p) <= SEL_EPS)
    diff = sorted(gs ^ os_)
    bad = [j for j in diff if abs(P[j] - p_cut) > SEL_EPS]
    if bad and boundary_cut and len(diff) == 1:
        bad = []
    assert not bad, (f"selection differs beyond tolerance: {len(diff)} tokens differ, e.g. "
                     f"{[(j, P[j], p_cut) for j in bad[:5]]}; |gpu|={len(gs)} |oracle|={len(os_)}")
    return False, len(diff)


def kidx_bound(inp, b: int, r: int, rows) -> np.ndarray:
    """Allowed |GPU - oracle| of stored indexer keys [len(rows), d]: the kernel
    accumulates W_k k_pre in fp32 (D products: error at most D 2^-24 sum|w k|)
    and rounds to the storage type, the oracle rounds the exact value; one
    storage rounding step (2^-7 relative for bf16, 2^-23 for fp32) on top."""
    sh = inp["shape"]
    h = sorted(sh.retrieval)[r]
    kp = np.abs(inp["k_pre"][b, np.asarray(rows), h].double().numpy())
    w = np.abs(inp["w_k"][r].double().numpy())
    acc = kp @ w.T
    exact = np.abs(inp["k_pre"][b, np.asarray(rows), h].double().numpy() @ inp["w_k"][r].double().numpy().T)
    rel = 2.0 ** -7 if sh.dtype == "bf16" else 2.0 ** -23
    return sh.head_dim * 2.0 ** -24 * acc * (1 + rel) + exact * rel + 1e-30


def oracle_cache_from_inputs(inp) -> OracleCache:
    sh = inp["shape"]
    c = OracleCache(sh, inp["max_ctx"])
    c.append_in_place(inp["k_pre"], inp["v"], inp["seq_len"], inp["w_k"])
    return c


def append_context(lay, inp, w_k, n_rows=None, dev="cuda"):
    """Append each sequence's context rows [0, n_rows[b]) (default seq_len[b])
    to the layer's cache.  In ring mode every sequence is appended on its own
    (a batch-1 view of its cache slice), so rows past its own length never
    take ring slots of its window."""
    import head_wise_sparse_local_b200 as rtp
    sh = inp["shape"]
    n_rows = inp["seq_len"] if n_rows is None else n_rows
    if not lay.ring:
        T = int(max(n_rows))
        lay.append(inp["k_pre"][:, :T].contiguous().to(dev), inp["v"][:, :T].contiguous().to(dev),
                   torch.zeros(sh.batch, dtype=torch.int32, device=dev), w_k)
        return
    c = lay.cfg
    cfg1 = rtp.rtp_layer_cfg.from_buffer_copy(c)
    cfg1.batch = 1
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    for b in range(sh.batch):
        L = int(n_rows[b])
        cache1 = rtp.rtp_cache(lay.k[b].data_ptr(), lay.v[b].data_ptr(), lay.kidx[b].data_ptr(),
                               lay.status.data_ptr())
        kp = inp["k_pre"][b:b + 1, :L].contiguous().to(dev)
        vv = inp["v"][b:b + 1, :L].contiguous().to(dev)
        rtp.rtp_append_kv(cfg1, cache1, kp, vv, zero, L, w_k)
        torch.cuda.synchronize()


def run_gpu_decode(inp, top_p=None, append_last_separately=True, with_bitmask=True,
                   also_timed_path=False, local_cap=0, ws_fill=None):
    """Fill a device cache with the context, append the decode token, decode.

    Returns dict(out [B,Hq,D] float64 numpy, bitmask, count, status, layer);
    with_bitmask=False passes no bitmask (bitmask None in the result).
    also_timed_path=True repeats the call without a bitmask on the same cache
    (the call the benchmark times) and adds out_timed / count_timed.
    local_cap > 0 runs the cache in ring mode; ws_fill fills the decode
    workspace with that byte first (it needs no initialisation)."""
    from head_wise_sparse_local_b200 import Layer
    sh = inp["shape"]
    if top_p is not None:
        sh = sh.replace(top_p=top_p)
    dev = torch.device("cuda")
    Lmax = inp["max_ctx"]
    lay = Layer(sh, Lmax, device=dev, local_cap=local_cap)
    if ws_fill is not None:
        lay.ws_decode.fill_(ws_fill)
    k_pre = inp["k_pre"].to(dev)
    v = inp["v"].to(dev)
    w_q = inp["w_q"].to(dev)
    w_k = inp["w_k"].to(dev)
    seq = torch.from_numpy(inp["seq_len"]).to(dev)
    if lay.ring:
        append_context(lay, inp, w_k, dev=dev)
    else:
        lay.append(k_pre, v, torch.zeros(sh.batch, dtype=torch.int32, device=dev), w_k)
    if append_last_separately:
        # re-append each sequence's last token as a decode step would (T = 1)
        last = (seq - 1).to(torch.int32)
        idx = last.long()
        bidx = torch.arange(sh.batch, device=dev)
        k1 = k_pre[bidx, idx][:, None].contiguous()
        v1 = v[bidx, idx][:, None].contiguous()
        lay.append(k1, v1, last, w_k)
    q = inp["q_pre"].to(dev)
    out = torch.empty((sh.batch, sh.n_q_heads, sh.head_dim), dtype=sh.torch_dtype, device=dev)
    words = (Lmax + 31) // 32
    NR = sh.n_retrieval * sh.group
    bm = torch.zeros((sh.batch, max(NR, 1), words), dtype=torch.int32, device=dev)
    cnt = torch.full((sh.batch, max(NR, 1)), -1, dtype=torch.int32, device=dev)
    if not with_bitmask:
        bm = None
    Lh = int(inp["seq_len"].max())
    lay.decode(q, seq, w_q, out, max_seq_len=Lh, sel_bitmask=bm, sel_count=cnt)
    res = dict(out=out.double().cpu().numpy(), bitmask=bm, count=cnt.cpu().numpy(), layer=lay, shape=sh)
    if with_bitmask and also_timed_path:
        # the call the benchmark times: no bitmask, kept counts only
        out2 = torch.empty_like(out)
        cnt2 = torch.full_like(cnt, -1)
        lay.decode(q, seq, w_q, out2, max_seq_len=Lh, sel_bitmask=None, sel_count=cnt2)
        res["out_timed"] = out2.double().cpu().numpy()
        res["count_timed"] = cnt2.cpu().numpy()
    torch.cuda.synchronize()
    res["status"] = lay.device_status()
    return res


def check_decode_parity(inp, top_p=None, oc=None, local_cap=0):
    """Full parity check of one decode step; returns stats."""
    sh = inp["shape"] if top_p is None else inp["shape"].replace(top_p=top_p)
    g = run_gpu_decode(inp, top_p, also_timed_path=True, local_cap=local_cap)
    assert g["status"] == 0, f"device status {g['status']}"
    oc = oc or oracle_cache_from_inputs(inp)
    oc.shape = sh
    out_o, topp_o, final_o = oracle.decode(oc, inp["q_pre"], inp["seq_len"], inp["w_q"])
    G = sh.group
    override = {}
    n_exact, n_heads, n_diff_tok = 0, 0, 0
    for b in range(sh.batch):
        L = int(inp["seq_len"][b])
        sets = bitmask_to_sets(g["bitmask"][b], [L] * (sh.n_retrieval * G))
        for r, h in enumerate(sh.retrieval):
            for gg in range(G):
                hq = h * G + gg
                rg = r * G + gg
                gset = sets[rg]
                assert g["count"][b, rg] == len(gset), (g["count"][b, rg], len(gset))
                qi = oracle.indexer_project(inp["q_pre"][b, hq], inp["w_q"][r])
                s = oracle.indexer_scores(qi, oc.indexer_keys(b, r, L))
                exact, nd = compare_selection(s, sh.top_p, gset, topp_o[(b, hq)])
                n_heads += 1
                n_exact += int(exact)
                n_diff_tok += nd
                if not exact:
                    sw = oracle.sink_window_set(L - 1, sh.n_sink, sh.window)
                    override[(b, hq)] = np.union1d(gset, sw)
    ref = out_o
    if override:
        ref2, _, _ = oracle.decode(oc, inp["q_pre"], inp["seq_len"], inp["w_q"],
                                   rows_override=override)
        ref = ref2
    atol, rtol = TOL[sh.dtype]
    err = np.abs(g["out"] - ref)
    lim = atol + rtol * np.abs(ref)
    worst = float((err / lim).max())
    assert np.all(err <= lim), f"output mismatch: max err {err.max():.3e}, worst ratio {worst:.3f}"
    # The timed call (no bitmask) runs the same selection: its kept counts must
    # equal the bitmask call's set sizes, and its output must match the oracle
    # on that set directly (not only through the bitmask call).
    assert np.array_equal(g["count_timed"], g["count"]), (g["count_timed"], g["count"])
    err_t = np.abs(g["out_timed"] - ref)
    worst_t = float((err_t / lim).max())
    assert np.all(err_t <= lim), f"timed-path output mismatch: max err {err_t.max():.3e}, worst {worst_t:.3f}"
    return dict(heads=n_heads, exact=n_exact, diff_tokens=n_diff_tok, worst_ratio=max(worst, worst_t),
                max_abs_err=float(max(err.max(), err_t.max())), counts=g["count"])


def run_gpu_prefill(inp, top_p=None, local_cap=0, with_bitmask=True):
    """Append the context and the chunk, then run one prefill over the chunk.

    Returns out [B, T, Hq, D] float64, bitmask [B, NR, T, words], count [B, NR, T].
    local_cap > 0 runs the cache in ring mode (the context before the chunk
    and the chunk are appended separately, as a serving loop would)."""
    from head_wise_sparse_local_b200 import Layer
    sh = inp["shape"]
    if top_p is not None:
        sh = sh.replace(top_p=top_p)
    dev = torch.device("cuda")
    Lmax = inp["max_ctx"]
    T = inp["T"]
    lay = Layer(sh, Lmax, device=dev, prefill_T=T, local_cap=local_cap)
    start = torch.from_numpy(inp["start_pos"]).to(dev)
    n_ctx = int(inp["start_pos"].max()) + T
    w_k = inp["w_k"].to(dev)
    if lay.ring:
        s0 = int(inp["start_pos"][0])
        assert np.all(inp["start_pos"] == s0)
        if s0 > 0:
            append_context(lay, inp, w_k, n_rows=np.full(sh.batch, s0), dev=dev)
        lay.append(inp["k_pre"][:, s0:n_ctx].contiguous().to(dev), inp["v"][:, s0:n_ctx].contiguous().to(dev),
                   start, w_k)
    else:
        lay.append(inp["k_pre"][:, :n_ctx].contiguous().to(dev), inp["v"][:, :n_ctx].contiguous().to(dev),
                   torch.zeros(sh.batch, dtype=torch.int32, device=dev), w_k)
    q = inp["q_pre"].to(dev)
    out = torch.empty((sh.batch, T, sh.n_q_heads, sh.head_dim), dtype=sh.torch_dtype, device=dev)
    NR = max(sh.n_retrieval * sh.group, 1)
    words = (Lmax + 31) // 32
    bm = torch.zeros((sh.batch, NR, T, words), dtype=torch.int32, device=dev) if with_bitmask else None
    cnt = torch.full((sh.batch, NR, T), -1, dtype=torch.int32, device=dev)
    tau = torch.zeros((sh.batch, NR, T), dtype=torch.float32, device=dev)
    jcut = torch.zeros((sh.batch, NR, T), dtype=torch.int32, device=dev)
    lay.prefill(q, start, inp["w_q"].to(dev), out, sel_bitmask=bm, sel_tau=tau, sel_jcut=jcut,
                sel_count=cnt)
    torch.cuda.synchronize()
    return dict(out=out.double().cpu().numpy(), bitmask=bm, count=cnt.cpu().numpy(),
                tau=tau.cpu().numpy(), jcut=jcut.cpu().numpy(), status=lay.device_status(),
                layer=lay, shape=sh)


def check_prefill_parity(inp, rows=None, top_p=None, g=None, local_cap=0):
    """Selection sets (per row, per retrieval q head) and outputs of the GPU
    prefill against the oracle, over `rows` (default: every row)."""
    sh = inp["shape"] if top_p is None else inp["shape"].replace(top_p=top_p)
    g = g or run_gpu_prefill(inp, top_p, local_cap=local_cap)
    assert g["status"] == 0, f"device status {g['status']}"
    T = inp["T"]
    rows = list(range(T)) if rows is None else list(rows)
    oc = OracleCache(sh, inp["max_ctx"])
    n_ctx = inp["start_pos"] + T
    oc.append_in_place(inp["k_pre"], inp["v"], n_ctx, inp["w_k"])
    out_o, topp_o = oracle.prefill(oc, inp["q_pre"], inp["start_pos"], inp["w_q"], rows=rows)
    G = sh.group
    bm = g["bitmask"].cpu().numpy().view(np.uint32)
    override = {}
    n_exact = n_heads = 0
    for b in range(sh.batch):
        for t in rows:
            i = int(inp["start_pos"][b]) + t
            for r, h in enumerate(sh.retrieval):
                for gg in range(G):
                    hq = h * G + gg
                    rg = r * G + gg
                    bits = np.unpackbits(bm[b, rg, t].view(np.uint8), bitorder="little")[: i + 1]
                    gset = np.nonzero(bits)[0]
                    assert g["count"][b, rg, t] == len(gset), (b, t, hq, g["count"][b, rg, t], len(gset))
                    qi = oracle.indexer_project(inp["q_pre"][b, t, hq], inp["w_q"][r])
                    s = oracle.indexer_scores(qi, oc.indexer_keys(b, r, i + 1))
                    exact, _ = compare_selection(s, sh.top_p, gset, topp_o[(b, t, hq)])
                    n_heads += 1
                    n_exact += int(exact)
                    if not exact:
                        override[(b, t, hq)] = np.union1d(gset, oracle.sink_window_set(i, sh.n_sink, sh.window))
    if override:
        out_o, _ = oracle.prefill(oc, inp["q_pre"], inp["start_pos"], inp["w_q"], rows=rows,
                                  rows_override=override)
    atol, rtol = TOL[sh.dtype]
    worst = 0.0
    for b in range(sh.batch):
        for t in rows:
            ref = out_o[(b, t)]
            got = g["out"][b, t]
            err = np.abs(got - ref)
            lim = atol + rtol * np.abs(ref)
            worst = max(worst, float((err / lim).max()))
            assert np.all(err <= lim), (b, t, float(err.max()), np.unravel_index(np.argmax(err / lim), err.shape))
    return dict(heads=n_heads, exact=n_exact, worst_ratio=worst, g=g)
