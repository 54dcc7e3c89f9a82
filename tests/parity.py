"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and compare with the fp64 oracle under the layer's stated tolerances.

Selection: the kept index sets must match exactly, except for tokens whose
indexer probability lies within 1e-6 of the probability of the last token the
oracle admitted; and when the oracle's cumulative mass at its cut is itself
within 1e-6 of p, the two cuts may differ by one token.

Outputs: |gpu - oracle| <= atol + rtol * |oracle| with (2e-2, 1e-2) for bf16
and (1e-5, 1e-5) for fp32, against the oracle evaluated on the GPU's own kept
set (identical to the oracle's own set whenever the selections agree).
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


def oracle_cache_from_inputs(inp) -> OracleCache:
    sh = inp["shape"]
    c = OracleCache(sh, inp["max_ctx"])
    c.append_in_place(inp["k_pre"], inp["v"], inp["seq_len"], inp["w_k"])
    return c


def run_gpu_decode(inp, top_p=None, append_last_separately=True, with_bitmask=True):
    """Fill a device cache with the context, append the decode token, decode.

    Returns dict(out [B,Hq,D] float64 numpy, bitmask, count, status, layer);
    with_bitmask=False passes no bitmask (bitmask None in the result)."""
    from head_wise_sparse_local_b200 import Layer
    sh = inp["shape"]
    if top_p is not None:
        sh = sh.replace(top_p=top_p)
    dev = torch.device("cuda")
    Lmax = inp["max_ctx"]
    lay = Layer(sh, Lmax, device=dev)
    k_pre = inp["k_pre"].to(dev)
    v = inp["v"].to(dev)
    w_q = inp["w_q"].to(dev)
    w_k = inp["w_k"].to(dev)
    seq = torch.from_numpy(inp["seq_len"]).to(dev)
    start0 = torch.zeros(sh.batch, dtype=torch.int32, device=dev)
    lay.append(k_pre, v, start0, w_k)
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
    lay.decode(q, seq, w_q, out, max_seq_len=int(inp["seq_len"].max()), sel_bitmask=bm, sel_count=cnt)
    torch.cuda.synchronize()
    return dict(out=out.double().cpu().numpy(), bitmask=bm, count=cnt.cpu().numpy(),
                status=lay.device_status(), layer=lay, shape=sh)


def check_decode_parity(inp, top_p=None, oc=None):
    """Full parity check of one decode step; returns stats."""
    sh = inp["shape"] if top_p is None else inp["shape"].replace(top_p=top_p)
    g = run_gpu_decode(inp, top_p)
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
    return dict(heads=n_heads, exact=n_exact, diff_tokens=n_diff_tok, worst_ratio=worst,
                max_abs_err=float(err.max()), counts=g["count"])


def run_gpu_prefill(inp, top_p=None):
    """Append the context and the chunk, then run one prefill over the chunk.

    Returns out [B, T, Hq, D] float64, bitmask [B, NR, T, words], count [B, NR, T]."""
    from head_wise_sparse_local_b200 import Layer
    sh = inp["shape"]
    if top_p is not None:
        sh = sh.replace(top_p=top_p)
    dev = torch.device("cuda")
    Lmax = inp["max_ctx"]
    T = inp["T"]
    lay = Layer(sh, Lmax, device=dev, prefill_T=T)
    start = torch.from_numpy(inp["start_pos"]).to(dev)
    n_ctx = int(inp["start_pos"].max()) + T
    lay.append(inp["k_pre"][:, :n_ctx].contiguous().to(dev), inp["v"][:, :n_ctx].contiguous().to(dev),
               torch.zeros(sh.batch, dtype=torch.int32, device=dev), inp["w_k"].to(dev))
    q = inp["q_pre"].to(dev)
    out = torch.empty((sh.batch, T, sh.n_q_heads, sh.head_dim), dtype=sh.torch_dtype, device=dev)
    NR = max(sh.n_retrieval * sh.group, 1)
    words = (Lmax + 31) // 32
    bm = torch.zeros((sh.batch, NR, T, words), dtype=torch.int32, device=dev)
    cnt = torch.full((sh.batch, NR, T), -1, dtype=torch.int32, device=dev)
    tau = torch.zeros((sh.batch, NR, T), dtype=torch.float32, device=dev)
    jcut = torch.zeros((sh.batch, NR, T), dtype=torch.int32, device=dev)
    lay.prefill(q, start, inp["w_q"].to(dev), out, sel_bitmask=bm, sel_tau=tau, sel_jcut=jcut,
                sel_count=cnt)
    torch.cuda.synchronize()
    return dict(out=out.double().cpu().numpy(), bitmask=bm, count=cnt.cpu().numpy(),
                tau=tau.cpu().numpy(), jcut=jcut.cpu().numpy(), status=lay.device_status(),
                layer=lay, shape=sh)


def check_prefill_parity(inp, rows=None, top_p=None, g=None):
    """Selection sets (per row, per retrieval q head) and outputs of the GPU
    prefill against the oracle, over `rows` (default: every row)."""
    sh = inp["shape"] if top_p is None else inp["shape"].replace(top_p=top_p)
    g = g or run_gpu_prefill(inp, top_p)
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
