"""GPU parity of rtp_decode_recall (attention mass recall of a decode step's
attended rows, atlas.scime.ai summary, "Experimental setup", metrics) against
the fp64 oracle, given the top-p sets the GPU decode step wrote.

Tolerance: the kernel's base-2 logits are fp32 dot products of length D of the
RoPE'd query (fp32) with the cached keys, about 2^-24 * D * |q||k| off the
exact logit (well under 1e-5 at these magnitudes), and the sums are fp32 over
at most 2^20 terms in a tree of partials (relative error under 1e-6): a recall
in [0, 1] lands within 1e-4 of the fp64 value."""

import numpy as np
import pytest
import torch

import oracle
from parity import bitmask_to_sets, oracle_cache_from_inputs, run_gpu_decode
from synth import make_decode_inputs, workload

pytestmark = pytest.mark.gpu

TOL_RECALL = 1e-4


def _gpu_recall(g, inp):
    lay, sh = g["layer"], g["shape"]
    dev = lay.k.device
    NR = sh.n_retrieval * sh.group
    rec = torch.full((sh.batch, max(NR, 1)), -1.0, dtype=torch.float32, device=dev)
    seq = torch.from_numpy(inp["seq_len"]).to(dev)
    lay.recall(inp["q_pre"].to(dev), seq, g["bitmask"], rec, max_seq_len=int(inp["seq_len"].max()))
    torch.cuda.synchronize()
    return rec.cpu().numpy()


def _attended(sh, L, kept):
    """The decode step's attended rows of a retrieval head: its top-p set united
    with the sinks and the window."""
    sink = np.arange(min(sh.n_sink, L))
    win = np.arange(max(0, L - sh.window), L)
    return np.union1d(np.union1d(kept, sink), win)


def _check(inp, top_p=None, heads_per_seq=None):
    sh = inp["shape"] if top_p is None else inp["shape"].replace(top_p=top_p)
    g = run_gpu_decode(inp, top_p)
    assert g["status"] == 0
    rec = _gpu_recall(g, inp)
    oc = oracle_cache_from_inputs(inp)
    NR = sh.n_retrieval * sh.group
    ranks = sorted(sh.retrieval)  # rank r of the bitmask = r-th retrieval head by index
    final = {}
    for b in range(sh.batch):
        L = int(inp["seq_len"][b])
        sets = bitmask_to_sets(g["bitmask"][b], [L] * NR)
        ids = range(NR) if heads_per_seq is None else range(min(NR, heads_per_seq))
        for rq in ids:
            hq = ranks[rq // sh.group] * sh.group + rq % sh.group
            final[(b, hq)] = _attended(sh, L, sets[rq])
    ref = oracle.decode_recall(oc, inp["q_pre"], inp["seq_len"], final)
    worst = 0.0
    for (b, hq), r in ref.items():
        rq = ranks.index(hq // sh.group) * sh.group + hq % sh.group
        worst = max(worst, abs(float(rec[b, rq]) - r))
        assert 0.0 <= rec[b, rq] <= 1.0 + 1e-6
    assert worst <= TOL_RECALL, worst
    return rec, ref


@pytest.mark.parametrize("p", [0.5, 0.9, 0.99])
def test_recall_small_several_chunks(p):
    """5000-token context: three key chunks with a ragged tail."""
    inp = make_decode_inputs(workload("decode_128k_bf16", ctx=5000, needles=16))
    rec, ref = _check(inp, top_p=p)
    assert min(ref.values()) > 0.0


def test_recall_is_one_at_p_one():
    """p = 1 keeps every token: the attended rows are the whole context."""
    inp = make_decode_inputs(workload("decode_128k_bf16", ctx=3000, needles=4))
    rec, _ = _check(inp, top_p=1.0)
    assert np.allclose(rec, 1.0, atol=1e-6)


def test_recall_fp32_layer():
    inp = make_decode_inputs(workload("tiny_decode_2k_fp32"))
    _check(inp)


def test_recall_ragged_batch():
    inp = make_decode_inputs(workload("ragged_decode_b8_8k_32k_bf16"))
    _check(inp, heads_per_seq=2)


def test_recall_128k_full_size():
    inp = make_decode_inputs(workload("decode_128k_bf16"))
    _check(inp)
