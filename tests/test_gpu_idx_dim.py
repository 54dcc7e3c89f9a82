"""GPU parity of the decode and prefill paths at the indexer widths of the
pages' dimension ablation (atlas.scime.ai summary, "Surprising findings":
dimension 4), d = 4, 8 and 32 beside the pages' 16: the stored indexer keys,
the kept sets and the outputs against the fp64 oracle at the same width."""

import numpy as np
import pytest

from parity import (check_decode_parity, check_prefill_parity, kidx_bound, oracle_cache_from_inputs,
                    run_gpu_decode, run_gpu_prefill)
from synth import LayerShape, make_decode_inputs, make_prefill_inputs, workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [4, 8, 32])
@pytest.mark.parametrize("p", [0.5, 0.95])
def test_decode_bf16_widths(d, p):
    # 5000 tokens: several score chunks with a ragged tail
    inp = make_decode_inputs(workload("decode_128k_bf16", ctx=5000, needles=16, shape_idx_dim=d))
    st = check_decode_parity(inp, top_p=p)
    assert st["exact"] >= st["heads"] - 1


@pytest.mark.parametrize("d", [4, 8, 32])
def test_decode_fp32_widths(d):
    sh = LayerShape(batch=2, n_q_heads=8, n_kv_heads=4, head_dim=64, n_sink=4, window=64,
                    top_p=0.8, retrieval=(1, 3), dtype="fp32", idx_dim=d)
    w = dict(kind="decode", seed=40 + d, ctx=(700, 2600), needles=5, shape=sh)
    st = check_decode_parity(make_decode_inputs(w))
    assert st["exact"] >= st["heads"] - 1


@pytest.mark.parametrize("d", [4, 32])
def test_append_indexer_keys_widths(d):
    """d = 4 with an odd capacity: 8-byte bf16 rows take an even row count per
    block, so the second retrieval head's block starts one row later."""
    inp = make_decode_inputs(workload("decode_128k_bf16", ctx=3001, needles=2, shape_idx_dim=d))
    g = run_gpu_decode(inp)
    lay, sh = g["layer"], g["shape"]
    assert g["status"] == 0
    assert lay.kidx_full.shape[2] == (3002 if d == 4 else 3001)
    oc = oracle_cache_from_inputs(inp)
    for r in range(sh.n_retrieval):
        kig = lay.kidx[0, r, :3001].double().cpu().numpy()
        kio = oc.indexer_keys(0, r, 3001)
        assert kig.shape == kio.shape == (3001, d)
        assert np.all(np.abs(kig - kio) <= kidx_bound(inp, 0, r, np.arange(3001)))
        assert np.mean(kig == kio) > 0.999


def test_decode_width4_odd_capacity_ragged():
    """Odd per-sequence lengths at d = 4: score chunks end on half of a 16-byte
    unit, which the copy rounds up inside the padded block."""
    w = workload("ragged_decode_b8_8k_32k_bf16", shape_batch=3, ctx=(1, 5000), needles=4, shape_idx_dim=4)
    inp = make_decode_inputs(w, max_ctx=5001)
    inp["seq_len"] = np.array([1025, 4097, 5001], dtype=np.int32)
    check_decode_parity(inp, top_p=0.9)


def test_decode_width8_static_topk():
    inp = make_decode_inputs(workload("decode_128k_bf16", ctx=4000, needles=8, shape_idx_dim=8,
                                      shape_top_k=100))
    st = check_decode_parity(inp)
    assert np.all(st["counts"] == 100)


@pytest.mark.parametrize("d", [4, 8, 32])
def test_prefill_widths(d):
    """A prefill chunk after a context, ragged rows (odd T and start: 8-byte
    keys of d = 4 end on half of a 16-byte unit)."""
    w = workload("prefill_32k_bf16", needles=12, shape_idx_dim=d, shape_n_sink=8, shape_window=96,
                 shape_top_p=0.9)
    inp = make_prefill_inputs(w, T=414, start_pos=301)  # capacity 715: odd, padded to 716 rows at d = 4
    st = check_prefill_parity(inp)  # every difference within the selection tolerance
    assert st["exact"] >= 0.995 * st["heads"]  # and few of them (3312 row heads)


@pytest.mark.parametrize("d", [4, 32])
def test_prefill_rows_equal_decode_steps_widths(d):
    """Prefill rows and decode steps share the score fragments at every width:
    a row's top-p set equals the decode step's at its position, bit for bit."""
    w = workload("prefill_32k_bf16", needles=16, shape_idx_dim=d, shape_n_sink=16, shape_window=64,
                 shape_top_p=0.9)
    inp = make_prefill_inputs(w, T=333)
    g = run_gpu_prefill(inp)
    sh = inp["shape"]
    bm_p = g["bitmask"].cpu().numpy().view(np.uint32)
    for t in [0, 63, 64, 200, 332]:
        dec = dict(shape=sh, seq_len=np.array([t + 1], dtype=np.int32), max_ctx=inp["max_ctx"],
                   q_pre=inp["q_pre"][:, t].contiguous(), k_pre=inp["k_pre"], v=inp["v"],
                   w_q=inp["w_q"], w_k=inp["w_k"])
        dg = run_gpu_decode(dec)
        bm_d = dg["bitmask"].cpu().numpy().view(np.uint32)
        for rg in range(sh.n_retrieval * sh.group):
            dset = np.nonzero(np.unpackbits(bm_d[0, rg].view(np.uint8), bitorder="little")[: t + 1])[0]
            pset = np.nonzero(np.unpackbits(bm_p[0, rg, t].view(np.uint8), bitorder="little")[: t + 1])[0]
            assert np.array_equal(pset, dset), (d, t, rg, len(pset), len(dset))
