"""CPU checks of the C ABI: the in-tree library loads, exports every entry
point include/rtp.h declares, and rejects bad arguments on the host (no call
here reaches a kernel launch)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "rtp.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rtp_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def rtp():
    import head_wise_sparse_local_b200 as m
    return m


def test_library_exports_every_declared_symbol(rtp):
    lib = ctypes.CDLL(rtp.library_path())
    declared = _declared()
    assert "rtp_decode_attn" in declared and "rtp_append_kv" in declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(rtp.EXPORTS)


def test_version(rtp):
    assert "sm_100a" in rtp.rtp_version()


def _cfg(rtp, **kw):
    base = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, max_ctx=131072, n_sink=64,
                window=2048, top_p=0.95, retrieval=(0, 5), dtype="bf16")
    base.update(kw)
    return rtp.make_cfg(**base)


def test_cache_and_workspace_sizes(rtp):
    k, v, ki = rtp.rtp_cache_bytes(_cfg(rtp))
    assert k == v == 1 * 8 * 131072 * 128 * 2
    assert ki == 1 * 2 * 131072 * 16 * 2
    kf, _, kif = rtp.rtp_cache_bytes(_cfg(rtp, dtype="fp32"))
    assert kf == 2 * k and kif == 2 * ki
    ws = rtp.rtp_decode_workspace_bytes(_cfg(rtp))
    assert ws >= 8 * 131072 * 4  # at least the fp32 score scratch
    assert ws % 256 == 0


@pytest.mark.parametrize("d,dtype,lmax,lk", [(4, "bf16", 1001, 1002), (4, "bf16", 1000, 1000),
                                              (4, "fp32", 1001, 1001), (8, "bf16", 1001, 1001),
                                              (32, "bf16", 777, 777)])
def test_indexer_cache_rows_per_width(rtp, d, dtype, lmax, lk):
    """kidx is [B][R][Lk][d]: Lk = Lmax except 8-byte rows (bf16, d = 4), which
    take an even row count so every (sequence, head) block is 16-byte aligned."""
    es = 2 if dtype == "bf16" else 4
    _, _, ki = rtp.rtp_cache_bytes(_cfg(rtp, idx_dim=d, dtype=dtype, max_ctx=lmax, window=64, n_sink=4))
    assert ki == 1 * 2 * lk * d * es
    assert (lk * d * es) % 16 == 0


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), 2), (dict(n_q_heads=24), 2), (dict(n_q_heads=30), 2),
    (dict(top_p=0.0), 1), (dict(top_p=1.5), 1), (dict(window=0), 1), (dict(n_sink=-1), 1),
    (dict(max_ctx=0), 2), (dict(max_ctx=(1 << 23) + 1), 2), (dict(retrieval=(9,)), 2),
    (dict(idx_dim=12), 2), (dict(rope_base=1.0), 1),
])
def test_invalid_cfg_rejected(rtp, kw, code):
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_decode_workspace_bytes(_cfg(rtp, **kw))
    assert e.value.code == code
    assert rtp.rtp_last_error() != ""


def test_invalid_dtype_rejected(rtp):
    c = _cfg(rtp)
    c.dtype = 7
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_cache_bytes(c)
    assert e.value.code == 3


def test_null_pointers_rejected_before_launch(rtp):
    c = _cfg(rtp)
    cache = rtp.rtp_cache(None, None, None, None)
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_decode_attn(c, cache, 0, 0, 0, 0, 0, workspace=None, stream=0)
    assert e.value.code == 1
    fake = 1 << 20  # never dereferenced: validation fails first
    cache = rtp.rtp_cache(fake, fake, fake, fake)
    with pytest.raises(rtp.RtpError) as e:  # null workspace
        rtp.rtp_decode_attn(c, cache, fake, fake, 0, fake, fake, workspace=None, stream=0)
    assert e.value.code == 4
    with pytest.raises(rtp.RtpError) as e:  # workspace too small
        rtp.rtp_decode_attn(c, cache, fake, fake, 0, fake, fake, workspace=fake,
                            workspace_bytes=100, stream=0)
    assert e.value.code == 4
    with pytest.raises(rtp.RtpError) as e:  # misaligned workspace
        rtp.rtp_decode_attn(c, cache, fake, fake, 0, fake, fake, workspace=fake + 16,
                            workspace_bytes=1 << 40, stream=0)
    assert e.value.code == 4
    with pytest.raises(rtp.RtpError) as e:  # max_seq_len beyond the cache
        rtp.rtp_decode_attn(c, cache, fake, fake, 131073, fake, fake, workspace=fake,
                            workspace_bytes=1 << 40, stream=0)
    assert e.value.code == 2
    with pytest.raises(rtp.RtpError) as e:  # misaligned cache
        bad = rtp.rtp_cache(fake + 2, fake, fake, fake)
        rtp.rtp_append_kv(c, bad, fake, fake, fake, 1, fake, stream=0)
    assert e.value.code == 1
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_append_kv(c, cache, fake, fake, fake, -1, fake, stream=0)
    assert e.value.code == 2
    rtp.rtp_append_kv(c, cache, fake, fake, fake, 0, fake, stream=0)  # T = 0 is a no-op
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_prefill_attn(c, cache, fake, fake, 0, fake, fake, workspace=fake, stream=0)
    assert e.value.code == 2
    with pytest.raises(rtp.RtpError) as e:  # prefill workspace too small
        rtp.rtp_prefill_attn(c, cache, fake, fake, 16, fake, fake, workspace=fake,
                             workspace_bytes=256, stream=0)
    assert e.value.code == 4
    cf = _cfg(rtp, dtype="fp32")
    with pytest.raises(rtp.RtpError) as e:  # prefill computes in bf16 only
        rtp.rtp_prefill_attn(cf, cache, fake, fake, 16, fake, fake, workspace=fake,
                             workspace_bytes=1 << 40, stream=0)
    assert e.value.code == 3
