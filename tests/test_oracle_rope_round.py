"""Pins of the oracle's RoPE and storage rounding: closed forms for small D,
RoPE's relative-position identity, and bf16 rounding against torch's own
fp32 -> bf16 conversion (a library routine) plus hand-derived ties."""

import math

import numpy as np
import pytest
import torch

from oracle import rope, rope_inv_freq, round_bf16, round_storage


def test_rope_d2_closed_form():
    # D = 2: one pair, inv_freq = 1, angle = pos.
    for pos in [0, 1, 2.5, 1000]:
        y = rope(np.array([1.0, 0.0]), pos, 10000.0)
        assert np.allclose(y, [math.cos(pos), math.sin(pos)], atol=1e-15)
        y = rope(np.array([0.0, 1.0]), pos, 10000.0)
        assert np.allclose(y, [-math.sin(pos), math.cos(pos)], atol=1e-15)


def test_rope_d4_closed_form():
    # D = 4, base 10000: inv_freq = [1, 10000^(-1/2)] = [1, 0.01]; pairs (x0, x2), (x1, x3).
    assert np.allclose(rope_inv_freq(4, 10000.0), [1.0, 0.01], rtol=1e-15)
    a, b, c, d = 0.3, -1.2, 0.7, 2.0
    pos = 7
    t0, t1 = pos * 1.0, pos * 0.01
    y = rope(np.array([a, b, c, d]), pos, 10000.0)
    want = [a * math.cos(t0) - c * math.sin(t0), b * math.cos(t1) - d * math.sin(t1),
            c * math.cos(t0) + a * math.sin(t0), d * math.cos(t1) + b * math.sin(t1)]
    assert np.allclose(y, want, atol=1e-14)


def test_rope_inv_freq_d128():
    f = rope_inv_freq(128, 10000.0)
    assert f[0] == 1.0 and abs(f[32] - 0.01) < 1e-17 and abs(f[63] - 10000.0 ** (-126 / 128)) < 1e-20


@pytest.mark.parametrize("seed", range(4))
def test_rope_relative_position_identity(seed):
    rng = np.random.default_rng(seed)
    q, k = rng.normal(size=128), rng.normal(size=128)
    i, j = int(rng.integers(0, 1 << 20)), int(rng.integers(0, 1 << 20))
    base = np.dot(rope(q, i, 1e4), rope(k, j, 1e4))
    for shift in [1, 17, 4096, 123457]:
        assert abs(np.dot(rope(q, i + shift, 1e4), rope(k, j + shift, 1e4)) - base) < 1e-9
    assert abs(np.linalg.norm(rope(q, i, 1e4)) - np.linalg.norm(q)) < 1e-12
    assert np.array_equal(rope(q, 0, 1e4), q)


def test_round_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    x = rng.normal(0, 3, size=200_000).astype(np.float32)
    # exact halfway cases between neighbouring bf16 values
    base = rng.normal(0, 3, size=5000).astype(np.float32)
    half = (base.view(np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    x = np.concatenate([x, half.view(np.float32), np.array([0.0, -0.0, 1e-30, 3e38], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    got = round_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_round_bf16_ties_to_even_by_hand():
    assert round_bf16(1.0 + 2.0 ** -8) == 1.0                     # halfway, even below
    assert round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6      # halfway, even above
    assert round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7
    assert round_bf16(-(1.0 + 2.0 ** -8)) == -1.0
    # fp64 value between two fp32 values: direct rounding, no double rounding
    x = 1.0 + 2.0 ** -8 + 2.0 ** -35
    assert round_bf16(x) == 1.0 + 2.0 ** -7


def test_round_storage_fp32():
    x = np.array([1.0 + 2.0 ** -30, math.pi])
    assert np.array_equal(round_storage(x, "fp32"), x.astype(np.float32).astype(np.float64))
