"""Pins of the FP8 (e4m3) cache oracle against things other than itself:
torch's float8_e4m3fn cast inside the finite range, every representable code
round-tripping exactly, saturation and the relative-error bound of 3 mantissa
bits, and brute force on indexer scores computed from dequantized keys."""
import math

import numpy as np
import torch

from oracle import fp8_cache as F
from oracle import msa_oracle as O


def _all_finite_codes():
    raw = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    v = raw[torch.isfinite(raw)].numpy()
    return np.unique(v)


def test_matches_torch_cast_inside_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000) * 3,
        rng.uniform(-448, 448, 20000),
        rng.uniform(-2 ** -6, 2 ** -6, 20000),                  # subnormal range
        (np.arange(-2000, 2000) + 0.5) * 2 ** -9,              # ties in the subnormal range
        np.array([1.0625, 1.1875, 3.0625, 240.0 + 8.0, 460.0, -460.0, 0.0, -0.0]),
    ])
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = F.round_e4m3(x)
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]


def test_every_code_roundtrips_exactly():
    codes = _all_finite_codes()
    assert len(codes) == 253          # 254 finite encodings, +0 and -0 equal
    assert np.array_equal(F.round_e4m3(codes), codes)
    for scale in (1.0, 0.0125, 3.0):
        np.testing.assert_array_equal(F.roundtrip(codes * scale, scale), codes * scale)


def test_saturation_and_relative_error():
    assert F.round_e4m3(np.array([1e6, -1e6, 449.0, 464.1]))[:2].tolist() == [448.0, -448.0]
    assert np.all(np.abs(F.round_e4m3(np.array([449.0, 464.1, 1e30]))) == 448.0)
    rng = np.random.default_rng(2)
    y = rng.uniform(2 ** -6, 448, 50000) * rng.choice([-1, 1], 50000)
    q = F.round_e4m3(y)
    assert np.max(np.abs(q - y) / np.abs(y)) <= 2.0 ** -4 + 1e-15
    # subnormal range: absolute error at most half the 2^-9 spacing
    z = rng.uniform(-2 ** -6, 2 ** -6, 50000)
    assert np.max(np.abs(F.round_e4m3(z) - z)) <= 2.0 ** -10 + 1e-18


def test_scores_from_dequantized_keys_brute_force():
    """Indexer block scores from FP8 keys equal pure-Python sums over the dequantized values."""
    rng = np.random.default_rng(3)
    T, H, n, bs = 3, 2, 8, 4
    q = rng.standard_normal((T, H, 4))
    k = rng.standard_normal((n, H, 4))
    scale = float(np.abs(k).max()) / 448.0
    kd = F.roundtrip(k, scale)
    pos = np.array([7, 5, 2])
    got = O.block_scores(q, kd, pos, num_kv_heads=1, block_size=bs, nb_out=2)
    for t in range(T):
        for b in range(2):
            js = [j for j in range(b * bs, min(n, (b + 1) * bs)) if j <= pos[t]]
            want = -math.inf if not js else sum(max(sum(q[t, h, c] * kd[j, h, c] for c in range(4)) for j in js)
                                                for h in range(H))
            assert (got[t, 0, b] == want) if want == -math.inf else abs(got[t, 0, b] - want) <= 1e-12


def test_pins_catch_plausible_slips():
    """Rounding ties away from zero, truncating, or letting values past 448 through would each
    break a pin above."""
    x = np.array([1.0625, 1.1875, 3.0625, 2 ** -10, 3 * 2 ** -10, 460.0, 1e6])
    want = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).to(torch.float64).numpy()

    def rounded(y, mode):
        a = np.abs(y)
        _, e = np.frexp(a)
        e = np.maximum(e - 1, -6)
        qn = np.ldexp(1.0, e - 3)
        m = a / qn
        r = {"away": np.floor(m + 0.5), "trunc": np.floor(m)}[mode]
        return np.copysign(r * qn, y)

    assert np.array_equal(F.round_e4m3(x), want)
    assert not np.array_equal(rounded(np.clip(x, -448, 448), "away"), want)
    assert not np.array_equal(rounded(np.clip(x, -448, 448), "trunc"), want)
    assert F.round_e4m3(np.array([1e6]))[0] == 448.0 != rounded(np.array([1e6]), "away")[0]


def test_decode_bits_matches_torch_for_every_pattern():
    bits = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(bits).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = F.decode_bits(bits)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    fin = ~np.isnan(want)
    assert np.array_equal(got[fin], want[fin])
    assert np.array_equal(np.signbit(got[fin]), np.signbit(want[fin]))   # -0 stays -0
    # a planted slip (bias 8 instead of 7) fails
    slip = np.where(((bits >> 3) & 0xF) == 0, got, got / 2)
    assert not np.array_equal(slip[fin], want[fin])
