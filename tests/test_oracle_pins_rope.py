"""Pins of the QK-norm / partial-RoPE / paged-insert oracle against things
other than itself: hand-worked fixtures (tests/golden/), closed forms of the
norm, the rotation restated as a complex exponential, the relative-position
invariant of rotary embeddings, and brute force on the cache writes."""
import json
import math
import os

import numpy as np

from oracle import qk_rope_insert as R

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_handworked():
    with open(os.path.join(GOLD, "qknorm_rope_handworked.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        x = np.array(c["x"], dtype=np.float64).reshape(1, 1, -1)
        y = R.rope_partial(R.rms_norm_heads(x, c["w"], c["eps"]), [c["pos"]], c["rotary_dim"], c["theta"])
        np.testing.assert_allclose(y.reshape(-1), c["expected"], rtol=0, atol=1e-12, err_msg=c["note"])


def test_rms_norm_closed_form_constant_head():
    """x = c * ones: x / sqrt(c^2 + eps) * w, whatever the head size."""
    rng = np.random.default_rng(1)
    for c in (-3.5, -1e-3, 0.25, 7.0):
        for d in (4, 64, 128):
            w = rng.standard_normal(d)
            eps = 1e-6
            got = R.rms_norm_heads(np.full((2, 3, d), c), w, eps)
            want = c / math.sqrt(c * c + eps) * w
            np.testing.assert_allclose(got, np.broadcast_to(want, got.shape), rtol=1e-14, atol=0)


def test_rms_norm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 4, 128))
    y = R.rms_norm_heads(x, np.ones(128), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(R.rms_norm_heads(37.0 * x, np.ones(128), 0.0), y, rtol=1e-13, atol=1e-15)


def test_rope_is_a_complex_rotation():
    """Pairs (i, i + r/2) as complex numbers a + ib, multiplied by exp(i p theta^(-2i/r))."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 3, 128))
    pos = np.array([0, 1, 17, 4095, 131071, 1048575])
    theta, r = 10000.0, 64
    got = R.rope_partial(x, pos, r, theta)
    half = r // 2
    z = x[..., :half] + 1j * x[..., half:r]
    freq = np.array([theta ** (-2.0 * i / r) for i in range(half)])
    rot = np.exp(1j * pos[:, None, None] * freq[None, None, :])
    zr = z * rot
    np.testing.assert_allclose(got[..., :half], zr.real, rtol=0, atol=1e-9)
    np.testing.assert_allclose(got[..., half:r], zr.imag, rtol=0, atol=1e-9)
    assert np.array_equal(got[..., r:], x[..., r:])          # pass-through channels untouched


def test_rope_identity_at_zero_and_norm_preserving():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 2, 128))
    np.testing.assert_array_equal(R.rope_partial(x, [0, 0, 0]), x)
    y = R.rope_partial(x, [5, 900, 70000])
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def test_rope_relative_position_invariant():
    """<rope(q, m), rope(k, n)> depends on m - n only."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))
    def dot(m, n):
        return float(np.sum(R.rope_partial(q, [m]) * R.rope_partial(k, [n])))
    for m, n in ((10, 3), (1000, 999), (5, 70)):
        for s in (1, 64, 12345):
            assert abs(dot(m, n) - dot(m + s, n + s)) <= 1e-9 * (1 + abs(dot(m, n)))


def test_insert_writes_exactly_the_rows_of_the_call():
    """Brute force: the cache equals the old cache except at (page, slot) of each new row."""
    rng = np.random.default_rng(6)
    bs, hkv, hq, d, pages = 4, 2, 4, 8, 7
    page_table = np.array([[3, 0, 5], [6, 1, 2]])
    # sequence 0 writes positions 5, 6 (page 0 slots 1, 2); sequence 1 writes position 8 (page 2 slot 0)
    pos = np.array([5, 6, 8])
    seq = np.array([0, 0, 1])
    q = rng.standard_normal((3, hq, d))
    k = rng.standard_normal((3, hkv, d))
    v = rng.standard_normal((3, hkv, d))
    wq, wk = rng.standard_normal(d), rng.standard_normal(d)
    kc = rng.standard_normal((pages, hkv, bs, d))
    vc = rng.standard_normal((pages, hkv, bs, d))
    q_out, kc2, vc2 = R.qknorm_rope_insert(q, k, v, wq, wk, pos, seq, page_table, kc, vc, block_size=bs,
                                           rotary_dim=4, theta=10000.0, eps=1e-6)
    kexp, vexp = kc.copy(), vc.copy()
    for t, (p, s) in enumerate(zip(pos, seq)):
        page, slot = page_table[s][p // bs], p % bs
        for h in range(hkv):
            row = k[t, h] / math.sqrt(float(np.mean(k[t, h] ** 2)) + 1e-6) * wk
            a0, b0 = row[0], row[2]
            a1, b1 = row[1], row[3]
            f0, f1 = 1.0, 10000.0 ** (-0.5)
            row = row.copy()
            row[0], row[2] = a0 * math.cos(p * f0) - b0 * math.sin(p * f0), b0 * math.cos(p * f0) + a0 * math.sin(p * f0)
            row[1], row[3] = a1 * math.cos(p * f1) - b1 * math.sin(p * f1), b1 * math.cos(p * f1) + a1 * math.sin(p * f1)
            kexp[page, h, slot] = row
            vexp[page, h, slot] = v[t, h]
    np.testing.assert_allclose(kc2, kexp, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(vc2, vexp)
    assert q_out.shape == q.shape


def test_fixtures_catch_plausible_slips():
    """The hand-worked cases fail for the slips a restatement could make: interleaved pairs
    (i, i+1) instead of (i, i + r/2), the rotation turned the other way, eps outside the root,
    and the frequency exponent -i/r instead of -2i/r."""
    with open(os.path.join(GOLD, "qknorm_rope_handworked.json")) as f:
        g = json.load(f)

    def norm(x, w, eps, outside=False):
        ms = np.mean(x * x)
        return (x / (np.sqrt(ms) + eps) if outside else x / np.sqrt(ms + eps)) * np.asarray(w, dtype=np.float64)

    def rope(x, p, r, theta, pairing="half", sign=1.0, expo=2.0):
        y = x.copy()
        for i in range(r // 2):
            a_i, b_i = (i, i + r // 2) if pairing == "half" else (2 * i, 2 * i + 1)
            ang = sign * p * theta ** (-expo * i / r)
            a, b = x[a_i], x[b_i]
            y[a_i], y[b_i] = a * math.cos(ang) - b * math.sin(ang), b * math.cos(ang) + a * math.sin(ang)
        return y

    def run(c, **kw):
        outside = kw.pop("outside", False)
        x = np.array(c["x"], dtype=np.float64)
        return rope(norm(x, c["w"], c["eps"], outside), c["pos"], c["rotary_dim"], c["theta"], **kw)

    def matches_all(**kw):
        return all(np.allclose(run(c, **dict(kw)), c["expected"], atol=1e-9) for c in g["cases"])

    assert matches_all()                                  # the restatement itself reproduces every case
    assert not matches_all(pairing="interleaved")
    assert not matches_all(sign=-1.0)
    assert not matches_all(outside=True)
    assert not matches_all(expo=1.0)
