"""The plain C++ oracle (oracle/msa_oracle.cpp) against the float64 numpy
oracle on random inputs: two independent restatements of the same
definitions must agree to rounding (1e-12), and the C++ results must not
depend on how many threads split the work.  Both oracles are also pinned, one
by one, by tests/test_oracle_pins.py."""
import numpy as np
import pytest

from oracle import cpp as C
from oracle import msa_oracle as N


def _inputs(seed, L=700, Hi=8, Hkv=4, Hq=64, d=128, di=64, n=40, f32=True):
    rng = np.random.default_rng(seed)
    dt = np.float32 if f32 else np.float64
    k = rng.standard_normal((L, Hkv, d)).astype(dt)
    v = rng.standard_normal((L, Hkv, d)).astype(dt)
    ik = rng.standard_normal((L, Hi, di)).astype(dt)
    q = rng.standard_normal((n, Hq, d)).astype(dt)
    iq = rng.standard_normal((n, Hi, di)).astype(dt)
    pos = np.sort(rng.integers(0, L, size=n))
    pos[-1] = L - 1
    return q, iq, k, v, ik, pos


@pytest.mark.parametrize("f32,bs,topk", [(True, 128, 4), (False, 32, 5), (True, 16, 16)])
def test_cpp_matches_numpy(f32, bs, topk):
    q, iq, k, v, ik, pos = _inputs(3, f32=f32)
    nb = (len(k) + bs - 1) // bs
    s_c = C.block_scores(iq, ik, pos, 4, bs, nb)
    s_n = N.block_scores(iq, ik, pos, 4, bs, nb)
    fin = np.isfinite(s_n)
    assert np.array_equal(np.isfinite(s_c), fin)
    assert np.abs(s_c[fin] - s_n[fin]).max() <= 1e-12 * max(1.0, np.abs(s_n[fin]).max())
    sel_c = C.select_blocks(s_c.astype(np.float32), pos, topk, bs)
    sel_n = N.select_blocks(s_n.astype(np.float32), pos, topk, bs)
    assert np.array_equal(sel_c, sel_n)
    for a, b in zip(C.boundary_gap(s_c, pos, topk, bs), N.boundary_gap(s_n, pos, topk, bs)):
        assert np.allclose(a, b, rtol=0, atol=1e-12, equal_nan=True)
    o_c, l_c = C.sparse_attention(q, k, v, pos, sel_n, bs)
    o_n, l_n = N.sparse_attention(q, k, v, pos, sel_n, bs)
    assert np.abs(o_c - o_n).max() <= 1e-12 and np.abs(l_c - l_n).max() <= 1e-12
    parts = [o_c[:20], o_c[20:]], [l_c[:20], l_c[20:]]
    m_c = C.merge_partials(*parts)
    m_n = N.merge_partials(*parts)
    assert np.abs(m_c[0] - m_n[0]).max() <= 1e-12 and np.abs(m_c[1] - m_n[1]).max() <= 1e-12


def test_cpp_results_do_not_depend_on_threads():
    q, iq, k, v, ik, pos = _inputs(4)
    old = C.threads()
    try:
        outs = []
        for t in (1, 3, 16):
            C.set_threads(t)
            s = C.block_scores(iq, ik, pos, 4, 128, 6)
            sel = C.select_blocks(s.astype(np.float32), pos, 4, 128)
            outs.append((s, sel) + C.sparse_attention(q, k, v, pos, sel, 128))
        for other in outs[1:]:
            for a, b in zip(outs[0], other):
                assert np.array_equal(a, b)
    finally:
        C.set_threads(old)


def test_cpp_empty_selection_and_merge_conventions():
    """A (row, group) with no visible key: out 0, lse -inf; a merge unit whose partials are all
    -inf: out 0, L -inf (conventions the kernels share)."""
    q, iq, k, v, ik, pos = _inputs(5, n=3)
    sel = np.full((3, 4, 4), -1, dtype=np.int32)
    sel[0, 1, 0] = 0
    out, lse = C.sparse_attention(q, k, v, pos, sel, 128)
    assert np.isfinite(lse[0, 16:32]).all() and np.isneginf(np.delete(lse, np.s_[16:32], axis=1)[0]).all()
    assert (out[1:] == 0).all() and np.isneginf(lse[1:]).all()
    o, l = C.merge_partials(np.zeros((2, 3, 8)), np.full((2, 3), -np.inf))
    assert (o == 0).all() and np.isneginf(l).all()
