"""Pins of the CPU oracles (float64 numpy and plain C++) against things other than themselves.

* hand-worked fixtures under tests/golden/ (each cites the page rule it follows);
* brute force with pure-Python loops on tiny integer inputs (exact in float64);
* closed forms and invariants (constant blocks, causality, positive scaling);
* library routines for special cases: torch's scaled_dot_product_attention
  in float64 (dense causal / explicitly masked attention) and full stable
  sorts (numpy lexsort) for the selection.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import cpp as oracle_cpp
from oracle import msa_oracle as oracle_numpy

GOLD = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(params=["numpy", "cpp"])
def O(request):
    """Every pin runs against both oracles: the float64 numpy one and the plain C++ one."""
    return oracle_numpy if request.param == "numpy" else oracle_cpp


def _num(x):
    if isinstance(x, str):
        return float(x)  # "-inf", "-0.0"
    if isinstance(x, list):
        return [_num(v) for v in x]
    return float(x)


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- golden fixtures

def test_golden_scores_handworked(O):
    g = _load("scores_handworked.json")
    k = np.array(g["idx_k"], dtype=np.float64)
    q = np.array(g["idx_q"], dtype=np.float64)
    s1 = O.block_scores(q, k, g["pos"], 1, g["block_size"], g["nb_out"])
    np.testing.assert_array_equal(s1, np.array(_num(g["expected_one_group"])))
    s2 = O.block_scores(q, k, g["pos"], 2, g["block_size"], g["nb_out"])
    np.testing.assert_array_equal(s2, np.array(_num(g["expected_two_groups"])))


def test_golden_topk_handworked(O):
    g = _load("topk_handworked.json")
    for c in g["cases"]:
        s = np.array(_num(c["scores"]), dtype=np.float32)[None, None, :]
        got = O.select_blocks(s, [c["pos"]], c["topk"], g["block_size"])
        assert got[0, 0].tolist() == c["expected"], c


def test_golden_attention_handworked(O):
    g = _load("attention_handworked.json")
    k = np.array(g["k"], dtype=np.float64)
    v = np.array(g["v"], dtype=np.float64)
    q = np.array(g["q"], dtype=np.float64)
    parts = {}
    for c in g["cases"]:
        sel = np.array(c["blocks"])[None, None, :]
        out, lse = O.sparse_attention(q, k, v, g["pos"], sel, g["block_size"], g["scale"])
        np.testing.assert_allclose(out[0], np.array(c["out"]), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0], np.array(c["lse"]), rtol=0, atol=1e-12)
        parts[tuple(c["blocks"])] = (out, lse)
    # two-phase: merging the block-0 and block-1 partials gives the full result
    (o0, l0), (o1, l1) = parts[(0, -1)], parts[(1, -1)]
    om, lm = O.merge_partials([o0, o1], [l0, l1])
    np.testing.assert_allclose(om, parts[(0, 1)][0], atol=1e-12)
    np.testing.assert_allclose(lm, parts[(0, 1)][1], atol=1e-12)


# ---------------------------------------------------------------- brute force

def _brute_scores(q, k, pos, Hkv, blk, nb):
    n, Hi, di = len(q), len(q[0]), len(q[0][0])
    per = Hi // Hkv
    out = [[[-math.inf] * nb for _ in range(Hkv)] for _ in range(n)]
    for r in range(n):
        for b in range(nb):
            tot = [0.0] * Hkv
            seen = False
            for h in range(Hi):
                best = -math.inf
                for j in range(b * blk, min((b + 1) * blk, len(k))):
                    if j > pos[r]:
                        continue
                    dot = 0
                    for c in range(di):
                        dot += q[r][h][c] * k[j][h][c]
                    best = max(best, dot)
                    seen = True
                tot[h // per] += best
            if seen:
                for g in range(Hkv):
                    out[r][g][b] = tot[g]
    return out


@pytest.mark.parametrize("Hi,Hkv", [(4, 2), (4, 1), (2, 2)])
def test_scores_brute_force_tiny(O, Hi, Hkv):
    rng = np.random.default_rng(1)
    L, blk, di, n = 37, 8, 5, 9
    k = rng.integers(-4, 5, size=(L, Hi, di)).astype(np.float64)
    q = rng.integers(-4, 5, size=(n, Hi, di)).astype(np.float64)
    pos = rng.integers(0, L, size=n)
    nb = (L + blk - 1) // blk
    got = O.block_scores(q, k, pos, Hkv, blk, nb)
    want = np.array(_brute_scores(q.tolist(), k.tolist(), pos.tolist(), Hkv, blk, nb))
    np.testing.assert_array_equal(got, want)   # integer data: exact in float64


def test_scores_closed_form_constant_block(O):
    rng = np.random.default_rng(2)
    L, blk, Hi, di = 64, 16, 4, 8
    k = rng.standard_normal((L, Hi, di))
    k[16:32] = k[20]            # block 1: all keys equal
    q = rng.standard_normal((3, Hi, di))
    pos = np.array([40, 63, 31])
    s = O.block_scores(q, k, pos, 2, blk, 4)
    for r in range(3):
        for g in range(2):
            want = sum(float(q[r, h] @ k[20, h]) for h in (2 * g, 2 * g + 1))
            assert abs(s[r, g, 1] - want) < 1e-12


def test_scores_single_dominant_key_and_causality(O):
    rng = np.random.default_rng(3)
    L, blk, Hi, di = 96, 32, 2, 4
    k = rng.standard_normal((L, Hi, di)) * 0.01
    q = np.ones((2, Hi, di))
    k[40, 0] = 10.0             # dominant key of block 1 for head 0
    k[70, :] = 100.0            # a huge key in block 2, after position 65
    pos = np.array([65, 95])
    s = O.block_scores(q, k, pos, 1, blk, 3)
    dots1 = [float(q[0, 1] @ k[j, 1]) for j in range(32, 64)]
    assert abs(s[0, 0, 1] - (40.0 + max(dots1))) < 1e-12
    # row at 65 sees block 2 only up to key 65: the huge key at 70 is not seen
    vis = [max(float(q[0, h] @ k[j, h]) for j in range(64, 66)) for h in range(2)]
    assert abs(s[0, 0, 2] - sum(vis)) < 1e-12
    assert s[1, 0, 2] > 700.0  # row at 95 does see it
    # blocks past the current one are -inf
    s2 = O.block_scores(q, k, np.array([10, 33]), 1, blk, 3)
    assert np.isneginf(s2[0, 0, 1:]).all() and np.isneginf(s2[1, 0, 2])


def test_scores_positive_scaling_keeps_selection(O):
    rng = np.random.default_rng(4)
    L, blk, Hi, di = 512, 16, 4, 8
    k = rng.standard_normal((L, Hi, di))
    q = rng.standard_normal((20, Hi, di))
    pos = rng.integers(0, L, size=20)
    s = O.block_scores(q, k, pos, 2, blk, 32)
    s3 = O.block_scores(q * 4.0, k, pos, 2, blk, 32)   # power of two: exact
    np.testing.assert_array_equal(s3, s * 4.0)
    a = O.select_blocks(s.astype(np.float32), pos, 5, blk)
    b = O.select_blocks(s3.astype(np.float32), pos, 5, blk)
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------- selection

def _lexsort_select(row, cur, topk):
    cand = np.array([b for b in range(min(cur, len(row))) if row[b] != -np.inf], dtype=np.int64)
    if cand.size:
        order = np.lexsort((cand, -row[cand].astype(np.float64)))
        best = cand[order][:topk - 1].tolist()
    else:
        best = []
    sel = sorted(best + [cur])
    return sel + [-1] * (topk - len(sel))


def test_topk_matches_full_stable_sort(O):
    rng = np.random.default_rng(5)
    n, G, nb, blk = 60, 3, 70, 4
    s = rng.standard_normal((n, G, nb)).astype(np.float32)
    s[::7, :, 3:9] = 0.25                      # exact ties
    s[::5, 1, ::4] = -np.inf
    s[3, 0, :] = 1.0                           # a row of all-equal scores
    pos = rng.integers(0, nb * blk, size=n)
    pos[0], pos[1] = 0, nb * blk - 1
    for topk in (1, 2, 5, 16, 80):
        got = O.select_blocks(s, pos, topk, blk)
        for r in range(n):
            for g in range(G):
                want = _lexsort_select(s[r, g], int(pos[r] // blk), topk)
                assert got[r, g].tolist() == want, (topk, r, g)


def test_topk_invariants(O):
    rng = np.random.default_rng(6)
    n, G, nb, blk, topk = 200, 2, 300, 128, 16
    s = rng.standard_normal((n, G, nb)).astype(np.float32)
    pos = rng.integers(0, nb * blk, size=n)
    sel = O.select_blocks(s, pos, topk, blk)
    for r in range(n):
        cur = int(pos[r] // blk)
        for g in range(G):
            row = sel[r, g]
            valid = row[row >= 0]
            assert cur in valid and valid.max() == cur
            assert len(set(valid.tolist())) == len(valid)
            assert (np.diff(valid) > 0).all()
            assert len(valid) == min(topk, cur + 1)
            assert (row[len(valid):] == -1).all()
            # every rejected earlier block scores no higher than the worst kept one
            kept = set(valid.tolist()) - {cur}
            if kept and len(kept) < cur:
                worst = min(s[r, g, b] for b in kept)
                for b in range(cur):
                    if b not in kept:
                        assert s[r, g, b] <= worst


def test_near_tie_report(O):
    blk = 1
    s = np.array([[[5.0, 3.0, 3.0005, 1.0, 0.0]], [[5.0, 3.0, 2.0, 1.0, 0.0]]])
    near, a, b = O.boundary_gap(s, [4, 4], 3, blk)   # 2 free slots
    assert near[0, 0] and not near[1, 0]
    assert a[0, 0] == 3.0005 and b[0, 0] == 3.0
    near, _, _ = O.boundary_gap(s, [4, 4], 5, blk)   # every candidate kept: no boundary
    assert not near.any()


# ---------------------------------------------------------------- attention

def _sdpa(q, k, v, mask, scale):
    """torch float64 scaled_dot_product_attention with GQA expansion."""
    n, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                       # [1][Hq][n][d]
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    m = torch.from_numpy(mask)                                            # [Hq][n][L] bool
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m[None], scale=scale)
    logits = (qt @ kt.transpose(-1, -2)) * scale
    lse = torch.logsumexp(logits.masked_fill(~m[None], -math.inf), dim=-1)
    return out[0].permute(1, 0, 2).numpy(), lse[0].permute(1, 0).numpy()


@pytest.mark.parametrize("L,blk", [(300, 32), (100, 128)])
def test_attention_all_blocks_is_dense_causal(O, L, blk):
    rng = np.random.default_rng(7)
    Hq, Hkv, d = 8, 2, 16
    q = rng.standard_normal((L, Hq, d))
    k = rng.standard_normal((L, Hkv, d))
    v = rng.standard_normal((L, Hkv, d))
    pos = np.arange(L)
    nb = (L + blk - 1) // blk
    sel = np.full((L, Hkv, nb), -1)
    for r in range(L):
        cur = r // blk
        sel[r, :, :cur + 1] = np.arange(cur + 1)
    out, lse = O.sparse_attention(q, k, v, pos, sel, blk)
    causal = np.tril(np.ones((L, L), dtype=bool))[None].repeat(Hq, 0)
    want, wlse = _sdpa(q, k, v, causal, 1.0 / math.sqrt(d))
    np.testing.assert_allclose(out, want, atol=1e-12)
    np.testing.assert_allclose(lse, wlse, atol=1e-12)


def test_attention_subset_is_masked_attention(O):
    rng = np.random.default_rng(8)
    L, blk, Hq, Hkv, d, topk = 256, 16, 6, 3, 8, 4
    q = rng.standard_normal((L, Hq, d))
    k = rng.standard_normal((L, Hkv, d))
    v = rng.standard_normal((L, Hkv, d))
    pos = np.arange(L)
    s = rng.standard_normal((L, Hkv, L // blk)).astype(np.float32)
    sel = O.select_blocks(s, pos, topk, blk)
    mask = np.zeros((Hq, L, L), dtype=bool)
    G = Hq // Hkv
    for r in range(L):
        for h in range(Hq):
            for b in sel[r, h // G]:
                if b >= 0:
                    mask[h, r, b * blk:(b + 1) * blk] = True
            mask[h, r, r + 1:] = False
    out, lse = O.sparse_attention(q, k, v, pos, sel, blk)
    want, wlse = _sdpa(q, k, v, mask, 1.0 / math.sqrt(d))
    np.testing.assert_allclose(out, want, atol=1e-12)
    np.testing.assert_allclose(lse, wlse, atol=1e-12)


def test_attention_value_special_cases(O):
    rng = np.random.default_rng(9)
    L, blk, Hq, Hkv, d = 64, 16, 4, 1, 8
    q = rng.standard_normal((L, Hq, d))
    k = rng.standard_normal((L, Hkv, d))
    pos = np.arange(L)
    sel = np.array([[[0, 1, 2, 3][:(r // blk) + 1] + [-1] * (3 - r // blk)] for r in range(L)])
    ones = np.ones((L, Hkv, d))
    out, _ = O.sparse_attention(q, k, ones, pos, sel, blk)
    np.testing.assert_allclose(out, 1.0, atol=1e-13)
    # one-hot values recover the softmax weight of key j
    j = 5
    onehot = np.zeros((L, Hkv, d))
    onehot[j, 0, 0] = 1.0
    out, lse = O.sparse_attention(q, k, onehot, pos, sel, blk)
    r = 20
    for h in range(Hq):
        logit = float(q[r, h] @ k[j, 0]) / math.sqrt(d)
        assert abs(out[r, h, 0] - math.exp(logit - lse[r, h])) < 1e-12


def test_merge_is_associative(O):
    rng = np.random.default_rng(10)
    L, blk, Hq, Hkv, d = 160, 16, 4, 2, 8
    q = rng.standard_normal((5, Hq, d))
    k = rng.standard_normal((L, Hkv, d))
    v = rng.standard_normal((L, Hkv, d))
    pos = np.array([159, 150, 100, 70, 17])
    full = np.array([[[b if b <= p // blk else -1 for b in range(10)]] * Hkv for p in pos])
    out, lse = O.sparse_attention(q, k, v, pos, full, blk)
    parts = []
    for split in ([0, 3, 7], [1, 2], [4, 5, 6, 8, 9]):
        sel = np.array([[[b if (b in split and b <= p // blk) else -1 for b in range(10)]] * Hkv
                        for p in pos])
        parts.append(sel)
    outs, lses = [], []
    for sel in parts:
        o = np.zeros((5, Hq, d))
        l = np.full((5, Hq), -np.inf)
        for r in range(5):
            if (sel[r] >= 0).any():
                o1, l1 = O.sparse_attention(q[r:r + 1], k, v, pos[r:r + 1], sel[r:r + 1], blk)
                o[r], l[r] = o1[0], l1[0]
        outs.append(o)
        lses.append(l)
    om, lm = O.merge_partials(outs, lses)
    np.testing.assert_allclose(om, out, atol=1e-12)
    np.testing.assert_allclose(lm, lse, atol=1e-12)


# ---------------------------------------------------------------- planted mistakes

def test_fixtures_catch_plausible_slips(O):
    """The hand-worked fixtures are sensitive to the slips a restatement could
    make: off-by-one causality, max instead of sum over a group's heads,
    mean instead of max pooling, and ties going to the higher block id."""
    g = _load("scores_handworked.json")
    k = np.array(g["idx_k"], dtype=np.float64)
    q = np.array(g["idx_q"], dtype=np.float64)
    good = np.array(_num(g["expected_one_group"]))
    assert not np.array_equal(O.block_scores(q, k, np.array(g["pos"]) + 1, 1, 2, 3), good)
    per_head = O.block_scores(q, k, g["pos"], 2, 2, 3)
    assert not np.array_equal(per_head.max(axis=1, keepdims=True), good)
    # mean pooling over the two keys of block 0 for row 0: heads give 1.5 and 1.0, not 2 and 3
    mean_b0 = sum(np.mean([q[0, h] @ k[j, h] for j in (0, 1)]) for h in range(2))
    assert mean_b0 != good[0, 0, 0]
    t = _load("topk_handworked.json")
    case = t["cases"][-1]
    cur = case["pos"] // t["block_size"]
    hi_ties = sorted(sorted(range(cur), key=lambda b: (-case["scores"][b], -b))[:case["topk"] - 1] + [cur])
    assert hi_ties != case["expected"]
