"""Parity of each CUDA kernel against the oracle on small and mid-size inputs
(several tiles, ragged tails, every launch variant)."""
import math

import numpy as np
import pytest
import torch

import block_sparse_long_13_b200 as msa
from oracle import cpp as O   # the plain C++ oracle (pinned, and checked against the numpy one)
from workloads import configs, gen

from . import harness as H

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------- top-k (integer exact)

def _topk_case(nb, topk, seed, nseq=24):
    """Sequences whose queries sit at varied positions, scores with exact ties,
    -inf entries and signed zeros."""
    rng = np.random.default_rng(seed)
    blk = 128
    ctx = [int(x) for x in rng.integers(1, nb * blk + 1, size=nseq)]
    ctx[0], ctx[1], ctx[2] = nb * blk, 1, min(nb * blk, 129)
    nq = [int(x) for x in rng.integers(1, 4, size=nseq)]
    nq = [min(n, c) for n, c in zip(nq, ctx)]
    qs = [0]
    for n in nq:
        qs.append(qs[-1] + n)
    T = qs[-1]
    scores = gen.random_scores(seed, T * 4, nb).view(T, 4, nb).clone()
    scores[::3, :, 5:40] = 0.5                       # exact ties
    scores[1::4, 1, ::7] = float("-inf")
    scores[2::5, 2, 0:6] = torch.tensor([0.0, -0.0, 0.0, -0.0, 1e-30, -1e-30])
    scores[3::6, 3, :] = 2.0                         # whole row tied
    pos = np.concatenate([np.arange(c - n, c) for c, n in zip(ctx, nq)])
    batch = msa.Batch.make(qs, ctx, torch.zeros(nseq, nb, dtype=torch.int32), 1)
    return scores, pos, batch


@pytest.mark.parametrize("nb,topk", [(16, 4), (256, 16), (200, 1), (1024, 16), (1000, 64), (2048, 16),
                                     (4096, 16), (8192, 16), (16384, 64)])
def test_topk_matches_oracle_exactly(cuda_ok, nb, topk):
    scores, pos, batch = _topk_case(nb, topk, seed=nb + topk)
    cfg = msa.Config(topk=topk)
    T = scores.shape[0]
    sel = torch.full((T, 4, topk), -9, dtype=torch.int32, device="cuda")
    msa.topk_blocks(cfg, batch, scores.cuda(), sel)
    assert msa.device_status() == msa.MSA_OK
    want = O.select_blocks(scores.numpy(), pos, topk, 128)
    got = sel.cpu().numpy()
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]


# ----------------------------------------------------------------- indexer scores

def _mixed_workload(seed, nq_big=True, nq=None):
    """Several sequences, random page table, ragged tails; queries at the end
    of each context (chunked-prefill positions)."""
    ctx = [1000, 3000, 129, 5000, 256]
    if nq is None:
        nq = [1000, 300, 129, 200, 1] if nq_big else [1, 4, 1, 3, 1]
    return gen.make_workload("mixed", seed=seed, ctx_len=ctx, nq=nq, num_q_heads=64, num_kv_heads=4,
                             idx_heads=8, topk=16, plant_frac=0.1, random_pages=True)


@pytest.mark.parametrize("which", ["tiny", "mixed_prefill", "mixed_decode", "tiny_decode", "decode_nq1",
                                   "decode_nq2"])
def test_index_scores_match_oracle(cuda_ok, which):
    if which == "tiny":
        wl = configs.tiny_prefill_2k()
    elif which in ("decode_nq1", "decode_nq2"):
        wl = _mixed_workload(13, nq=[1] * 5 if which == "decode_nq1" else [2, 1, 2, 2, 1])
    elif which == "tiny_decode":
        wl = gen.make_workload("tinyd", seed=5, ctx_len=[2048, 700, 4000], nq=[1, 2, 8], num_q_heads=16,
                               num_kv_heads=1, idx_heads=4, topk=4, plant_count=2, random_pages=True)
    else:
        wl = _mixed_workload(3, nq_big=(which == "mixed_prefill"))
    d = H.device_inputs(wl)
    got = H.run_index(d).cpu().numpy()
    assert msa.device_status() == msa.MSA_OK
    pos = wl.positions().numpy()
    worst = -np.inf
    for s in range(wl.num_seqs):
        rows = list(H.seq_rows(wl, s))
        if len(rows) > 400:
            rows = rows[:64] + rows[len(rows) // 2 - 32:len(rows) // 2 + 32] + rows[-64:]
        ref = H.oracle_scores_rows(d, s, rows)
        worst = max(worst, H.compare_scores(got[rows], ref, pos[rows], wl.block_size))
    assert worst <= 0, worst


# ----------------------------------------------------------------- attention

def _oracle_selection(wl, seed):
    """A valid selection drawn from random scores by the oracle's rule."""
    T = wl.total_q
    s = gen.random_scores(seed, T * wl.num_kv_heads, wl.max_blocks).view(T, wl.num_kv_heads, wl.max_blocks)
    return O.select_blocks(s.numpy(), wl.positions().numpy(), wl.topk, wl.block_size)


@pytest.mark.parametrize("which,path", [("tiny", "prefill"), ("tiny", "decode"), ("mixed_prefill", "prefill"),
                                        ("mixed_decode", "decode"), ("mixed_decode", "prefill")])
def test_attention_matches_oracle(cuda_ok, which, path):
    wl = configs.tiny_prefill_2k() if which == "tiny" else _mixed_workload(4, nq_big=(which == "mixed_prefill"))
    d = H.device_inputs(wl)
    sel = _oracle_selection(wl, 11)
    out, lse = H.run_attn(d, torch.from_numpy(sel).cuda(), path)
    assert msa.device_status() == msa.MSA_OK
    errs, lerr = [], []
    for s in range(wl.num_seqs):
        rows = list(H.seq_rows(wl, s))
        if len(rows) > 300:
            rows = rows[:48] + rows[-48:]
        ref, ref_lse = H.oracle_attention_rows(d, s, rows, sel[rows])
        errs.append(H.attn_errors(out[rows], ref))
        lerr.append(float(np.abs(lse[rows].cpu().numpy() - ref_lse).max()))
    mx = max(e[0] for e in errs)
    mean = float(np.mean([e[1] for e in errs]))
    assert mx <= H.ATTN_MAX_ABS and mean <= H.ATTN_MEAN_ABS, (mx, mean)
    assert max(lerr) <= H.LSE_MAX_ABS, max(lerr)


def test_wide_selection_rows_match_oracle(cuda_ok):
    """k = 32 over 4 groups: 128 entries per query row, more than the prefill schedule's per-CTA
    bucket table holds, so its per-entry counting path builds the tiles."""
    wl = gen.make_workload("mixed_k32", seed=8, ctx_len=[1000, 3000, 129, 5000, 256], nq=[1000, 300, 129, 200, 1],
                           num_q_heads=64, num_kv_heads=4, idx_heads=8, topk=32, plant_frac=0.1, random_pages=True)
    d = H.device_inputs(wl)
    sel = _oracle_selection(wl, 13)
    out, lse = H.run_attn(d, torch.from_numpy(sel).cuda(), "prefill")
    assert msa.device_status() == msa.MSA_OK
    errs, lerr = [], []
    for s in range(wl.num_seqs):
        rows = list(H.seq_rows(wl, s))
        if len(rows) > 300:
            rows = rows[:48] + rows[-48:]
        ref, ref_lse = H.oracle_attention_rows(d, s, rows, sel[rows])
        errs.append(H.attn_errors(out[rows], ref))
        lerr.append(float(np.abs(lse[rows].cpu().numpy() - ref_lse).max()))
    mx = max(e[0] for e in errs)
    mean = float(np.mean([e[1] for e in errs]))
    assert mx <= H.ATTN_MAX_ABS and mean <= H.ATTN_MEAN_ABS, (mx, mean)
    assert max(lerr) <= H.LSE_MAX_ABS, max(lerr)


def test_all_blocks_selected_is_dense_causal(cuda_ok):
    """k >= number of blocks: every row attends to its whole causal prefix."""
    wl = configs.tiny_prefill_2k()
    wl.topk = 16
    d = H.device_inputs(wl)
    T = wl.total_q
    pos = wl.positions().numpy()
    sel = np.full((T, 1, 16), -1, dtype=np.int32)
    for t in range(T):
        cur = pos[t] // 128
        sel[t, 0, :cur + 1] = np.arange(cur + 1)
    out, lse = H.run_attn(d, torch.from_numpy(sel).cuda(), "prefill")
    rows = list(range(0, T, 97)) + [T - 1]
    ref, ref_lse = H.oracle_attention_rows(d, 0, rows, sel[rows])
    mx, mean = H.attn_errors(out[rows], ref)
    assert mx <= H.ATTN_MAX_ABS and mean <= H.ATTN_MEAN_ABS


def test_prefill_and_decode_paths_agree(cuda_ok):
    wl = _mixed_workload(6, nq_big=False)
    d = H.device_inputs(wl)
    sel = torch.from_numpy(_oracle_selection(wl, 12)).cuda()
    o1, l1 = H.run_attn(d, sel, "prefill")
    o2, l2 = H.run_attn(d, sel, "decode")
    assert float((o1.float() - o2.float()).abs().max()) <= 1.6e-2
    assert float((l1 - l2).abs().max()) <= 1e-3
