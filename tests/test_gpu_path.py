"""The whole hot path (indexer -> top-k -> attention) against the oracle:
every row of the 2K-token workload, sampled rows of the full-size workloads
in the launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import block_sparse_long_13_b200 as msa
from workloads import configs, gen

from . import harness as H

pytestmark = pytest.mark.gpu


def _check_chain(d, rows_by_seq, path, report):
    """Run the chain on the device, then for the sampled rows: scores within
    tolerance, selections exact outside near-ties, and attention (fed the
    oracle's selection for those rows) within the stated tolerances."""
    wl = d.wl
    scores = H.run_index(d)
    sel = H.run_topk(d, scores)
    assert msa.device_status() == msa.MSA_OK
    got_s = scores.cpu().numpy()
    got_sel = sel.cpu().numpy()
    pos = wl.positions().numpy()
    ref_sel_rows = {}
    tot_near = tot_mism = tot_bad = 0
    worst = -np.inf
    for s, rows in rows_by_seq.items():
        ref64 = H.oracle_scores_rows(d, s, rows)
        worst = max(worst, H.compare_scores(got_s[rows], ref64, pos[rows], wl.block_size))
        from oracle import cpp as O
        ref_sel = O.select_blocks(ref64.astype(np.float32), pos[rows], wl.topk, wl.block_size)
        n, m, b = H.compare_selection(got_sel[rows], ref_sel, ref64, pos[rows], wl.topk, wl.block_size)
        tot_near, tot_mism, tot_bad = tot_near + n, tot_mism + m, tot_bad + b
        ref_sel_rows[s] = ref_sel
    report.update(near_ties=tot_near, mismatches=tot_mism, score_excess=worst)
    assert worst <= 0, worst
    assert tot_bad == 0, (tot_near, tot_mism, tot_bad)
    # attention on the oracle's selection for the sampled rows
    for s, rows in rows_by_seq.items():
        sel[rows] = torch.from_numpy(ref_sel_rows[s]).cuda()
    out, lse = H.run_attn(d, sel, path)
    assert msa.device_status() == msa.MSA_OK
    mx = mean = 0.0
    n = 0
    for s, rows in rows_by_seq.items():
        ref, ref_lse = H.oracle_attention_rows(d, s, rows, ref_sel_rows[s])
        a, b = H.attn_errors(out[rows], ref)
        mx = max(mx, a)
        mean += b * len(rows)
        n += len(rows)
        assert float(np.abs(lse[rows].cpu().numpy() - ref_lse).max()) <= H.LSE_MAX_ABS
    mean /= n
    report.update(attn_max_abs=mx, attn_mean_abs=mean)
    assert mx <= H.ATTN_MAX_ABS and mean <= H.ATTN_MEAN_ABS, (mx, mean)


def test_tiny_prefill_every_row(cuda_ok):
    wl = configs.tiny_prefill_2k()
    d = H.device_inputs(wl)
    rep = {}
    _check_chain(d, {0: list(range(wl.total_q))}, "prefill", rep)
    print("tiny_prefill_2k", rep)


def _sample(rng, lo, hi, n, extra=()):
    pick = set(int(x) for x in rng.integers(lo, hi, size=n))
    pick.update(x for x in extra if lo <= x < hi)
    return sorted(pick)


@pytest.mark.slow
def test_prefill_32k_sampled(cuda_ok):
    wl = configs.prefill_32k()
    d = H.device_inputs(wl)
    rng = np.random.default_rng(0)
    T = wl.total_q
    rows = _sample(rng, 0, T, 40, extra=[0, 1, 127, 128, 4095, T - 129, T - 1])
    rep = {}
    _check_chain(d, {0: rows}, "prefill", rep)
    print("prefill_32k", rep)


@pytest.mark.slow
def test_chunked_prefill_128k_sampled(cuda_ok):
    chunks = configs.chunked_prefill_128k()
    caches = {}
    rng = np.random.default_rng(1)
    for c in (0, 3, 7):
        wl = chunks[c]
        d = H.device_inputs(wl, caches=caches)
        rows = _sample(rng, 0, wl.total_q, 12, extra=[0, wl.total_q - 1])
        rep = {}
        _check_chain(d, {0: rows}, "prefill", rep)
        print(f"chunk {c}", rep)
        del d
    caches.clear()
    torch.cuda.empty_cache()


@pytest.mark.slow
@pytest.mark.parametrize("name", ["decode_128k", "decode_1m", "verify_ragged"])
def test_decode_sampled(cuda_ok, name):
    wl = configs.ALL[name]()
    d = H.device_inputs(wl)
    rng = np.random.default_rng(2)
    nseq = 2 if name == "decode_1m" else 4
    seqs = sorted(set(int(x) for x in rng.integers(0, wl.num_seqs, size=nseq)) | {wl.num_seqs - 1})
    rep = {}
    _check_chain(d, {s: list(H.seq_rows(wl, s)) for s in seqs}, "decode", rep)
    print(name, rep)
    del d
    torch.cuda.empty_cache()
