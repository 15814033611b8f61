"""msa_index_topk (indexer and top-k in one pass) through the C ABI.

The fused call must give exactly the selection of msa_index_scores followed
by msa_topk_blocks (same fp32 scores, same rule), integer for integer, and
agree with the oracle's selection outside reported near-ties."""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_long_13_b200 as msa
from oracle import cpp as O   # the plain C++ oracle (pinned, and checked against the numpy one)
from workloads import configs, gen

from . import harness as H

pytestmark = pytest.mark.gpu


def _fused(d, topk=None):
    k = d.wl.topk if topk is None else topk
    sel = torch.full((d.wl.total_q, d.wl.num_kv_heads, k), -7, dtype=torch.int32, device="cuda")
    cfg = d.cfg if topk is None else dataclasses.replace(d.cfg, topk=topk)
    msa.index_topk(cfg, d.batch, d.idx_q, d.idx_k_cache, sel)
    assert msa.device_status() == msa.MSA_OK
    return sel


def _two_calls(d, topk=None):
    scores = H.run_index(d)
    cfg = d.cfg if topk is None else dataclasses.replace(d.cfg, topk=topk)
    k = d.wl.topk if topk is None else topk
    sel = torch.full((d.wl.total_q, d.wl.num_kv_heads, k), -7, dtype=torch.int32, device="cuda")
    msa.topk_blocks(cfg, d.batch, scores, sel)
    assert msa.device_status() == msa.MSA_OK
    return sel


def _mixed(seed, random_pages=True):
    return gen.make_workload("mixed_fused", seed=seed, ctx_len=[1000, 3000, 129, 5000, 256, 9000],
                             nq=[1000, 300, 129, 200, 1, 700], num_q_heads=64, num_kv_heads=4, idx_heads=8,
                             topk=16, plant_frac=0.1, random_pages=random_pages)


@pytest.mark.parametrize("which", ["tiny", "mixed", "mixed_identity_pages"])
def test_fused_equals_two_calls(cuda_ok, which):
    wl = configs.tiny_prefill_2k() if which == "tiny" else _mixed(21, random_pages=(which == "mixed"))
    d = H.device_inputs(wl)
    a = _fused(d).cpu().numpy()
    b = _two_calls(d).cpu().numpy()
    assert np.array_equal(a, b), np.argwhere(a != b)[:5]


@pytest.mark.parametrize("topk", [1, 2, 5, 16])
def test_fused_every_topk(cuda_ok, topk):
    d = H.device_inputs(_mixed(22))
    a = _fused(d, topk).cpu().numpy()
    b = _two_calls(d, topk).cpu().numpy()
    assert np.array_equal(a, b), np.argwhere(a != b)[:5]


def test_fused_ties_go_to_the_lower_block(cuda_ok):
    """Blocks that map to one physical page have equal scores for every row:
    the selection must keep the lower block ids first, as the two-call path does."""
    wl = _mixed(23)
    pt = wl.page_table.clone()
    # sequence 5 (9000 tokens, 71 blocks): blocks 10..39 all read page of block 10
    pt[5, 10:40] = pt[5, 10]
    wl.page_table = pt
    d = H.device_inputs(wl)
    a = _fused(d).cpu().numpy()
    b = _two_calls(d).cpu().numpy()
    assert np.array_equal(a, b), np.argwhere(a != b)[:5]
    rows = list(H.seq_rows(wl, 5))
    # at least one row keeps several of the tied blocks, and keeps the lowest ones
    kept = [sorted(x for x in a[r, g] if 10 <= x < 40) for r in rows[-50:] for g in range(4)]
    assert any(len(k) >= 2 for k in kept)
    for k in kept:
        assert k == list(range(10, 10 + len(k)))


def test_fused_matches_oracle_on_tiny(cuda_ok):
    wl = configs.tiny_prefill_2k()
    d = H.device_inputs(wl)
    got = _fused(d).cpu().numpy()
    pos = wl.positions().numpy()
    rows = list(H.seq_rows(wl, 0))
    ref64 = H.oracle_scores_rows(d, 0, rows)
    ref_sel = O.select_blocks(ref64.astype(np.float32), pos[rows], wl.topk, wl.block_size)
    n_near, mism, bad = H.compare_selection(got[rows], ref_sel, ref64, pos[rows], wl.topk, wl.block_size)
    assert bad == 0, (n_near, mism, bad)


@pytest.mark.slow
def test_fused_equals_two_calls_on_last_128k_chunk(cuda_ok):
    """The benchmark's longest chunk (16384 queries against 131072 keys)."""
    wl = configs.chunked_prefill_128k(chunk=7)
    d = H.device_inputs(wl)
    a = _fused(d).cpu().numpy()
    b = _two_calls(d).cpu().numpy()
    assert np.array_equal(a, b), np.argwhere(a != b)[:5]
