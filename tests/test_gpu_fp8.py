"""msa_index_scores_fp8 (e4m3 indexer-key cache) against the oracle.

The cache writer is played by torch on the device: codes = e4m3(clamp(k / s,
+-448)) of the workload's bf16 indexer keys, s = max|k| / 448 (input
preparation, not the library).  The oracle decodes the same bit patterns
itself (oracle/fp8_cache.py `decode_bits`, pinned against torch's decode of
every pattern), multiplies by s and computes the block scores of the
read-back keys in double (the C++ oracle), so the selection that follows is
checked too (exact outside near-ties)."""
import numpy as np
import pytest
import torch

import block_sparse_long_13_b200 as msa
from oracle import cpp as O
from oracle import fp8_cache as F
from workloads import gen

from . import harness as H
from .test_gpu_kernels import _mixed_workload

pytestmark = pytest.mark.gpu


def _fp8_cache(k: torch.Tensor):
    s = float(k.float().abs().max()) / 448.0
    codes = torch.clamp(k.float() / s, -448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    return codes, s


def _oracle_scores(d, codes, s, seq, rows):
    wl = d.wl
    nb = (wl.ctx_len[seq] + wl.block_size - 1) // wl.block_size
    pages = wl.page_table[seq, :nb].long().cuda()
    bits = codes.index_select(0, pages).permute(0, 2, 1, 3).reshape(nb * 128, codes.shape[1], 64)
    keys = F.decode_bits(bits.cpu().numpy()) * np.float64(np.float32(s))
    pos = wl.positions()[list(rows)].numpy()
    iq = d.idx_q[list(rows)].float().cpu().numpy()
    return O.block_scores(iq, keys, pos, wl.num_kv_heads, wl.block_size, wl.max_blocks), pos


@pytest.mark.parametrize("which", ["decode", "decode_nq1", "tiny_verify"])
def test_fp8_index_scores_and_selection_match_oracle(cuda_ok, which):
    if which == "decode":
        wl = _mixed_workload(31, nq_big=False)
    elif which == "decode_nq1":
        wl = _mixed_workload(32, nq=[1] * 5)
    else:
        wl = gen.make_workload("tinyv", seed=33, ctx_len=[2048, 700, 4000], nq=[1, 2, 8], num_q_heads=16,
                               num_kv_heads=1, idx_heads=4, topk=4, plant_count=2, random_pages=True)
    d = H.device_inputs(wl)
    codes, s = _fp8_cache(d.idx_k_cache)
    scores = torch.full((wl.total_q, wl.num_kv_heads, wl.max_blocks), float("nan"), device="cuda")
    msa.index_scores_fp8(d.cfg, d.batch, d.idx_q, codes, s, scores)
    sel = H.run_topk(d, scores)
    assert msa.device_status() == msa.MSA_OK
    got = scores.cpu().numpy()
    got_sel = sel.cpu().numpy()
    worst = -np.inf
    bad = 0
    for seq in range(wl.num_seqs):
        rows = list(H.seq_rows(wl, seq))
        ref64, pos = _oracle_scores(d, codes, s, seq, rows)
        worst = max(worst, H.compare_scores(got[rows], ref64, pos, wl.block_size))
        ref_sel = O.select_blocks(ref64.astype(np.float32), pos, wl.topk, wl.block_size)
        _, _, b = H.compare_selection(got_sel[rows], ref_sel, ref64, pos, wl.topk, wl.block_size)
        bad += b
    assert worst <= 0, worst
    assert bad == 0


def test_fp8_rejects_bad_scale_and_prefill_shapes(cuda_ok):
    wl = _mixed_workload(34, nq_big=False)
    d = H.device_inputs(wl)
    codes, _ = _fp8_cache(d.idx_k_cache)
    scores = torch.empty((wl.total_q, wl.num_kv_heads, wl.max_blocks), device="cuda")
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(msa.MsaError) as ei:
            msa.index_scores_fp8(d.cfg, d.batch, d.idx_q, codes, bad, scores)
        assert ei.value.status == msa.MSA_ERR_INVALID_ARG
    wlp = _mixed_workload(35, nq_big=True)
    dp = H.device_inputs(wlp)
    codesp, s = _fp8_cache(dp.idx_k_cache)
    sp = torch.empty((wlp.total_q, wlp.num_kv_heads, wlp.max_blocks), device="cuda")
    with pytest.raises(msa.MsaError) as ei:
        msa.index_scores_fp8(dp.cfg, dp.batch, dp.idx_q, codesp, s, sp)
    assert ei.value.status == msa.MSA_ERR_UNSUPPORTED


@pytest.mark.slow
def test_fp8_decode_128k_sampled(cuda_ok):
    from workloads import configs
    wl = configs.decode_128k(batch=8)
    d = H.device_inputs(wl)
    codes, s = _fp8_cache(d.idx_k_cache)
    scores = torch.full((wl.total_q, wl.num_kv_heads, wl.max_blocks), float("nan"), device="cuda")
    msa.index_scores_fp8(d.cfg, d.batch, d.idx_q, codes, s, scores)
    assert msa.device_status() == msa.MSA_OK
    got = scores.cpu().numpy()
    for seq in (0, 7):
        rows = list(H.seq_rows(wl, seq))
        ref64, pos = _oracle_scores(d, codes, s, seq, rows)
        assert H.compare_scores(got[rows], ref64, pos, wl.block_size) <= 0
