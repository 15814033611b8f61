"""Properties that hold at any size, and the failure paths (no GPU fault)."""
import numpy as np
import pytest
import torch

import block_sparse_long_13_b200 as msa
from workloads import configs, gen

from . import harness as H
from .test_gpu_kernels import _mixed_workload, _oracle_selection

pytestmark = pytest.mark.gpu


def _chain(d, path):
    s = H.run_index(d)
    sel = H.run_topk(d, s)
    out, lse = H.run_attn(d, sel, path)
    return s, sel, out, lse


@pytest.mark.parametrize("nq_big,path", [(False, "decode"), (True, "prefill")])
def test_page_permutation_leaves_results_bit_identical(cuda_ok, nq_big, path):
    wl = _mixed_workload(7, nq_big=nq_big)
    d = H.device_inputs(wl)
    a = _chain(d, path)
    perm = torch.randperm(wl.num_pages, generator=torch.Generator().manual_seed(3))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(wl.num_pages)
    pt = wl.page_table.clone()
    m = pt >= 0
    pt[m] = inv[pt[m].long()].to(torch.int32)   # page p moves to inv[p]
    d2 = H.DeviceInputs(wl=wl, cfg=d.cfg, batch=msa.Batch.make(wl.q_start, wl.ctx_len, pt, wl.num_pages),
                        q=d.q, idx_q=d.idx_q, k_cache=d.k_cache[perm.cuda()].contiguous(),
                        v_cache=d.v_cache[perm.cuda()].contiguous(),
                        idx_k_cache=d.idx_k_cache[perm.cuda()].contiguous())
    b = _chain(d2, path)
    pos = wl.positions()
    for x, y, name in zip(a, b, ("scores", "sel", "out", "lse")):
        if name == "scores":
            for t in range(wl.total_q):   # defined entries only
                cur = int(pos[t]) // 128
                assert torch.equal(x[t, :, :cur + 1], y[t, :, :cur + 1]), t
        else:
            assert torch.equal(x, y), name


@pytest.mark.parametrize("path", ["prefill", "decode"])
def test_repeated_runs_are_bit_identical(cuda_ok, path):
    wl = _mixed_workload(8, nq_big=(path == "prefill"))
    d = H.device_inputs(wl)
    a = _chain(d, path)
    b = _chain(d, path)
    pos = wl.positions()
    for t in range(wl.total_q):
        cur = int(pos[t]) // 128
        assert torch.equal(a[0][t, :, :cur + 1], b[0][t, :, :cur + 1])
    for x, y in zip(a[1:], b[1:]):
        assert torch.equal(x, y)


@pytest.mark.parametrize("path", ["prefill", "decode"])
def test_constant_values_give_constant_output(cuda_ok, path):
    wl = _mixed_workload(9, nq_big=(path == "prefill"))
    d = H.device_inputs(wl)
    d.v_cache = torch.ones_like(d.v_cache)
    sel = torch.from_numpy(_oracle_selection(wl, 5)).cuda()
    out, _ = H.run_attn(d, sel, path)
    assert float((out.float() - 1.0).abs().max()) <= 8e-3


def test_out_of_range_page_is_reported_not_faulted(cuda_ok):
    wl = _mixed_workload(10, nq_big=False)
    d = H.device_inputs(wl)
    pt = wl.page_table.clone()
    pt[1, 3] = wl.num_pages + 5          # a visible block of sequence 1
    d.batch = msa.Batch.make(wl.q_start, wl.ctx_len, pt, wl.num_pages)
    H.run_index(d)
    assert msa.device_status() == msa.MSA_ERR_DEVICE_BOUNDS
    sel = torch.from_numpy(_oracle_selection(wl, 6))
    row = wl.q_start[1]                  # first query of sequence 1 selects the bad block 3 in group 0
    if 3 not in sel[row, 0].tolist():
        sel[row, 0, 0] = 3
    sel = sel.cuda()
    # both attention calls document the bad page id as MSA_ERR_DEVICE_BOUNDS (access skipped)
    H.run_attn(d, sel, "decode")
    assert msa.device_status() == msa.MSA_ERR_DEVICE_BOUNDS
    H.run_attn(d, sel, "prefill")
    assert msa.device_status() == msa.MSA_ERR_DEVICE_BOUNDS
    # the context is still usable
    d.batch = H.batch_of(wl)
    H.run_index(d)
    assert msa.device_status() == msa.MSA_OK


def test_selected_block_after_the_query_is_reported(cuda_ok):
    wl = _mixed_workload(11, nq_big=False)
    d = H.device_inputs(wl)
    sel = torch.from_numpy(_oracle_selection(wl, 7)).cuda()
    assert int(wl.positions()[0]) // 128 < wl.max_blocks - 1
    sel[0, 0, 0] = wl.max_blocks - 1     # a block after row 0's own block
    H.run_attn(d, sel, "decode")
    assert msa.device_status() == msa.MSA_ERR_DEVICE_BOUNDS
    H.run_attn(d, sel, "prefill")
    assert msa.device_status() == msa.MSA_ERR_DEVICE_BOUNDS


def test_bounded_wait_times_out_and_context_survives(cuda_ok):
    msa.set_wait_limit_ns(20_000_000)  # 20 ms
    try:
        msa.debug_wait_timeout()
        assert msa.device_status() == msa.MSA_ERR_TIMEOUT
    finally:
        msa.set_wait_limit_ns(2_000_000_000)
    wl = configs.tiny_prefill_2k()
    d = H.device_inputs(wl)
    H.run_index(d)
    assert msa.device_status() == msa.MSA_OK


def test_generator_is_bit_identical_on_cpu_and_gpu(cuda_ok):
    wl = gen.make_workload("g", seed=4, ctx_len=[700, 300], nq=[3, 2], num_q_heads=16, num_kv_heads=1,
                           idx_heads=4, topk=4, plant_count=1, random_pages=True)
    for tid in (gen.TID_K, gen.TID_V, gen.TID_IDX_K):
        assert torch.equal(gen.paged_cache(wl, tid, device="cuda").cpu(), gen.paged_cache(wl, tid))
    for tid in (gen.TID_Q, gen.TID_IDX_Q):
        assert torch.equal(gen.query_rows(wl, tid, device="cuda").cpu(), gen.query_rows(wl, tid))
