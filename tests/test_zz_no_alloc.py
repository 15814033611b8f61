"""msa_attn_decode_noalloc: the decode attention for callers that cannot
allocate (no workspace argument; its scratch is a fixed device array inside
the library).  Collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.

Checked through the C ABI against msa_attn_decode with a caller workspace, on
two calls in a row with different batches (the second call must not be
disturbed by what the first left in the shared array)."""
import numpy as np
import pytest
import torch

import block_sparse_long_13_b200 as msa
from oracle import cpp as O   # the plain C++ oracle (pinned, and checked against the numpy one)
from workloads import gen

from . import harness as H

pytestmark = pytest.mark.gpu


def _case(seed, ctx, nq):
    wl = gen.make_workload("noalloc", seed=seed, ctx_len=ctx, nq=nq, num_q_heads=64, num_kv_heads=4,
                           idx_heads=8, topk=16, plant_frac=0.05, random_pages=True)
    d = H.device_inputs(wl)
    T = wl.total_q
    s = gen.random_scores(seed, T * 4, wl.max_blocks).view(T, 4, wl.max_blocks)
    sel = torch.from_numpy(O.select_blocks(s.numpy(), wl.positions().numpy(), 16, 128)).cuda()
    return d, sel


def test_noalloc_decode_matches_workspace_decode_twice(cuda_ok):
    cases = [_case(21, [9000, 300, 70000, 128], [1, 4, 2, 1]),
             _case(22, [4096, 131072, 5000], [4, 1, 3])]
    for d, sel in cases:
        out_ref, lse_ref = H.run_attn(d, sel, "decode")
        out = torch.full_like(d.q, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        msa.attn_decode_noalloc(d.cfg, d.batch, d.q, d.k_cache, d.v_cache, sel, out, lse)
        assert msa.device_status() == msa.MSA_OK
        err = float((out.float() - out_ref.float()).abs().max())
        assert err <= H.ATTN_MAX_ABS, err
        assert float((lse - lse_ref).abs().max()) <= H.LSE_MAX_ABS


def test_noalloc_rejects_batches_beyond_its_scratch(cuda_ok):
    # 4096 single-query rows x 4 groups need far more than 16 MiB of split-K scratch
    n = 4096
    wl = gen.make_workload("big", seed=1, ctx_len=[256] * n, nq=[1] * n, num_q_heads=64, num_kv_heads=4,
                           idx_heads=8, topk=16, plant_count=0)
    cfg = H.config_of(wl)
    batch = H.batch_of(wl)
    assert msa.decode_workspace_bytes(cfg, batch) > (16 << 20)
    q = torch.zeros((n, 64, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((wl.num_pages, 4, 128, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((n, 4, 16), dtype=torch.int32, device="cuda")
    with pytest.raises(msa.MsaError) as ei:
        msa.attn_decode_noalloc(cfg, batch, q, kv, kv, sel, torch.empty_like(q))
    assert ei.value.status == msa.MSA_ERR_UNSUPPORTED and "16777216" in str(ei.value)
