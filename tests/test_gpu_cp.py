"""Context-parallel MSA through the library on one GPU.

* msa_merge_partials element by element against the oracle's log-sum-exp
  merge: 1 to 16 partials, partials with lse = -inf, rows whose partials are
  all -inf, lse gaps far beyond exp's range.
* decode / verify: one sequence's blocks split into 1, 2 and 3 shards (each in
  its own page order), the step functions of block_sparse_long_13_b200/cp.py
  driven shard by shard through the library (CudaOps), the per-shard lists
  standing in for the all-gathers; the selection must match the oracle's
  outside near-ties and the merged attention (fed the oracle's selection) must
  match the oracle's attention.
* cp.decode and cp.prefill themselves on a one-rank NCCL group.
* prefill: the query chunks of 2 and 3 emulated ranks, their pages gathered,
  each chunk run against its causal context, sampled rows against the oracle.

Several ranks' kernels never wait on one another here: every emulated rank's
calls finish before the next step reads their results."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import block_sparse_long_13_b200 as msa
from block_sparse_long_13_b200 import cp
from workloads import gen

from . import harness as H

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------- merge kernel

@pytest.mark.parametrize("n", [1, 2, 5, 16])
def test_merge_partials_matches_oracle(cuda_ok, n):
    O = H.oracle()
    g = torch.Generator().manual_seed(n)
    rows, heads, d = 37, 8, 128
    outs = torch.randn((n, rows, heads, d), generator=g).to(torch.bfloat16)
    lses = torch.randn((n, rows, heads), generator=g) * 4
    lses[:, ::3] += torch.linspace(-90, 90, n).view(n, 1, 1)     # gaps far beyond exp's range
    drop = torch.rand((n, rows, heads), generator=g) < 0.3
    lses[drop] = float("-inf")
    lses[:, 5] = float("-inf")                                    # every partial of row 5 is empty
    if n > 1:
        lses[1:, 6] = float("-inf")                               # only the first partial of row 6 counts
    out = torch.empty((rows, heads, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((rows, heads), dtype=torch.float32, device="cuda")
    msa.merge_partials(outs.cuda(), lses.cuda(), out, lse)
    assert msa.device_status() == msa.MSA_OK
    got, got_lse = out.float().cpu().numpy(), lse.cpu().numpy()
    empty = np.isneginf(lses.numpy()).all(axis=0)                # [rows][heads]
    assert (got[empty] == 0).all() and np.isneginf(got_lse[empty]).all()
    live = ~empty
    ref, ref_lse = O.merge_partials(outs.float().numpy()[:, live], lses.numpy()[:, live])
    err = np.abs(got[live] - ref)
    assert err.max() <= H.ATTN_MAX_ABS and err.mean() <= H.ATTN_MEAN_ABS, (err.max(), err.mean())
    assert np.abs(got_lse[live] - ref_lse).max() <= H.LSE_MAX_ABS
    if n > 1:                                                     # weight exactly 1 on the one partial
        one = np.isfinite(lses[0, 6].numpy())
        np.testing.assert_array_equal(got[6][one], outs[0, 6].float().numpy()[one])


def test_merge_partials_rejects_mismatched_shapes(cuda_ok):
    outs = torch.zeros((2, 4, 3, 128), dtype=torch.bfloat16, device="cuda")
    lses = torch.zeros((2, 4, 3), device="cuda")
    with pytest.raises(msa.MsaError):
        msa.merge_partials(outs, lses[:, :3], torch.empty((4, 3, 128), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(msa.MsaError):
        msa.merge_partials(outs, lses, torch.empty((4, 2, 128), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(msa.MsaError):
        msa.merge_partials(outs, lses, torch.empty((4, 3, 128), dtype=torch.bfloat16, device="cuda"),
                           torch.empty((5,), device="cuda"))


# ----------------------------------------------------------------- decode / verify, emulated ranks

def _sequence(ctx, n_q, seed):
    wl = gen.make_workload("cp", seed=seed, ctx_len=[ctx], nq=[n_q], num_q_heads=64, num_kv_heads=4,
                           idx_heads=8, topk=16, plant_frac=0.05, random_pages=True)
    return H.device_inputs(wl)


def _shards(d, world):
    """Rank r holds its blocks in its own shuffled page order plus one unused page."""
    wl = d.wl
    nb = (wl.ctx_len[0] - 1) // 128 + 1
    shards = []
    for r, (b0, b1) in enumerate(cp.block_ranges(nb, world)):
        n_loc = b1 - b0
        perm = torch.randperm(n_loc + 1, generator=torch.Generator().manual_seed(50 + r)).tolist()
        page_ids = perm[:n_loc]
        caches = []
        for full in (d.k_cache, d.v_cache, d.idx_k_cache):
            c = torch.zeros((n_loc + 1,) + tuple(full.shape[1:]), dtype=full.dtype, device="cuda")
            for i in range(n_loc):
                c[page_ids[i]] = full[int(wl.page_table[0, b0 + i])]
            caches.append(c)
        shards.append(cp.Shard(b0, b1, page_ids, caches[0], caches[1], caches[2], n_loc + 1))
    return shards


def _oracle_rows(d):
    rows = list(range(d.wl.total_q))
    ref64 = H.oracle_scores_rows(d, 0, rows)
    pos = d.wl.positions().numpy()
    ref_sel = H.oracle().select_blocks(ref64.astype(np.float32), pos, d.wl.topk, 128)
    ref, ref_lse = H.oracle_attention_rows(d, 0, rows, ref_sel)
    return ref64, ref_sel, ref, ref_lse, pos


@pytest.mark.parametrize("world,ctx,n_q", [(1, 3000, 1), (2, 3000, 1), (3, 3000, 1), (3, 1537, 1),
                                           (2, 2690, 4), (3, 1538, 4), (2, 131, 4)])
def test_cp_decode_steps_through_the_library(cuda_ok, world, ctx, n_q):
    d = _sequence(ctx, n_q, seed=world * 100 + n_q)
    ops = cp.CudaOps()
    shards = _shards(d, world)
    pos = ctx - 1
    nb = pos // 128 + 1
    ranges = cp.block_ranges(nb, world)
    width = max(b1 - b0 for b0, b1 in ranges)
    parts = [cp.local_scores(d.cfg, sh, d.idx_q, pos, width, ops) for sh in shards]
    row = cp.assemble(parts, ranges, nb)
    sel = cp.select(d.cfg, row, pos, ops)
    ref64, ref_sel, ref, ref_lse, qpos = _oracle_rows(d)
    got = row.cpu().numpy()
    assert H.compare_scores(got, ref64, qpos, 128) <= 0
    near, mism, bad = H.compare_selection(sel.cpu().numpy(), ref_sel, ref64, qpos, 16, 128)
    assert bad == 0, (near, mism, bad)
    # attention of every shard on the oracle's selection, merged by msa_merge_partials
    rs = torch.from_numpy(ref_sel).cuda()
    outs, lses = zip(*[cp.local_attention(d.cfg, sh, d.q, rs, pos, ops) for sh in shards])
    out, lse = ops.merge(torch.stack(outs), torch.stack(lses))
    assert msa.device_status() == msa.MSA_OK
    mx, mean = H.attn_errors(out, ref)
    assert mx <= H.ATTN_MAX_ABS and mean <= H.ATTN_MEAN_ABS, (mx, mean)
    assert float(np.abs(lse.cpu().numpy() - ref_lse).max()) <= H.LSE_MAX_ABS


# ----------------------------------------------------------------- one-rank process group

@pytest.fixture
def one_rank_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        yield
    finally:
        dist.destroy_process_group()


def test_cp_decode_on_a_one_rank_group(cuda_ok, one_rank_group):
    """With one rank, cp.decode runs the single-process path on the shard's own page order,
    plus a merge of one partial (weight 1): the results must be bit-identical."""
    d = _sequence(2000, 4, seed=5)
    sh = _shards(d, 1)[0]
    out, lse = cp.decode(d.cfg, sh, d.q, d.idx_q, 1999)
    want_sel = H.run_topk(d, H.run_index(d))
    want, want_lse = H.run_attn(d, want_sel, "decode")
    assert msa.device_status() == msa.MSA_OK
    assert torch.equal(out, want) and torch.equal(lse, want_lse)


def _prefill_inputs(n_tok, seed):
    wl = gen.make_workload("cpp", seed=seed, ctx_len=[n_tok], nq=[n_tok], num_q_heads=64, num_kv_heads=4,
                           idx_heads=8, topk=16, plant_frac=0.05, random_pages=False)
    return H.device_inputs(wl)


def test_cp_prefill_on_a_one_rank_group(cuda_ok, one_rank_group):
    d = _prefill_inputs(1500, seed=6)
    sel, out, lse = cp.prefill(d.cfg, d.q, d.idx_q, d.k_cache[:12], d.v_cache[:12], d.idx_k_cache[:12], 1500)
    want = H.run_topk(d, H.run_index(d))
    assert torch.equal(sel, want)
    ref_out, ref_lse = H.run_attn(d, want, "prefill")
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    assert msa.device_status() == msa.MSA_OK


@pytest.mark.parametrize("world,n_tok", [(2, 3000), (3, 2100)])
def test_cp_prefill_chunks_match_oracle(cuda_ok, world, n_tok):
    d = _prefill_inputs(n_tok, seed=world)
    ops = cp.CudaOps()
    ranges = cp.chunk_ranges(n_tok, world, 128)
    counts = [(b - a + 127) // 128 for a, b in ranges]
    pieces = {name: [full[a // 128:(b + 127) // 128] for a, b in ranges]
              for name, full in (("k", d.k_cache), ("v", d.v_cache), ("ik", d.idx_k_cache))}
    width = max(counts)

    def gather_of(name):
        padded = [torch.cat([p, p.new_zeros((width - p.shape[0],) + tuple(p.shape[1:]))]) for p in pieces[name]]
        return lambda x: padded

    rng = np.random.default_rng(world)
    O = H.oracle()
    for r, (t0, t1) in enumerate(ranges):
        k = cp.gather_pages(pieces["k"][r], gather_of("k"), counts)
        v = cp.gather_pages(pieces["v"][r], gather_of("v"), counts)
        ik = cp.gather_pages(pieces["ik"][r], gather_of("ik"), counts)
        assert torch.equal(k, d.k_cache[:k.shape[0]]) and torch.equal(ik, d.idx_k_cache[:ik.shape[0]])
        sel, out, lse = cp.prefill_chunk(d.cfg, d.q[t0:t1], d.idx_q[t0:t1], k, v, ik, t0, t1, ops)
        rows = sorted(set(int(x) for x in rng.integers(t0, t1, size=12)) | {t0, t1 - 1})
        ref64 = H.oracle_scores_rows(d, 0, rows)
        pos = np.asarray(rows)
        ref_sel = O.select_blocks(ref64.astype(np.float32), pos, 16, 128)
        loc = [x - t0 for x in rows]
        near, mism, bad = H.compare_selection(sel[loc].cpu().numpy(), ref_sel, ref64, pos, 16, 128)
        assert bad == 0, (r, near, mism, bad)
        # attention of the chunk on the oracle's selection for the sampled rows
        sel[loc] = torch.from_numpy(ref_sel).cuda()
        out, lse = ops.attn(d.cfg, ops.batch(t1, list(range(k.shape[0])), k.shape[0], t1 - t0),
                            d.q[t0:t1], k, v, sel)
        ref, ref_lse = H.oracle_attention_rows(d, 0, rows, ref_sel)
        mx, mean = H.attn_errors(out[loc], ref)
        assert mx <= H.ATTN_MAX_ABS and mean <= H.ATTN_MEAN_ABS, (r, mx, mean)
    assert msa.device_status() == msa.MSA_OK
