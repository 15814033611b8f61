"""Context-parallel MSA (block_sparse_long_13_b200/cp.py) on CPU: gloo ranks.

Decode / verify: each rank holds a contiguous range of one sequence's KV
blocks (pages in its own order); the all-gathered scores, the common top-k and
the log-sum-exp merge of the per-rank partials must reproduce the
single-process path, for 1 and 4 query rows, with query rows on both sides of
a block boundary and on both sides of a rank boundary.

Prefill: each rank holds a contiguous chunk of the queries and its chunk's
new pages; after the all-gather of the pages every rank's chunk must give the
single-process result.

The kernels' place is taken here by the float64 oracle (test infrastructure),
so these tests check the exchange and bookkeeping logic; the kernels have
their own tests, and tests/test_gpu_cp.py drives the same steps through the
library on one GPU."""
import os
import socket
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

BS, HQ, HKV, HI, D, DI, TOPK = 128, 32, 2, 4, 128, 64, 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _tokens(cache, page_ids):
    """[pages][H][bs][d] pages in the given order -> [n*bs][H][d] keys in token order."""
    x = cache[list(page_ids)]
    return x.permute(0, 2, 1, 3).reshape(-1, x.shape[1], x.shape[3])


class OracleOps:
    """The library's calls, computed by the float64 oracle on CPU tensors."""

    def __init__(self):
        from oracle import msa_oracle as O
        self.O = O

    def batch(self, ctx_len, page_ids, num_pages, n_q=1):
        return SimpleNamespace(ctx=int(ctx_len), page_ids=list(page_ids), max_blocks_per_seq=len(page_ids),
                               total_q=int(n_q), max_q_per_seq=int(n_q))

    @staticmethod
    def _pos(b):
        return np.arange(b.ctx - b.total_q, b.ctx)

    def index_scores(self, cfg, b, idx_q, idx_k_cache):
        keys = _tokens(idx_k_cache, b.page_ids)
        s = self.O.block_scores(idx_q, keys, self._pos(b), cfg.num_kv_heads, cfg.block_size, len(b.page_ids))
        return torch.from_numpy(s.astype(np.float32))

    def topk(self, cfg, b, scores):
        sel = self.O.select_blocks(scores.numpy(), self._pos(b), cfg.topk, cfg.block_size)
        return torch.from_numpy(np.asarray(sel, dtype=np.int32))

    def attn(self, cfg, b, q, k_cache, v_cache, sel):
        k, v = _tokens(k_cache, b.page_ids), _tokens(v_cache, b.page_ids)
        s = sel.numpy().copy()
        empty = [(i, g) for i in range(s.shape[0]) for g in range(cfg.num_kv_heads) if not (s[i, g] >= 0).any()]
        for i, g in empty:
            s[i, g, 0] = 0                                   # any block; its result is replaced below
        out, lse = self.O.sparse_attention(q, k, v, self._pos(b), s, cfg.block_size)
        G = cfg.num_q_heads // cfg.num_kv_heads
        for i, g in empty:
            out[i, g * G:(g + 1) * G] = 0.0
            lse[i, g * G:(g + 1) * G] = -np.inf
        return torch.from_numpy(out), torch.from_numpy(lse)

    def merge(self, outs, lses):
        out, lse = self.O.merge_partials(outs.numpy(), lses.numpy())
        return torch.from_numpy(out), torch.from_numpy(lse)


def _data(ctx, seed, n_q=1):
    g = torch.Generator().manual_seed(seed)
    nb = (ctx + BS - 1) // BS
    full = {"k": torch.randn(nb, HKV, BS, D, generator=g, dtype=torch.float64),
            "v": torch.randn(nb, HKV, BS, D, generator=g, dtype=torch.float64),
            "idx_k": torch.randn(nb, HI, BS, DI, generator=g, dtype=torch.float64)}
    q = torch.randn(n_q, HQ, D, generator=g, dtype=torch.float64)
    idx_q = torch.randn(n_q, HI, DI, generator=g, dtype=torch.float64) * 2
    return full, q, idx_q


def _reference(full, q, idx_q, positions):
    from oracle import msa_oracle as O
    nb = int(positions[-1]) // BS + 1
    ident = list(range(nb))
    s64 = O.block_scores(idx_q, _tokens(full["idx_k"], ident), positions, HKV, BS, nb)
    sel = O.select_blocks(s64.astype(np.float32), np.asarray(positions), TOPK, BS)
    out, lse = O.sparse_attention(q, _tokens(full["k"], ident), _tokens(full["v"], ident), positions, sel, BS)
    return sel, out, lse


def _init(rank, ws, port):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))


def _decode_worker(rank, ws, port, ctx, n_q, seed, qout):
    _init(rank, ws, port)
    try:
        import block_sparse_long_13_b200 as msa
        from block_sparse_long_13_b200 import cp
        cfg = msa.Config(num_q_heads=HQ, num_kv_heads=HKV, idx_heads=HI, topk=TOPK)
        full, q, idx_q = _data(ctx, seed, n_q)
        pos = ctx - 1
        nb = pos // BS + 1
        b0, b1 = cp.block_ranges(nb, ws)[rank]
        n_loc = b1 - b0
        # this rank's pages: its blocks in a shuffled local order, plus two unused pages
        perm = torch.randperm(n_loc + 2, generator=torch.Generator().manual_seed(100 + rank)).tolist()
        page_ids = perm[:n_loc]
        local = {}
        for name, t in full.items():
            c = torch.randn((n_loc + 2,) + tuple(t.shape[1:]), dtype=torch.float64)
            for i in range(n_loc):
                c[page_ids[i]] = t[b0 + i]
            local[name] = c
        shard = cp.Shard(b0, b1, page_ids, local["k"], local["v"], local["idx_k"], n_loc + 2)
        out, lse = cp.decode(cfg, shard, q, idx_q, pos, ops=OracleOps())
        _, ref, ref_lse = _reference(full, q, idx_q, np.arange(ctx - n_q, ctx))
        qout.put((rank, float(np.abs(out.numpy() - ref).max()), float(np.abs(lse.numpy() - ref_lse).max())))
    finally:
        dist.destroy_process_group()


def _run(target, ws, *args):
    c = mp.get_context("spawn")
    q = c.Queue()
    port = _free_port()
    procs = [c.Process(target=target, args=(r, ws, port) + args + (q,)) for r in range(ws)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("ws,ctx,n_q", [(2, 1500, 1), (3, 1500, 1), (3, 200, 1), (1, 1500, 1), (2, 1536, 1),
                                        (3, 1537, 1), (2, 1538, 4), (3, 1500, 4), (4, 1030, 4), (2, 131, 4)])
def test_context_parallel_decode_matches_single_process(ws, ctx, n_q):
    # (2, 1538, 4): the 4 queries straddle the block boundary at 1536; (4, 1030, 4): 9 blocks over
    # 4 ranks, queries in the last block; (2, 131, 4): 2 blocks, one per rank, queries on both
    for rank, d_out, d_lse in _run(_decode_worker, ws, ctx, n_q, 7):
        assert d_out <= 1e-10 and d_lse <= 1e-10, (rank, d_out, d_lse)


def _prefill_worker(rank, ws, port, n_tok, seed, qout):
    _init(rank, ws, port)
    try:
        import block_sparse_long_13_b200 as msa
        from block_sparse_long_13_b200 import cp
        cfg = msa.Config(num_q_heads=HQ, num_kv_heads=HKV, idx_heads=HI, topk=TOPK)
        full, q, idx_q = _data(n_tok, seed, n_tok)
        t0, t1 = cp.chunk_ranges(n_tok, ws, BS)[rank]
        p0, p1 = t0 // BS, (t1 + BS - 1) // BS
        sel, out, lse = cp.prefill(cfg, q[t0:t1], idx_q[t0:t1], full["k"][p0:p1], full["v"][p0:p1],
                                   full["idx_k"][p0:p1], n_tok, ops=OracleOps())
        ref_sel, ref, ref_lse = _reference(full, q, idx_q, np.arange(n_tok))
        ok_sel = bool(np.array_equal(sel.numpy(), ref_sel[t0:t1]))
        d_out = float(np.abs(out.numpy() - ref[t0:t1]).max()) if t1 > t0 else 0.0
        d_lse = float(np.abs(lse.numpy() - ref_lse[t0:t1]).max()) if t1 > t0 else 0.0
        qout.put((rank, ok_sel, d_out, d_lse))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,n_tok", [(2, 700), (3, 640), (3, 200)])
def test_context_parallel_prefill_matches_single_process(ws, n_tok):
    # (3, 200): 2 blocks over 3 ranks, one rank without queries
    for rank, ok_sel, d_out, d_lse in _run(_prefill_worker, ws, n_tok, 11):
        assert ok_sel and d_out <= 1e-10 and d_lse <= 1e-10, (rank, ok_sel, d_out, d_lse)


def test_block_ranges_cover_every_block_once():
    from block_sparse_long_13_b200 import cp
    for nb in (1, 2, 5, 1024, 8192):
        for world in (1, 2, 3, 8):
            r = cp.block_ranges(nb, world)
            assert r[0][0] == 0 and r[-1][1] == nb
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            assert max(b1 - b0 for b0, b1 in r) - min(b1 - b0 for b0, b1 in r) <= 1


def test_local_view_positions():
    """Local positions keep in-block offsets; queries past the range see every local key."""
    from block_sparse_long_13_b200 import cp
    sh = lambda b0, b1: cp.Shard(b0, b1, list(range(b1 - b0)), None, None, None, b1 - b0)  # noqa: E731
    # 4 queries at 1534..1537 (blocks 11, 11, 12, 12)
    v = cp.local_view(sh(0, 6), 1537, 4, 128)         # entirely before: first query at the last local key
    assert (v.i0, v.ctx) == (0, 6 * 128 - 1 + 4) and len(v.page_ids) == 7
    v = cp.local_view(sh(6, 12), 1537, 4, 128)        # holds block 11: queries at their own offsets
    assert (v.i0, v.ctx) == (0, 1538 - 6 * 128) and len(v.page_ids) == 7
    v = cp.local_view(sh(12, 13), 1537, 4, 128)       # holds block 12 only: the first two see nothing
    assert (v.i0, v.ctx) == (2, 2) and len(v.page_ids) == 1
    assert cp.local_view(sh(3, 3), 1537, 4, 128) is None


def test_chunk_ranges_are_block_aligned():
    from block_sparse_long_13_b200 import cp
    for n in (1, 127, 128, 700, 16384):
        for w in (1, 2, 3, 5):
            r = cp.chunk_ranges(n, w, 128)
            assert r[0][0] == 0 and r[-1][1] == n
            assert all(a[1] == b[0] and a[1] % 128 == 0 for a, b in zip(r, r[1:]) if a[1] < n)
