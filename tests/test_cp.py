"""Context-parallel decode (block_sparse_long_13_b200/cp.py) on CPU: gloo ranks
each hold a contiguous range of one sequence's KV blocks (pages in their own
order); the all-gathered scores, the common top-k and the log-sum-exp merge of
the per-rank partials must reproduce the single-process path.  The kernels'
place is taken here by the float64 oracle (test infrastructure), so the test
checks the exchange and bookkeeping logic; the kernels have their own tests."""
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
    """The library's four calls, computed by the float64 oracle on CPU tensors."""

    def __init__(self):
        from oracle import msa_oracle as O
        self.O = O

    def batch(self, ctx_len, page_ids, num_pages):
        return SimpleNamespace(ctx=int(ctx_len), page_ids=list(page_ids), max_blocks_per_seq=len(page_ids))

    def index_scores(self, cfg, b, idx_q, idx_k_cache):
        keys = _tokens(idx_k_cache, b.page_ids)
        s = self.O.block_scores(idx_q, keys, [b.ctx - 1], cfg.num_kv_heads, cfg.block_size, len(b.page_ids))
        return torch.from_numpy(s.astype(np.float32))

    def topk(self, cfg, b, scores):
        sel = self.O.select_blocks(scores.numpy(), np.array([b.ctx - 1]), cfg.topk, cfg.block_size)
        return torch.from_numpy(np.asarray(sel, dtype=np.int32))

    def attn(self, cfg, b, q, k_cache, v_cache, sel):
        k, v = _tokens(k_cache, b.page_ids), _tokens(v_cache, b.page_ids)
        s = sel.numpy().copy()
        empty = [g for g in range(cfg.num_kv_heads) if not (s[0, g] >= 0).any()]
        for g in empty:
            s[0, g, 0] = 0                                   # any block; its result is replaced below
        out, lse = self.O.sparse_attention(q, k, v, [b.ctx - 1], s, cfg.block_size)
        G = cfg.num_q_heads // cfg.num_kv_heads
        for g in empty:
            out[:, g * G:(g + 1) * G] = 0.0
            lse[:, g * G:(g + 1) * G] = -np.inf
        return torch.from_numpy(out), torch.from_numpy(lse)

    def no_keys(self, cfg, q):
        return torch.zeros_like(q), torch.full((1, cfg.num_q_heads), float("-inf"), dtype=torch.float64)

    def merge(self, outs, lses):
        out, lse = self.O.merge_partials(outs.numpy(), lses.numpy())
        return torch.from_numpy(out), torch.from_numpy(lse)


def _data(ctx, seed):
    g = torch.Generator().manual_seed(seed)
    nb = (ctx + BS - 1) // BS
    full = {"k": torch.randn(nb, HKV, BS, D, generator=g, dtype=torch.float64),
            "v": torch.randn(nb, HKV, BS, D, generator=g, dtype=torch.float64),
            "idx_k": torch.randn(nb, HI, BS, DI, generator=g, dtype=torch.float64)}
    q = torch.randn(1, HQ, D, generator=g, dtype=torch.float64)
    idx_q = torch.randn(1, HI, DI, generator=g, dtype=torch.float64) * 2
    return full, q, idx_q


def _worker(rank, ws, port, ctx, seed, qout):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        import block_sparse_long_13_b200 as msa
        from block_sparse_long_13_b200 import cp
        from oracle import msa_oracle as O
        cfg = msa.Config(num_q_heads=HQ, num_kv_heads=HKV, idx_heads=HI, topk=TOPK)
        full, q, idx_q = _data(ctx, seed)
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
        # the single-process path over the whole sequence
        ident = list(range(nb))
        s64 = O.block_scores(idx_q, _tokens(full["idx_k"], ident), [pos], HKV, BS, nb)
        sel = O.select_blocks(s64.astype(np.float32), np.array([pos]), TOPK, BS)
        ref, ref_lse = O.sparse_attention(q, _tokens(full["k"], ident), _tokens(full["v"], ident), [pos], sel, BS)
        qout.put((rank, float(np.abs(out.numpy() - ref).max()), float(np.abs(lse.numpy() - ref_lse).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,ctx", [(2, 1500), (3, 1500), (3, 200), (1, 1500), (2, 1536), (3, 1537)])
def test_context_parallel_decode_matches_single_process(ws, ctx):
    c = mp.get_context("spawn")
    q = c.Queue()
    port = _free_port()
    procs = [c.Process(target=_worker, args=(r, ws, port, ctx, 7, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, d_out, d_lse in res:
        assert d_out <= 1e-10 and d_lse <= 1e-10, (rank, d_out, d_lse)


def test_block_ranges_cover_every_block_once():
    from block_sparse_long_13_b200 import cp
    for nb in (1, 2, 5, 1024, 8192):
        for world in (1, 2, 3, 8):
            r = cp.block_ranges(nb, world)
            assert r[0][0] == 0 and r[-1][1] == nb
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            assert max(b1 - b0 for b0, b1 in r) - min(b1 - b0 for b0, b1 in r) <= 1
