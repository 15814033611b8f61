"""Context-parallel MSA decode: one long sequence whose KV blocks are split
over the ranks of a process group (one GPU per rank).

The pages list context parallelism among the upcoming serving work (daily.dev
"MiniMax M3: 1M-token multimodal reasoning model ...", section "What's
coming").  The method itself fixes what each rank must agree on: the block
scores (every visible block, "MiniMax-M3" inteligile model page, row
"Indexer-selected sparse attention"), the one top-k selection per query group
made from all of them, and the log-sum-exp merge of partial attentions over
disjoint key sets (tags "LSE fusion", "Two-phase forward").  So a decode step
takes four steps, two of which exchange data:

1. every rank scores its own blocks: its pages form a local sequence in which
   each key keeps its offset inside its block, and whose last position is the
   query's position when the rank holds the query's own block (else every
   local key is visible);
2. the local scores are all-gathered and every rank assembles the same
   global score row and runs the same top-k on it (the query's own block
   forced, ties to the lower block id);
3. every rank attends over the selected blocks that it holds (none: lse = -inf);
4. the partial (out, lse) pairs are all-gathered and merged by log-sum-exp.

Every compute step is a library call (`CudaOps`); the collectives are
torch.distributed's.  Ranks hold contiguous block ranges (`block_ranges`);
one query row per call.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple

import torch
import torch.distributed as dist


def block_ranges(num_blocks: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous split of blocks 0 .. num_blocks-1 over `world` ranks: rank r holds
    [r * B // world, (r + 1) * B // world)."""
    return [(r * num_blocks // world, (r + 1) * num_blocks // world) for r in range(world)]


@dataclass
class Shard:
    """What one rank holds of the sequence: global blocks [b0, b1), their pages in this rank's
    caches (page_ids[i] holds block b0 + i) and the caches themselves."""
    b0: int
    b1: int
    page_ids: List[int]
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    idx_k_cache: torch.Tensor
    num_pages: int


class CudaOps:
    """The library's calls on this rank's GPU."""

    def __init__(self):
        import block_sparse_long_13_b200 as msa
        self.msa = msa

    def batch(self, ctx_len: int, page_ids, num_pages: int):
        return self.msa.Batch.make([0, 1], [ctx_len], [list(page_ids)], num_pages, device="cuda")

    def index_scores(self, cfg, batch, idx_q, idx_k_cache):
        s = torch.empty((1, cfg.num_kv_heads, batch.max_blocks_per_seq), dtype=torch.float32, device="cuda")
        self.msa.index_scores(cfg, batch, idx_q, idx_k_cache, s)
        return s

    def topk(self, cfg, batch, scores):
        sel = torch.empty((1, cfg.num_kv_heads, cfg.topk), dtype=torch.int32, device="cuda")
        self.msa.topk_blocks(cfg, batch, scores, sel)
        return sel

    def attn(self, cfg, batch, q, k_cache, v_cache, sel):
        out = torch.empty_like(q)
        lse = torch.empty((1, cfg.num_q_heads), dtype=torch.float32, device="cuda")
        ws = torch.empty(self.msa.decode_workspace_bytes(cfg, batch), dtype=torch.uint8, device="cuda")
        self.msa.attn_decode(cfg, batch, q, k_cache, v_cache, sel, out, lse, ws)
        return out, lse

    def no_keys(self, cfg, q):
        """The partial of a rank that holds none of the selected blocks: weight zero."""
        return torch.zeros_like(q), torch.full((1, cfg.num_q_heads), float("-inf"), dtype=torch.float32, device="cuda")

    def merge(self, outs, lses):
        out = torch.empty_like(outs[0])
        lse = torch.empty_like(lses[0])
        self.msa.merge_partials(outs, lses, out, lse)
        return out, lse


def decode(cfg, shard: Shard, q, idx_q, pos: int, group=None, ops=None):
    """One query row at absolute position `pos` of a sequence spread over the group.
    q: [1][Hq][head_dim], idx_q: [1][Hi][idx_dim] (the same on every rank).
    Returns (out [1][Hq][head_dim], lse [1][Hq]), the same on every rank."""
    ops = ops or CudaOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    bs = cfg.block_size
    nb = pos // bs + 1                                  # blocks 0 .. the query's own block
    ranges = block_ranges(nb, world)
    if (shard.b0, shard.b1) != ranges[rank]:
        raise ValueError(f"rank {rank} holds blocks [{shard.b0}, {shard.b1}), expected {ranges[rank]}")
    n_loc = shard.b1 - shard.b0
    width = max(b1 - b0 for b0, b1 in ranges)
    hkv = cfg.num_kv_heads

    # 1. local scores: the rank's blocks as one local sequence, offsets inside blocks kept
    loc = None
    scores = torch.full((1, hkv, width), float("-inf"), dtype=torch.float32, device=q.device)
    if n_loc > 0:
        ctx = n_loc * bs if shard.b1 < nb else (n_loc - 1) * bs + pos % bs + 1
        loc = ops.batch(ctx, shard.page_ids, shard.num_pages)
        scores[..., :n_loc] = ops.index_scores(cfg, loc, idx_q, shard.idx_k_cache)[..., :n_loc]
    # 2. every rank assembles the same global row and selects on it
    parts = [torch.empty_like(scores) for _ in range(world)]
    dist.all_gather(parts, scores, group=group)
    row = torch.full((1, hkv, nb), float("-inf"), dtype=torch.float32, device=q.device)
    for (b0, b1), part in zip(ranges, parts):
        row[..., b0:b1] = part[..., :b1 - b0]
    glob = ops.batch(pos + 1, [0] * nb, 1)              # top-k reads only positions and sizes
    sel = ops.topk(cfg, glob, row)
    # 3. attention over the selected blocks this rank holds
    if loc is not None:
        mine = (sel >= shard.b0) & (sel < shard.b1)
        local_sel = torch.where(mine, sel - shard.b0, torch.full_like(sel, -1))
        if bool(mine.any()):
            out, lse = ops.attn(cfg, loc, q, shard.k_cache, shard.v_cache, local_sel)
        else:
            out, lse = ops.no_keys(cfg, q)
    else:
        out, lse = ops.no_keys(cfg, q)
    # 4. all partials to every rank, merged by log-sum-exp
    outs = [torch.empty_like(out) for _ in range(world)]
    lses = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(outs, out.contiguous(), group=group)
    dist.all_gather(lses, lse.contiguous(), group=group)
    return ops.merge(torch.stack(outs), torch.stack(lses))
