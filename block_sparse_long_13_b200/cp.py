"""Context-parallel MSA: one long sequence spread over the ranks of a process
group (one GPU per rank).

The pages list context parallelism among the upcoming serving work (daily.dev
"MiniMax M3: 1M-token multimodal reasoning model ...", section "What's
coming").  The method itself fixes what the ranks must agree on: the block
scores (every visible block, "MiniMax-M3" inteligile model page, row
"Indexer-selected sparse attention"), the one top-k selection per query group
made from all of them, and the log-sum-exp merge of partial attentions over
disjoint key sets (tags "LSE fusion", "Two-phase forward").

Decode and verify (`decode`): the sequence's KV blocks are split over the
ranks in contiguous ranges (`block_ranges`); the call's few query rows (the
last tokens of the context, causal among themselves) are on every rank.  Four
steps, two of which exchange data:

1. `local_scores`: every rank scores its own blocks.  Its pages form a local
   sequence in which each key keeps its offset inside its block; a query that
   lies past the rank's range sees every local key, one inside it sees the
   local keys up to its own position, one before it sees none (its scores
   there are -inf);
2. the local scores are all-gathered; every rank assembles the same global
   score rows (`assemble`) and runs the same top-k on them (`select`: the
   query's own block kept, ties to the lower block id);
3. `local_attention`: every rank attends over the selected blocks it holds
   (none: out = 0, lse = -inf, weight zero);
4. the partial (out, lse) pairs are all-gathered and merged by log-sum-exp.

Prefill (`prefill`): the query tokens are split instead, in contiguous
block-aligned chunks, one per rank; each rank writes its chunk's keys, values
and indexer keys into its own pages.  One all-gather of those pages gives
every rank the causal context of its chunk, and each rank then runs the
chunked-prefill path (indexer, top-k, block-major attention) on its own
queries: the selection and the attention of a query need nothing else, so no
partial results cross ranks.

Every compute step is a library call (`CudaOps`); the collectives are
torch.distributed's.  The step functions also run without a process group
(a list of per-rank tensors in place of each all-gather), which is how one GPU
drives several emulated ranks in the tests.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence, Tuple

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

    def batch(self, ctx_len: int, page_ids, num_pages: int, n_q: int = 1):
        return self.msa.Batch.make([0, n_q], [ctx_len], [list(page_ids)], num_pages, device="cuda")

    def index_scores(self, cfg, batch, idx_q, idx_k_cache):
        s = torch.empty((batch.total_q, cfg.num_kv_heads, batch.max_blocks_per_seq), dtype=torch.float32,
                        device="cuda")
        self.msa.index_scores(cfg, batch, idx_q, idx_k_cache, s)
        return s

    def topk(self, cfg, batch, scores):
        sel = torch.empty((batch.total_q, cfg.num_kv_heads, cfg.topk), dtype=torch.int32, device="cuda")
        self.msa.topk_blocks(cfg, batch, scores, sel)
        return sel

    def attn(self, cfg, batch, q, k_cache, v_cache, sel):
        out = torch.empty_like(q)
        lse = torch.empty((batch.total_q, cfg.num_q_heads), dtype=torch.float32, device="cuda")
        if batch.max_q_per_seq <= 8:
            ws = torch.empty(self.msa.decode_workspace_bytes(cfg, batch), dtype=torch.uint8, device="cuda")
            self.msa.attn_decode(cfg, batch, q, k_cache, v_cache, sel, out, lse, ws)
        else:
            ws = torch.empty(self.msa.prefill_workspace_bytes(cfg, batch), dtype=torch.uint8, device="cuda")
            self.msa.attn_prefill(cfg, batch, q, k_cache, v_cache, sel, out, lse, ws)
        return out, lse

    def merge(self, outs, lses):
        out = torch.empty_like(outs[0])
        lse = torch.empty_like(lses[0])
        self.msa.merge_partials(outs, lses, out, lse)
        return out, lse


# ------------------------------------------------------------------ decode / verify: KV blocks split

@dataclass
class LocalView:
    """How one rank presents its blocks to the library for a call's queries."""
    i0: int                 # queries i0 .. n_q-1 see at least one local key; earlier ones see none
    ctx: int                # local context length (the local queries are its last tokens)
    page_ids: List[int]     # local block -> page, padded past the rank's range (never selected)


def local_view(shard: Shard, pos_last: int, n_q: int, bs: int) -> Optional[LocalView]:
    """Local positions keep every key's offset inside its block.  Query i (global
    position P_i = pos_last - n_q + 1 + i) sits at local position P_i - b0 * bs when
    it lies inside the rank's range; queries past the range see every local key, so
    the first of them may sit anywhere at or after the last local key."""
    n_loc = shard.b1 - shard.b0
    if n_loc <= 0:
        return None
    p0 = pos_last - n_q + 1
    i0 = max(0, shard.b0 * bs - p0)
    if i0 >= n_q:
        return None
    p_first = min(p0 + i0, shard.b1 * bs - 1) - shard.b0 * bs
    ctx = p_first + (n_q - i0)
    need = (ctx - 1) // bs + 1
    pages = list(shard.page_ids) + [shard.page_ids[-1]] * max(0, need - n_loc)
    return LocalView(i0=i0, ctx=ctx, page_ids=pages)


def local_scores(cfg, shard: Shard, idx_q, pos_last: int, width: int, ops) -> torch.Tensor:
    """Step 1: scores [n_q][H_kv][width] of this rank's blocks (local block j in column j);
    entries a query cannot see are -inf."""
    n_q = idx_q.shape[0]
    bs = cfg.block_size
    out = torch.full((n_q, cfg.num_kv_heads, width), float("-inf"), dtype=torch.float32, device=idx_q.device)
    lv = local_view(shard, pos_last, n_q, bs)
    if lv is None:
        return out
    n_loc = shard.b1 - shard.b0
    loc = ops.batch(lv.ctx, lv.page_ids, shard.num_pages, n_q - lv.i0)
    s = ops.index_scores(cfg, loc, idx_q[lv.i0:], shard.idx_k_cache)[..., :n_loc]
    # local block j is visible to query i when j <= its local block (later entries are undefined)
    p_loc = lv.ctx - (n_q - lv.i0) + torch.arange(n_q - lv.i0, device=s.device)
    vis = torch.arange(n_loc, device=s.device)[None, :] <= (p_loc // bs)[:, None]
    out[lv.i0:, :, :n_loc] = torch.where(vis[:, None, :], s, torch.full_like(s, float("-inf")))
    return out


def assemble(parts: Sequence[torch.Tensor], ranges: Sequence[Tuple[int, int]], nb: int) -> torch.Tensor:
    """Step 2a: the global score rows [n_q][H_kv][nb] from every rank's local scores."""
    n_q, hkv = parts[0].shape[:2]
    row = torch.full((n_q, hkv, nb), float("-inf"), dtype=torch.float32, device=parts[0].device)
    for (b0, b1), part in zip(ranges, parts):
        row[..., b0:b1] = part[..., :b1 - b0]
    return row


def select(cfg, row: torch.Tensor, pos_last: int, ops) -> torch.Tensor:
    """Step 2b: the common top-k on the assembled rows (reads only positions and sizes)."""
    n_q, _, nb = row.shape
    glob = ops.batch(pos_last + 1, [0] * nb, 1, n_q)
    return ops.topk(cfg, glob, row)


def local_attention(cfg, shard: Shard, q, sel: torch.Tensor, pos_last: int, ops):
    """Step 3: (out [n_q][H_q][d], lse [n_q][H_q]) over the selected blocks this rank holds."""
    n_q = q.shape[0]
    out = torch.zeros_like(q)
    lse_dtype = torch.float64 if q.dtype == torch.float64 else torch.float32   # float64: oracle stand-ins
    lse = torch.full((n_q, cfg.num_q_heads), float("-inf"), dtype=lse_dtype, device=q.device)
    lv = local_view(shard, pos_last, n_q, cfg.block_size)
    if lv is None:
        return out, lse
    s = sel[lv.i0:]
    mine = (s >= shard.b0) & (s < shard.b1)
    if not bool(mine.any()):
        return out, lse
    local_sel = torch.where(mine, s - shard.b0, torch.full_like(s, -1)).contiguous()
    loc = ops.batch(lv.ctx, lv.page_ids, shard.num_pages, n_q - lv.i0)
    o, l = ops.attn(cfg, loc, q[lv.i0:].contiguous(), shard.k_cache, shard.v_cache, local_sel)
    out[lv.i0:] = o
    lse[lv.i0:] = l
    return out, lse


def _all_gather(x: torch.Tensor, group) -> List[torch.Tensor]:
    parts = [torch.empty_like(x) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, x.contiguous(), group=group)
    return parts


def decode(cfg, shard: Shard, q, idx_q, pos: int, group=None, ops=None):
    """The call's n_q = q.shape[0] query rows (1 for decode, a few for a verify step)
    at positions pos - n_q + 1 .. pos of a sequence spread over the group.
    q: [n_q][Hq][head_dim], idx_q: [n_q][Hi][idx_dim] (the same on every rank).
    Returns (out [n_q][Hq][head_dim], lse [n_q][Hq]), the same on every rank."""
    ops = ops or CudaOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    nb = pos // cfg.block_size + 1                      # blocks 0 .. the last query's own block
    ranges = block_ranges(nb, world)
    if (shard.b0, shard.b1) != ranges[rank]:
        raise ValueError(f"rank {rank} holds blocks [{shard.b0}, {shard.b1}), expected {ranges[rank]}")
    width = max(b1 - b0 for b0, b1 in ranges)
    scores = local_scores(cfg, shard, idx_q, pos, width, ops)
    row = assemble(_all_gather(scores, group), ranges, nb)
    sel = select(cfg, row, pos, ops)
    out, lse = local_attention(cfg, shard, q, sel, pos, ops)
    return ops.merge(torch.stack(_all_gather(out, group)), torch.stack(_all_gather(lse, group)))


# ------------------------------------------------------------------ prefill: query chunks split

def chunk_ranges(num_tokens: int, world: int, bs: int) -> List[Tuple[int, int]]:
    """Contiguous query chunks [t0, t1) of a prefill, one per rank, cut at block boundaries so
    that every rank's new keys fill whole pages of its own (the last chunk may end mid-block)."""
    nb = (num_tokens + bs - 1) // bs
    return [(min(num_tokens, b0 * bs), min(num_tokens, b1 * bs)) for b0, b1 in block_ranges(nb, world)]


def gather_pages(local: torch.Tensor, gather: Callable[[torch.Tensor], List[torch.Tensor]],
                 counts: Sequence[int]) -> torch.Tensor:
    """The sequence's pages in block order from every rank's pages of its own chunk.
    local: [n_r][H][bs][d] (ranks pad to the widest count for the collective)."""
    width = max(counts)
    pad = local
    if local.shape[0] < width:
        pad = torch.cat([local, local.new_zeros((width - local.shape[0],) + tuple(local.shape[1:]))])
    parts = gather(pad)
    return torch.cat([p[:n] for p, n in zip(parts, counts)]).contiguous()


def prefill_chunk(cfg, q, idx_q, k_cache, v_cache, idx_k_cache, t0: int, t1: int, ops):
    """One rank's chunk of queries [t0, t1) against the causal context [0, t1) held in
    block-ordered caches (page b holds block b).  Returns (block_idx, out, lse)."""
    n = t1 - t0
    nb = (t1 + cfg.block_size - 1) // cfg.block_size
    b = ops.batch(t1, list(range(nb)), k_cache.shape[0], n)
    scores = ops.index_scores(cfg, b, idx_q, idx_k_cache)
    sel = ops.topk(cfg, b, scores)
    out, lse = ops.attn(cfg, b, q, k_cache, v_cache, sel)
    return sel, out, lse


def prefill(cfg, q, idx_q, k_pages, v_pages, idx_k_pages, num_tokens: int, group=None, ops=None):
    """This rank's chunk of a prefill of `num_tokens` tokens spread over the group.
    q / idx_q: the rank's chunk rows; k_pages / v_pages / idx_k_pages: the pages of its
    chunk's new keys, values and indexer keys ([n][H][bs][d], block order).  The pages of
    every rank are all-gathered, then the chunk runs against its causal context.
    Returns (block_idx, out, lse) of the chunk."""
    ops = ops or CudaOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    bs = cfg.block_size
    ranges = chunk_ranges(num_tokens, world, bs)
    t0, t1 = ranges[rank]
    if q.shape[0] != t1 - t0:
        raise ValueError(f"rank {rank} holds {q.shape[0]} query rows, its chunk is [{t0}, {t1})")
    counts = [(b - a + bs - 1) // bs for a, b in ranges]
    gather = lambda x: _all_gather(x, group)  # noqa: E731
    k = gather_pages(k_pages, gather, counts)
    v = gather_pages(v_pages, gather, counts)
    ik = gather_pages(idx_k_pages, gather, counts)
    if t1 == t0:
        return (torch.empty((0, cfg.num_kv_heads, cfg.topk), dtype=torch.int32, device=q.device),
                torch.empty_like(q), torch.empty((0, cfg.num_q_heads), dtype=torch.float32, device=q.device))
    return prefill_chunk(cfg, q, idx_q, k, v, ik, t0, t1, ops)
