"""The MSA workloads, by name and size.

Shapes follow the MiniMax-M3 attention configuration (64 query heads over 4
KV heads, head_dim 128, 128-token KV blocks, 16 selected blocks); the
indexer's size (8 heads x 64), its max-pooling and the planted blocks are the
workload's own choices, stated here.

``tiny_prefill_2k``      1 x 2048 tokens, 16/1 heads, indexer 4x64, k=4, 4 planted blocks
``prefill_32k``          1 x 32768 tokens, 64/4 heads, indexer 8x64, k=16, 5% planted
``chunked_prefill_128k`` 131072 context as 8 chunks of 16384 queries, 3% planted per chunk
``decode_128k``          64 sequences x 131072 cached tokens, 1 query each, random page table, 2% planted
``decode_1m``            8 sequences x 1048576 cached tokens, 1 query each, random page table, 1% planted
``verify_ragged``        32 sequences, context log-uniform in [4096, 2^20], 4 queries each, 1% planted
"""
from __future__ import annotations

from typing import List

from .gen import Workload, make_workload, ragged_ctx_lens

M3_HEADS = dict(num_q_heads=64, num_kv_heads=4, head_dim=128, idx_heads=8, idx_dim=64,
                block_size=128, topk=16)


def tiny_prefill_2k(seed: int = 0) -> Workload:
    return make_workload("tiny_prefill_2k", seed=seed, ctx_len=[2048], nq=[2048],
                         num_q_heads=16, num_kv_heads=1, head_dim=128, idx_heads=4, idx_dim=64,
                         block_size=128, topk=4, plant_count=4)


def prefill_32k(seed: int = 0) -> Workload:
    return make_workload("prefill_32k", seed=seed, ctx_len=[32768], nq=[32768],
                         plant_frac=0.05, **M3_HEADS)


def prefill_8k(seed: int = 0) -> Workload:
    """A smaller M3-shaped prefill (8192 tokens, 5% planted) for profiling."""
    return make_workload("prefill_8k", seed=seed, ctx_len=[8192], nq=[8192], plant_frac=0.05, **M3_HEADS)


def chunked_prefill_128k(seed: int = 0, chunk: int = None) -> List[Workload] | Workload:
    """The 8 chunks (or one of them).  Chunk c queries positions
    [16384c, 16384(c+1)) against the causal context 16384(c+1); all chunks
    share one sequence whose chunk c owns its own direction and 4 planted
    blocks among its 128 new key blocks."""
    n_chunks, per = 8, 16384
    full = make_workload("chunked_prefill_128k", seed=seed, ctx_len=[n_chunks * per],
                         nq=[per], plant_count=4, chunk_dirs=n_chunks, **M3_HEADS)
    out = []
    for c in range(n_chunks):
        wl = make_workload(f"chunked_prefill_128k/c{c}", seed=seed, ctx_len=[n_chunks * per],
                           nq=[per], plant_count=4, chunk_dirs=n_chunks, **M3_HEADS)
        wl.ctx_len = [per * (c + 1)]
        nb = wl.ctx_len[0] // 128
        wl.page_table = full.page_table[:, :nb].clone()
        wl.plant_dir = [full.plant_dir[0].clone()]
        wl.num_pages = full.num_pages
        out.append(wl)
    return out if chunk is None else out[chunk]


def decode_128k(seed: int = 0, batch: int = 64) -> Workload:
    return make_workload("decode_128k", seed=seed, ctx_len=[131072] * batch, nq=[1] * batch,
                         plant_frac=0.02, random_pages=True, **M3_HEADS)


def decode_1m(seed: int = 0, batch: int = 8) -> Workload:
    return make_workload("decode_1m", seed=seed, ctx_len=[1 << 20] * batch, nq=[1] * batch,
                         plant_frac=0.01, random_pages=True, **M3_HEADS)


def verify_ragged(seed: int = 0, batch: int = 32) -> Workload:
    ctx = ragged_ctx_lens(seed, batch)
    return make_workload("verify_ragged", seed=seed, ctx_len=ctx, nq=[4] * batch,
                         plant_frac=0.01, random_pages=True, **M3_HEADS)


ALL = {
    "tiny_prefill_2k": tiny_prefill_2k,
    "prefill_32k": prefill_32k,
    "chunked_prefill_128k": chunked_prefill_128k,
    "decode_128k": decode_128k,
    "decode_1m": decode_1m,
    "verify_ragged": verify_ragged,
}
