"""Shared helpers of the parity tests: device inputs from the seeded generator,
calls through the C ABI, oracle evaluation on host rows, comparisons."""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import block_sparse_long_13_b200 as msa
from oracle import cpp as O   # the plain C++ oracle (pinned, and checked against the numpy one)
from workloads import gen

# tolerances (bf16 inputs, fp32 accumulation, fp64 oracle)
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
LSE_MAX_ABS = 2e-3
NEAR_TIE_REL = 1e-3


def oracle():
    """The oracle module the parity tests compare against."""
    return O


def score_tol(ref: np.ndarray) -> np.ndarray:
    """Indexer scores: fp32 sums of exact bf16 products vs float64."""
    return 1e-3 + 1e-5 * np.abs(ref)


@dataclass
class DeviceInputs:
    wl: gen.Workload
    cfg: msa.Config
    batch: msa.Batch
    q: torch.Tensor
    idx_q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    idx_k_cache: torch.Tensor


def config_of(wl: gen.Workload) -> msa.Config:
    return msa.Config(num_q_heads=wl.num_q_heads, num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim,
                      idx_heads=wl.idx_heads, idx_dim=wl.idx_dim, block_size=wl.block_size, topk=wl.topk)


def batch_of(wl: gen.Workload, device="cuda") -> msa.Batch:
    return msa.Batch.make(wl.q_start, wl.ctx_len, wl.page_table, wl.num_pages, device=device)


def device_inputs(wl: gen.Workload, device="cuda", caches: Optional[Dict[str, torch.Tensor]] = None) -> DeviceInputs:
    """Materialise a workload on the device (caches may be shared between
    workloads that use the same pages, e.g. the chunks of one prefill)."""
    caches = caches if caches is not None else {}
    if "k" not in caches:
        caches["k"] = gen.paged_cache(wl, gen.TID_K, device=device)
        caches["v"] = gen.paged_cache(wl, gen.TID_V, device=device)
        caches["idx_k"] = gen.paged_cache(wl, gen.TID_IDX_K, device=device)
    return DeviceInputs(wl=wl, cfg=config_of(wl), batch=batch_of(wl, device),
                        q=gen.query_rows(wl, gen.TID_Q, device=device),
                        idx_q=gen.query_rows(wl, gen.TID_IDX_Q, device=device),
                        k_cache=caches["k"], v_cache=caches["v"], idx_k_cache=caches["idx_k"])


# ----------------------------------------------------------------- CUDA path calls

def run_index(d: DeviceInputs) -> torch.Tensor:
    s = torch.full((d.wl.total_q, d.wl.num_kv_heads, d.wl.max_blocks), float("nan"), device=d.q.device)
    msa.index_scores(d.cfg, d.batch, d.idx_q, d.idx_k_cache, s)
    return s


def run_topk(d: DeviceInputs, scores: torch.Tensor) -> torch.Tensor:
    sel = torch.full((d.wl.total_q, d.wl.num_kv_heads, d.wl.topk), -7, dtype=torch.int32, device=d.q.device)
    msa.topk_blocks(d.cfg, d.batch, scores, sel)
    return sel


def run_attn(d: DeviceInputs, sel: torch.Tensor, path: str = "prefill"):
    out = torch.empty_like(d.q)
    lse = torch.empty((d.wl.total_q, d.wl.num_q_heads), dtype=torch.float32, device=d.q.device)
    if path == "prefill":
        nb = msa.prefill_workspace_bytes(d.cfg, d.batch)
        ws = torch.empty(nb, dtype=torch.uint8, device=d.q.device)
        msa.attn_prefill(d.cfg, d.batch, d.q, d.k_cache, d.v_cache, sel, out, lse, ws)
    else:
        nb = msa.decode_workspace_bytes(d.cfg, d.batch)
        ws = torch.empty(nb, dtype=torch.uint8, device=d.q.device)
        msa.attn_decode(d.cfg, d.batch, d.q, d.k_cache, d.v_cache, sel, out, lse, ws)
    return out, lse


# ----------------------------------------------------------------- host views for the oracle

class PagedSeq:
    """Token-order view of one sequence of a paged device cache, fetched on
    demand block by block (slices must cover whole blocks or parts of one)."""

    def __init__(self, cache: torch.Tensor, page_row: torch.Tensor, block_size: int):
        self.cache = cache
        self.pages = page_row.cpu().tolist()
        self.blk = block_size
        self._memo: Dict[int, np.ndarray] = {}

    def block(self, b: int) -> np.ndarray:
        if b not in self._memo:
            if len(self._memo) > 2048:
                self._memo.clear()
            t = self.cache[self.pages[b]]                       # [H][blk][D]
            self._memo[b] = t.permute(1, 0, 2).float().cpu().numpy()
        return self._memo[b]

    def __getitem__(self, sl: slice) -> np.ndarray:
        a, z = sl.start, sl.stop
        parts = []
        while a < z:
            b = a // self.blk
            off = a - b * self.blk
            n = min(z - a, self.blk - off)
            parts.append(self.block(b)[off:off + n])
            a += n
        return np.concatenate(parts) if parts else np.zeros((0,))


class WholeSeq:
    """Whole logical sequence copied to host at once (for the indexer keys)."""

    def __init__(self, cache: torch.Tensor, page_row: torch.Tensor, nb: int):
        pages = page_row[:nb].long()
        t = cache.index_select(0, pages.to(cache.device))       # [nb][H][blk][D]
        self.arr = t.permute(0, 2, 1, 3).reshape(-1, t.shape[1], t.shape[3]).float().cpu().numpy()

    def __getitem__(self, sl: slice) -> np.ndarray:
        return self.arr[sl]


def seq_rows(wl: gen.Workload, s: int) -> range:
    qs = wl.q_start
    return range(qs[s], qs[s + 1])


def oracle_scores_rows(d: DeviceInputs, s: int, rows: Sequence[int]) -> np.ndarray:
    """float64 [len(rows)][Hkv][max_blocks] for query rows of sequence s."""
    wl = d.wl
    nb = (wl.ctx_len[s] + wl.block_size - 1) // wl.block_size
    keys = WholeSeq(d.idx_k_cache, wl.page_table[s], nb)
    pos = wl.positions()[list(rows)].numpy()
    iq = d.idx_q[list(rows)].float().cpu().numpy()
    return O.block_scores(iq, keys, pos, wl.num_kv_heads, wl.block_size, wl.max_blocks)


def oracle_attention_rows(d: DeviceInputs, s: int, rows: Sequence[int], sel: np.ndarray):
    wl = d.wl
    k = PagedSeq(d.k_cache, wl.page_table[s], wl.block_size)
    v = PagedSeq(d.v_cache, wl.page_table[s], wl.block_size)
    pos = wl.positions()[list(rows)].numpy()
    q = d.q[list(rows)].float().cpu().numpy()
    return O.sparse_attention(q, k, v, pos, sel, wl.block_size)


# ----------------------------------------------------------------- comparisons

def compare_scores(got: np.ndarray, ref: np.ndarray, pos: np.ndarray, blk: int) -> float:
    """Max excess over tolerance on the visible entries (b <= cur); <= 0 passes."""
    worst = -np.inf
    for i in range(ref.shape[0]):
        cur = int(pos[i] // blk)
        g = got[i, :, :cur + 1].astype(np.float64)
        r = ref[i, :, :cur + 1]
        assert np.isfinite(g).all(), f"row {i}: non-finite score in the visible range"
        worst = max(worst, float((np.abs(g - r) - score_tol(r)).max()))
    return worst


def compare_selection(got: np.ndarray, ref_sel: np.ndarray, ref_scores64: np.ndarray, pos: np.ndarray,
                      topk: int, blk: int):
    """Exact set equality except at reported near-ties, where differing
    blocks must lie inside the tie band of the boundary score.
    Returns (near_tie_rows, mismatched_rows, bad_rows)."""
    near, sa, sb = O.boundary_gap(ref_scores64, pos, topk, blk)
    n_near = int(near.sum())
    mism = bad = 0
    for i in range(got.shape[0]):
        for g in range(got.shape[1]):
            a = set(int(x) for x in got[i, g] if x >= 0)
            b = set(int(x) for x in ref_sel[i, g] if x >= 0)
            if a == b and list(got[i, g]) == list(ref_sel[i, g]):
                continue
            mism += 1
            if not near[i, g] or len(a) != len(b):
                bad += 1
                continue
            band = NEAR_TIE_REL * max(abs(sa[i, g]), 1e-6)
            for blk_id in a ^ b:
                v = ref_scores64[i, g, blk_id]
                if not (sb[i, g] - band <= v <= sa[i, g] + band):
                    bad += 1
                    break
    return n_near, mism, bad


def attn_errors(got: torch.Tensor, ref: np.ndarray):
    g = got.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    return float(err.max()), float(err.mean())
