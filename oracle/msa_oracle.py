"""Plain CPU oracle for the MiniMax Sparse Attention (MSA) hot path.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke check and
the benchmark's CPU-baseline / reference arm may import this module.  It shares
no code with the CUDA library and imports nothing from it.

Everything is computed in float64 with numpy, one definition at a time, in the
order the method states them.  Sources (page title, then section):

* [daily.dev] "MiniMax M3: 1M-token multimodal reasoning model now available
  with NVIDIA and vLLM support", sections "Summary" and "What makes M3
  different": the KV sequence is cut into 128-token blocks, every block is
  scored, and only the top blocks are attended per query.
* [inteligile] "MiniMax-M3" model page, table "Checked in its code":
  - row "Indexer-selected sparse attention": a lightweight indexer scores the
    keys per head and pools the scores into blocks; k = min(topk_blocks,
    number of key blocks) blocks are kept per query; a kept slot whose score
    is -inf is reported as index -1; sparse_topk_blocks = 16;
  - row "Grouped-query attention": 64 query heads share 4 KV heads, query
    head h reading KV head h // (64 / 4);
  - row "Learnable attention sink": plain softmax, no extra sink logit;
  - row "Gated attention output": no output gate.
  - tag list "inference kernel" / "unfiled": "Exp-free TopK kernel",
    "Two-phase forward", "LSE fusion".
* [24-ai.news] "MiniMax M3 in vLLM: Day-0-Unterstuetzung ...", section "Warum
  ist ein Million-Token-Kontext eine Serving-Herausforderung?": each query or
  GQA query group scores all available 128-token blocks with light indexer
  kernels and keeps the most relevant ones.

Readings where the pages leave a step open (each is also a workload choice):

* pooling = max over the block's causally visible tokens (key j <= query
  position p);
* indexer heads are split contiguously across the KV groups and a group's
  block score is the SUM of its heads' pooled scores;
* raw dot products (no scale, no ReLU, no weights);
* the query's own (current) block cur = p // block_size always takes one of
  the k slots; the other k-1 slots go to the highest-scoring earlier blocks,
  ties broken by the lower block index; blocks after cur are never visible;
* softmax scale 1/sqrt(head_dim);
* selected ids are reported ascending, padded with -1.

Parity pins: see tests/test_oracle_pins.py (brute force on tiny inputs,
closed forms, torch's scaled_dot_product_attention in float64 as the dense
special case, full stable sorts for the selection, hand-worked fixtures under
tests/golden/).
"""
from __future__ import annotations

import math
from typing import Tuple

import numpy as np

NEG_INF = -np.inf


def _f64(x) -> np.ndarray:
    """bf16/fp32 inputs widened exactly to float64."""
    if hasattr(x, "detach"):  # a torch tensor
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# 1. Indexer block scores
# ---------------------------------------------------------------------------

def block_scores(idx_q, idx_k, pos, num_kv_heads: int, block_size: int, nb_out: int) -> np.ndarray:
    """Per-group block scores S[n][num_kv_heads][nb_out] (float64).

    For query row r at position p = pos[r], indexer head h and block b:
        pooled_h(r, b) = max over keys j of block b with j <= p of  q_h(r) . k_h(j)
    and the group score is the sum over the group's indexer heads
        S_g(r, b) = sum_{h in heads(g)} pooled_h(r, b),
    heads(g) = {g*Hi/Hkv, ..., (g+1)*Hi/Hkv - 1}.  A block with no visible key
    (b > p // block_size) scores -inf.  [inteligile, "Indexer-selected sparse
    attention"; 24-ai.news, block scoring per query group]

    idx_q: [n][Hi][di]; idx_k: the sequence's keys in token order, any
    array-like that slices as idx_k[a:b] -> [b-a][Hi][di].
    """
    q = _f64(idx_q)
    n, Hi, di = q.shape
    pos = np.asarray(pos, dtype=np.int64)
    per_group = Hi // num_kv_heads
    out = np.full((n, num_kv_heads, nb_out), NEG_INF)
    for b in range(nb_out):
        lo = b * block_size
        rows = np.nonzero(pos >= lo)[0]          # rows that can see at least key lo
        if rows.size == 0:
            continue
        keys = _f64(idx_k[lo:lo + block_size])   # [<=blk][Hi][di]
        if keys.shape[0] == 0:
            continue
        j = lo + np.arange(keys.shape[0])
        visible = j[None, :] <= pos[rows][:, None]            # [rows][blk]
        acc = np.zeros((rows.size, num_kv_heads))
        for h in range(Hi):
            dots = q[rows, h, :] @ keys[:, h, :].T            # [rows][blk]
            dots = np.where(visible, dots, NEG_INF)
            acc[:, h // per_group] += dots.max(axis=1)
        out[rows, :, b] = acc
    return out


# ---------------------------------------------------------------------------
# 2. Top-k block selection
# ---------------------------------------------------------------------------

def select_blocks(scores, pos, topk: int, block_size: int) -> np.ndarray:
    """Selected block ids [n][Hkv][topk] int32, ascending, -1 padded.

    For row r, group g, cur = pos[r] // block_size:
      R = {cur} U (the min(topk-1, #candidates) best candidates b < cur),
    candidates being the earlier blocks whose score is not -inf (a -inf
    score is reported as -1, never kept), ranked by (score descending, block
    ascending).  The comparison is made on the values given (the kernel
    compares fp32 scores, so callers pass fp32 here).  [inteligile,
    "Indexer-selected sparse attention": k = min(topk, #blocks), -inf -> -1]
    """
    s = np.asarray(scores)
    n, G, nb = s.shape
    pos = np.asarray(pos, dtype=np.int64)
    out = np.full((n, G, topk), -1, dtype=np.int32)
    for r in range(n):
        cur = int(pos[r] // block_size)
        for g in range(G):
            row = s[r, g, :min(cur, nb)]
            cand = [b for b in range(row.shape[0]) if row[b] != NEG_INF]
            ranked = sorted(cand, key=lambda b: (-float(row[b]), b))
            chosen = sorted(ranked[:topk - 1] + [cur])
            out[r, g, :len(chosen)] = chosen
    return out


def boundary_gap(scores64, pos, topk: int, block_size: int):
    """Near-tie report of the selection boundary, per (row, group).

    Ranks the non-forced candidates by (score desc, block asc); s_a is the
    (topk-1)-th ranked score (the last one kept) and s_b the next one.  The
    row is a near-tie when |s_a - s_b| < 1e-3 * max(|s_a|, 1e-6).  Returns
    (near_tie [n][G] bool, s_a [n][G], s_b [n][G]); rows with no rejected
    candidate are never near-ties.
    """
    s = np.asarray(scores64, dtype=np.float64)
    n, G, nb = s.shape
    pos = np.asarray(pos, dtype=np.int64)
    near = np.zeros((n, G), dtype=bool)
    sa = np.full((n, G), np.nan)
    sb = np.full((n, G), np.nan)
    m = topk - 1
    for r in range(n):
        cur = int(pos[r] // block_size)
        for g in range(G):
            row = s[r, g, :min(cur, nb)]
            vals = sorted((float(v) for v in row if v != NEG_INF), reverse=True)
            if m < 1 or len(vals) <= m:
                continue
            a, b = vals[m - 1], vals[m]
            sa[r, g], sb[r, g] = a, b
            near[r, g] = abs(a - b) < 1e-3 * max(abs(a), 1e-6)
    return near, sa, sb


# ---------------------------------------------------------------------------
# 3. Sparse GQA attention over the selected blocks
# ---------------------------------------------------------------------------

def sparse_attention(q, k, v, pos, block_idx, block_size: int,
                     scale: float | None = None) -> Tuple[np.ndarray, np.ndarray]:
    """out [n][Hq][d] and lse [n][Hq] (float64).

    Query head h belongs to group g = h // (Hq/Hkv) and reads KV head g.  Its
    keys are the tokens j <= p of the selected blocks; with s_j = scale *
    q_h . k_j, m = max_j s_j:
        out = sum_j exp(s_j - m) v_j / sum_j exp(s_j - m),
        lse = m + log sum_j exp(s_j - m).
    Plain softmax: no sink logit, no output gate, scale 1/sqrt(d).
    [inteligile, "Grouped-query attention", "Learnable attention sink",
    "Gated attention output"; daily.dev, "What makes M3 different"]

    k, v: the sequence's keys / values in token order, array-likes slicing as
    k[a:b] -> [b-a][Hkv][d].  block_idx: [n][Hkv][topk], -1 = empty slot.
    """
    qq = _f64(q)
    n, Hq, d = qq.shape
    sel = np.asarray(block_idx)
    Hkv = sel.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    pos = np.asarray(pos, dtype=np.int64)
    out = np.zeros((n, Hq, d))
    lse = np.zeros((n, Hq))
    cache = {}

    def block(arr, name, b):
        key = (name, b)
        if key not in cache:
            cache[key] = _f64(arr[b * block_size:(b + 1) * block_size])
        return cache[key]

    for r in range(n):
        p = int(pos[r])
        for g in range(Hkv):
            blocks = [int(b) for b in sel[r, g] if b >= 0]
            ks, vs = [], []
            for b in blocks:
                kb, vb = block(k, "k", b), block(v, "v", b)
                j = b * block_size + np.arange(kb.shape[0])
                keep = j <= p
                ks.append(kb[keep, g, :])
                vs.append(vb[keep, g, :])
            K = np.concatenate(ks)
            V = np.concatenate(vs)
            Qg = qq[r, g * G:(g + 1) * G, :]          # [G][d]
            s = scale * (Qg @ K.T)                    # [G][m]
            mx = s.max(axis=1, keepdims=True)
            e = np.exp(s - mx)
            l = e.sum(axis=1)
            out[r, g * G:(g + 1) * G, :] = (e @ V) / l[:, None]
            lse[r, g * G:(g + 1) * G] = mx[:, 0] + np.log(l)
        if len(cache) > 4096:
            cache.clear()
    return out, lse


# ---------------------------------------------------------------------------
# 4. Two-phase forward: combine partial results by their log-sum-exp
# ---------------------------------------------------------------------------

def merge_partials(outs, lses) -> Tuple[np.ndarray, np.ndarray]:
    """Combine S partial attentions over disjoint key sets.

    outs: [S][...][d] each normalised over its own keys; lses: [S][...].
    L = log sum_s exp(lse_s); out = sum_s exp(lse_s - L) out_s.  Partials
    with lse = -inf (no keys) carry zero weight.  ["LSE fusion",
    "Two-phase forward" tags, inteligile model page]
    """
    o = np.asarray(outs, dtype=np.float64)
    l = np.asarray(lses, dtype=np.float64)
    mx = l.max(axis=0)
    w = np.exp(l - mx[None])
    tot = w.sum(axis=0)
    L = mx + np.log(tot)
    out = (w[..., None] * o).sum(axis=0) / tot[..., None]
    return out, L


# ---------------------------------------------------------------------------
# Whole path for one sequence (used by the CPU baseline and sampled parity)
# ---------------------------------------------------------------------------

def msa_rows(q, idx_q, k, v, idx_k, pos, num_kv_heads: int, block_size: int, topk: int,
             nb_out: int, scale: float | None = None):
    """Indexer scores -> top-k (decided on fp32-rounded scores, as the
    kernel) -> sparse attention, for query rows of ONE sequence."""
    s64 = block_scores(idx_q, idx_k, pos, num_kv_heads, block_size, nb_out)
    sel = select_blocks(s64.astype(np.float32), pos, topk, block_size)
    out, lse = sparse_attention(q, k, v, pos, sel, block_size, scale)
    return s64, sel, out, lse
