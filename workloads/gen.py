"""Seeded, device-independent synthetic inputs for the MSA hot path.

This module only decides *what the inputs are*: it holds none of the
method's arithmetic (no dot products, pooling, selection or softmax).  Tests,
the benchmark and the oracle's callers all draw their inputs from here, so the
CUDA path and the CPU oracle see bit-identical tensors without either one
producing data for the other.

Every value is a pure function of (seed, tensor id, logical coordinates):

* a 32-bit integer hash ("lowbias32", C. Wellons, *Hash function prospector*,
  2018: xorshift-multiply rounds with multipliers 0x7feb352d and 0x846ca68b)
  evaluated in int64 torch arithmetic that never overflows, so CPU and CUDA
  give the same bits;
* four 16-bit uniforms from two hash words, summed (Irwin-Hall, n = 4) and
  rescaled to unit variance: an approximately N(0, 1) value that is computed
  in integers, converted exactly to fp32 and multiplied once (one IEEE
  rounding), then optionally shifted by a planted fp32 vector (one IEEE
  addition) and rounded to bf16 (round-to-nearest-even).

Logical coordinates are (sequence, position, head, channel).  Paged caches are
filled by mapping each physical page back to its (sequence, block), so the
same token has the same value whatever page it lands on.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import torch

M32 = 0xFFFFFFFF
POS_STRIDE = 1 << 21  # logical positions per sequence in the counter space (> 1M tokens)

# tensor ids: one independent stream per logical tensor
TID_Q, TID_K, TID_V, TID_IDX_Q, TID_IDX_K = 1, 2, 3, 4, 5
TID_PLANT, TID_U_IDX, TID_U_ATTN, TID_CTX, TID_PERM, TID_SCORES = 10, 11, 12, 13, 14, 15


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for int64 x in [0, 2^32): split c in 16-bit halves so
    no intermediate exceeds 2^49."""
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + ((x * hi) & 0xFFFF) * 65536) & M32


def hash32(x: torch.Tensor) -> torch.Tensor:
    """lowbias32 on int64 tensors holding values in [0, 2^32)."""
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _hash_int(x: int) -> int:
    t = torch.tensor([x & M32], dtype=torch.int64)
    return int(hash32(t)[0])


def stream_key(seed: int, tid: int) -> int:
    """Per-(seed, tensor) 32-bit key."""
    return _hash_int(_hash_int((seed * 0x9E3779B1) & M32) ^ (tid * 0x85EBCA77 & M32))


def hash_words(counter: torch.Tensor, key: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """Two 32-bit words for each non-negative int64 counter (< 2^53)."""
    lo = counter & M32
    hi = counter >> 32
    h = hash32(lo ^ key)
    h = hash32(h ^ ((hi * 0x9E3779B1 + key) & M32))
    w0 = h
    w1 = hash32(h ^ 0xA511E9B3)
    return w0, w1


_SQRT3_OVER_65536 = None


def _scale(device) -> torch.Tensor:
    return torch.tensor([math.sqrt(3.0) / 65536.0], dtype=torch.float32, device=device)


def normal_f32(counter: torch.Tensor, key: int) -> torch.Tensor:
    """Approximately N(0,1) fp32 values, bit-identical on every device."""
    w0, w1 = hash_words(counter, key)
    s = (w0 & 0xFFFF) + (w0 >> 16) + (w1 & 0xFFFF) + (w1 >> 16)  # < 2^18, exact
    return (s - 131070).to(torch.float32) * _scale(counter.device)


def uniform_f64(counter: torch.Tensor, key: int) -> torch.Tensor:
    """Uniform (0, 1) doubles from 53 hash bits (host-side decisions only)."""
    w0, w1 = hash_words(counter, key)
    top = (w0 << 21) | (w1 >> 11)  # 53 bits
    return (top.to(torch.float64) + 0.5) / float(1 << 53)


def unit_vector(seed: int, tid: int, which: int, dim: int) -> torch.Tensor:
    """A seeded random unit direction in R^dim, returned as fp32 (CPU)."""
    cnt = torch.arange(dim, dtype=torch.int64) + which * 4096
    v = normal_f32(cnt, stream_key(seed, tid)).to(torch.float64)
    v = v / torch.linalg.vector_norm(v)
    return v.to(torch.float32)


# ---------------------------------------------------------------------------
# Workload description
# ---------------------------------------------------------------------------

@dataclass
class Workload:
    """A concrete batch: shapes, positions, planted blocks and page layout.

    All index tensors are CPU int32/int64; tensors are materialised on demand.
    ``ctx_len[s]`` counts the KV tokens of sequence s *including* this call's
    queries, which sit at positions ``ctx_len[s] - nq[s] .. ctx_len[s] - 1``.
    """
    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    idx_heads: int
    idx_dim: int
    block_size: int
    topk: int
    ctx_len: List[int]
    nq: List[int]
    page_table: torch.Tensor              # [B][max_blocks] int32 (physical page or -1)
    num_pages: int
    plant_dir: List[torch.Tensor]         # per seq: [nb] int64, -1 = not planted, else direction id
    query_dir: List[int]                  # per seq: direction id added to its queries (-1 none)
    q_pos_offset: List[int] = field(default_factory=list)  # first query position per seq

    @property
    def num_seqs(self) -> int:
        return len(self.ctx_len)

    @property
    def total_q(self) -> int:
        return sum(self.nq)

    @property
    def max_blocks(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def q_start(self) -> List[int]:
        out = [0]
        for n in self.nq:
            out.append(out[-1] + n)
        return out

    def positions(self) -> torch.Tensor:
        """Query positions, one per query row, int64 [total_q]."""
        return torch.cat([torch.arange(c - n, c, dtype=torch.int64)
                          for c, n in zip(self.ctx_len, self.nq)])

    def row_seq(self) -> torch.Tensor:
        return torch.cat([torch.full((n,), s, dtype=torch.int64) for s, n in enumerate(self.nq)])

    def dirs(self, tid_u: int, dim: int) -> torch.Tensor:
        """0.5 * u_d for every direction id used, as fp32 [ndirs+1][dim]; the
        last row is zero (for 'not planted')."""
        nd = max([int(d.max()) if d.numel() else -1 for d in self.plant_dir] + self.query_dir) + 1
        nd = max(nd, getattr(self, "_chunk_dirs", None) or 0)
        rows = [unit_vector(self.seed, tid_u, i, dim) * 0.5 for i in range(nd)]
        rows.append(torch.zeros(dim, dtype=torch.float32))
        return torch.stack(rows)


def _round_half_even(x: float) -> int:
    return int(round(x))


def choose_planted(seed: int, seq: int, candidates: Sequence[int], count: int) -> List[int]:
    """Deterministically pick ``count`` blocks from ``candidates`` (smallest hash)."""
    if count <= 0 or not candidates:
        return []
    c = torch.tensor(list(candidates), dtype=torch.int64)
    h = hash32((c + seq * 1_000_003) & M32 ^ stream_key(seed, TID_PLANT))
    order = sorted(range(len(candidates)), key=lambda i: (int(h[i]), int(c[i])))
    return sorted(int(c[i]) for i in order[:count])


def page_permutation(seed: int, num_pages: int) -> torch.Tensor:
    """A seeded random permutation of physical page ids."""
    h = uniform_f64(torch.arange(num_pages, dtype=torch.int64), stream_key(seed, TID_PERM))
    return torch.argsort(h, stable=True).to(torch.int32)


def make_workload(name: str, *, seed: int, ctx_len: Sequence[int], nq: Sequence[int],
                  num_q_heads: int, num_kv_heads: int, head_dim: int = 128,
                  idx_heads: int, idx_dim: int = 64, block_size: int = 128, topk: int,
                  plant_frac: Optional[float] = None, plant_count: Optional[int] = None,
                  random_pages: bool = False, chunk_dirs: Optional[int] = None,
                  max_blocks: Optional[int] = None) -> Workload:
    """Build a workload.

    Planting: in each sequence ``plant_count`` (or round(plant_frac * nb))
    blocks get every key shifted by +0.5 u along a seeded unit direction u,
    and every query row gets +0.5 u too.  With ``chunk_dirs = C`` the context
    is split in C equal chunks, each with its own direction and its own
    planted blocks among its new key blocks; chunk c's queries use u_c.
    """
    B = len(ctx_len)
    blk = block_size
    nbs = [(c + blk - 1) // blk for c in ctx_len]
    mb = max_blocks if max_blocks is not None else max(nbs)
    total_pages = sum(nbs)
    pt = torch.full((B, mb), -1, dtype=torch.int32)
    if random_pages:
        perm = page_permutation(seed, total_pages)
    else:
        perm = torch.arange(total_pages, dtype=torch.int32)
    off = 0
    for s, nb in enumerate(nbs):
        pt[s, :nb] = perm[off:off + nb]
        off += nb
    plant_dir: List[torch.Tensor] = []
    query_dir: List[int] = []
    for s, nb in enumerate(nbs):
        d = torch.full((nb,), -1, dtype=torch.int64)
        if chunk_dirs:
            per = nb // chunk_dirs
            cnt = plant_count if plant_count is not None else _round_half_even(plant_frac * per)
            for c in range(chunk_dirs):
                for b in choose_planted(seed, s * 64 + c, range(c * per, (c + 1) * per), cnt):
                    d[b] = c
            query_dir.append(-2)  # per-chunk: resolved by position
        else:
            cnt = plant_count if plant_count is not None else _round_half_even(plant_frac * nb)
            for b in choose_planted(seed, s, range(nb), cnt):
                d[b] = 0
            query_dir.append(0)
        plant_dir.append(d)
    wl = Workload(name=name, seed=seed, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                  head_dim=head_dim, idx_heads=idx_heads, idx_dim=idx_dim, block_size=blk,
                  topk=topk, ctx_len=list(ctx_len), nq=list(nq), page_table=pt,
                  num_pages=total_pages, plant_dir=plant_dir, query_dir=query_dir)
    wl._chunk_dirs = chunk_dirs
    return wl


def query_dir_for(wl: Workload, seq: int, pos: torch.Tensor) -> torch.Tensor:
    """Direction id for each query position of sequence ``seq``."""
    qd = wl.query_dir[seq]
    if qd == -2:
        per_tokens = (len(wl.plant_dir[seq]) // wl._chunk_dirs) * wl.block_size
        return (pos // per_tokens).clamp(max=wl._chunk_dirs - 1)
    return torch.full_like(pos, qd)


# ---------------------------------------------------------------------------
# Materialisation
# ---------------------------------------------------------------------------

def _logical_counter(seq: torch.Tensor, pos: torch.Tensor, H: int, D: int) -> torch.Tensor:
    """Counters for a [n][H][D] slab of tokens (seq, pos given per token)."""
    dev = pos.device
    base = (seq * POS_STRIDE + pos).view(-1, 1, 1) * (H * D)
    h = torch.arange(H, dtype=torch.int64, device=dev).view(1, H, 1) * D
    c = torch.arange(D, dtype=torch.int64, device=dev).view(1, 1, D)
    return base + h + c


def _values(counter: torch.Tensor, key: int, add: Optional[torch.Tensor]) -> torch.Tensor:
    x = normal_f32(counter, key)
    if add is not None:
        x = x + add
    return x.to(torch.bfloat16)


def token_tensor(wl: Workload, tid: int, seq: int, pos: torch.Tensor, device="cpu") -> torch.Tensor:
    """bf16 [n][H][D] values of tensor ``tid`` for sequence ``seq`` at the
    given positions (keys/values/queries alike), planted as the workload says."""
    H, D, tid_u, kind = _tensor_shape(wl, tid)
    pos = pos.to(device=device, dtype=torch.int64)
    seq_t = torch.full_like(pos, seq)
    cnt = _logical_counter(seq_t, pos, H, D)
    add = None
    if tid_u is not None:
        dirs = wl.dirs(tid_u, D).to(device)
        if kind == "key":
            pd = wl.plant_dir[seq].to(device)
            blk = torch.clamp(pos // wl.block_size, max=pd.numel() - 1)
            d = pd[blk]
        else:
            d = query_dir_for(wl, seq, pos.cpu()).to(device)
        d = torch.where(d < 0, torch.full_like(d, dirs.shape[0] - 1), d)
        add = dirs[d].view(-1, 1, D)
    return _values(cnt, stream_key(wl.seed, tid), add)


def _tensor_shape(wl: Workload, tid: int):
    if tid == TID_Q:
        return wl.num_q_heads, wl.head_dim, TID_U_ATTN, "query"
    if tid == TID_K:
        return wl.num_kv_heads, wl.head_dim, TID_U_ATTN, "key"
    if tid == TID_V:
        return wl.num_kv_heads, wl.head_dim, None, "value"
    if tid == TID_IDX_Q:
        return wl.idx_heads, wl.idx_dim, TID_U_IDX, "query"
    if tid == TID_IDX_K:
        return wl.idx_heads, wl.idx_dim, TID_U_IDX, "key"
    raise ValueError(tid)


def query_rows(wl: Workload, tid: int, device="cpu") -> torch.Tensor:
    """Query tensor [total_q][H][D] bf16 (tid = TID_Q or TID_IDX_Q)."""
    parts = []
    for s, (c, n) in enumerate(zip(wl.ctx_len, wl.nq)):
        parts.append(token_tensor(wl, tid, s, torch.arange(c - n, c), device))
    return torch.cat(parts)


def page_owner(wl: Workload) -> Tuple[torch.Tensor, torch.Tensor]:
    """For each physical page: (seq, block), -1 for unused pages."""
    seq = torch.full((wl.num_pages,), -1, dtype=torch.int64)
    blk = torch.full((wl.num_pages,), -1, dtype=torch.int64)
    for s in range(wl.num_seqs):
        nb = (wl.ctx_len[s] + wl.block_size - 1) // wl.block_size
        pages = wl.page_table[s, :nb].to(torch.int64)
        seq[pages] = s
        blk[pages] = torch.arange(nb, dtype=torch.int64)
    return seq, blk


def paged_cache(wl: Workload, tid: int, device="cpu", out: Optional[torch.Tensor] = None,
                pages_per_chunk: int = 512) -> torch.Tensor:
    """Paged cache [num_pages][H][block][D] bf16 for keys/values/indexer keys.

    Built page by page from logical coordinates; fills ``out`` in place when
    given (e.g. a preallocated device buffer)."""
    H, D, tid_u, kind = _tensor_shape(wl, tid)
    blk = wl.block_size
    if out is None:
        out = torch.empty((wl.num_pages, H, blk, D), dtype=torch.bfloat16, device=device)
    dev = out.device
    owner_s, owner_b = page_owner(wl)
    key = stream_key(wl.seed, tid)
    page_dir = torch.full((wl.num_pages,), -1, dtype=torch.int64)
    for si in range(wl.num_seqs):
        nb = (wl.ctx_len[si] + blk - 1) // blk
        page_dir[wl.page_table[si, :nb].to(torch.int64)] = wl.plant_dir[si][:nb]
    dirs = wl.dirs(tid_u, D).to(dev) if tid_u is not None else None
    hcoef = torch.arange(H, dtype=torch.int64, device=dev).view(1, H, 1, 1) * D
    ccoef = torch.arange(D, dtype=torch.int64, device=dev).view(1, 1, 1, D)
    icoef = torch.arange(blk, dtype=torch.int64, device=dev).view(1, 1, blk, 1)
    for p0 in range(0, wl.num_pages, pages_per_chunk):
        p1 = min(wl.num_pages, p0 + pages_per_chunk)
        s = owner_s[p0:p1].to(dev)
        b = owner_b[p0:p1].to(dev)
        valid = s >= 0
        s = torch.where(valid, s, torch.zeros_like(s))
        b = torch.where(valid, b, torch.zeros_like(b))
        base = (s * POS_STRIDE + b * blk).view(-1, 1, 1, 1)
        cnt = (base + icoef) * (H * D) + hcoef + ccoef
        add = None
        if dirs is not None:
            d = page_dir[p0:p1].to(dev)
            d = torch.where(d < 0, torch.full_like(d, dirs.shape[0] - 1), d)
            add = dirs[d].view(-1, 1, 1, D)
        out[p0:p1] = _values(cnt, key, add)
    return out


def logical_cache(wl: Workload, tid: int, seq: int, upto: Optional[int] = None,
                  device="cpu") -> torch.Tensor:
    """Logical (unpaged) keys/values [L][H][D] bf16 of one sequence, L = upto
    or the sequence's context length rounded up to whole blocks."""
    blk = wl.block_size
    L = upto if upto is not None else ((wl.ctx_len[seq] + blk - 1) // blk) * blk
    return token_tensor(wl, tid, seq, torch.arange(L), device)


def random_scores(seed: int, rows: int, nb: int, device="cpu") -> torch.Tensor:
    """fp32 [rows][nb] test scores for the top-k step alone (N(0,1)-like)."""
    cnt = torch.arange(rows * nb, dtype=torch.int64, device=device)
    return normal_f32(cnt, stream_key(seed, TID_SCORES)).view(rows, nb)


def ragged_ctx_lens(seed: int, n: int, lo: int = 4096, hi: int = 1 << 20) -> List[int]:
    """Context lengths drawn log-uniform in [lo, hi] (floor of exp)."""
    u = uniform_f64(torch.arange(n, dtype=torch.int64), stream_key(seed, TID_CTX))
    a, b = math.log(lo), math.log(hi)
    return [max(lo, min(hi, int(math.floor(math.exp(a + float(x) * (b - a)))))) for x in u]
