"""Python face of the plain C++ CPU oracle (oracle/msa_oracle.cpp, built as
oracle/liboracle.so with g++): the same functions, arguments and results as
oracle/msa_oracle.py, so the pins and the parity tests run against either.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke check and
the benchmark's CPU-baseline / reference arm may import this module.  It shares
no code with the CUDA library and imports nothing from it.  This module only
marshals arrays; every step of the arithmetic is in the C++ file, whose header
cites the passages it follows.

Inputs that are float32 (bf16 data widened exactly) are passed as float32 and
widened to double inside the oracle; anything else is passed as float64.  The
threads (std::thread) split independent outputs; `set_threads` fixes their
number (default: the CPUs this process may run on).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "msa_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")
CXXFLAGS = ["-O2", "-std=c++17", "-pthread", "-shared", "-fPIC"]

_lib = None
_lock = threading.Lock()
_threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (building the checker, not running it)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp"
        subprocess.run(["g++", *CXXFLAGS, "-o", tmp, SRC], check=True)
        os.replace(tmp, LIB)
    return LIB


def set_threads(n: int) -> None:
    global _threads
    _threads = max(1, int(n))


def threads() -> int:
    return _threads


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
            for name in ("oracle_block_scores_f32", "oracle_block_scores_f64"):
                f = getattr(lib, name)
                f.argtypes = [P, P, i64, i32, i32, P, i64, i32, i32, i32, P, i32]
                f.restype = ctypes.c_int
            lib.oracle_select_blocks.argtypes = [P, P, i64, i32, i32, i32, i32, P]
            lib.oracle_boundary_gap.argtypes = [P, P, i64, i32, i32, i32, i32, P, P, P]
            for name in ("oracle_sparse_attention_f32", "oracle_sparse_attention_f64"):
                f = getattr(lib, name)
                f.argtypes = [P, P, i64, i32, i32, P, P, P, i64, i32, P, i32, i32, dbl, P, P, i32]
                f.restype = ctypes.c_int
            lib.oracle_merge_partials.argtypes = [P, P, i32, i64, i32, P, P]
            _lib = lib
    return _lib


def hardware_threads() -> int:
    return int(_load().oracle_hardware_threads())


def _np(x) -> np.ndarray:
    """torch tensors and array-likes to numpy; float32 stays float32, the rest float64."""
    if hasattr(x, "detach"):                     # a torch tensor
        t = x.detach().to("cpu")
        narrow = str(t.dtype) in ("torch.bfloat16", "torch.float16", "torch.float32")
        x = t.float().numpy() if narrow else t.double().numpy()
    x = np.asarray(x)
    return x if x.dtype == np.float32 else x.astype(np.float64)


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _common(*arrays):
    """One dtype for all inputs: float32 when every one is float32, else float64."""
    f32 = all(a.dtype == np.float32 for a in arrays)
    dt = np.float32 if f32 else np.float64
    return f32, [np.ascontiguousarray(a, dtype=dt) for a in arrays]


# ---------------------------------------------------------------------------
# 1. Indexer block scores
# ---------------------------------------------------------------------------

def block_scores(idx_q, idx_k, pos, num_kv_heads: int, block_size: int, nb_out: int) -> np.ndarray:
    """Per-group block scores S[n][num_kv_heads][nb_out] (float64); see msa_oracle.cpp (1).
    idx_k: the sequence's keys in token order, any array-like slicing as idx_k[a:b] -> [b-a][Hi][di]."""
    q = _np(idx_q)
    n, Hi, di = q.shape
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    out = np.empty((n, num_kv_heads, nb_out), dtype=np.float64)
    if n == 0 or nb_out == 0:
        return out
    upto = int(min(nb_out * block_size, int(pos.max()) + 1))
    keys = _np(idx_k[0:upto]) if upto > 0 else np.zeros((0, Hi, di))
    keys = keys.reshape(-1, Hi, di)
    f32, (q, keys) = _common(q, keys)
    fn = _load().oracle_block_scores_f32 if f32 else _load().oracle_block_scores_f64
    rc = fn(_ptr(q), _ptr(pos), n, Hi, di, _ptr(keys), keys.shape[0], num_kv_heads, block_size, nb_out, _ptr(out),
            _threads)
    if rc:
        raise ValueError(f"oracle_block_scores: bad arguments ({rc})")
    return out


# ---------------------------------------------------------------------------
# 2. Top-k block selection and the near-tie report
# ---------------------------------------------------------------------------

def select_blocks(scores, pos, topk: int, block_size: int) -> np.ndarray:
    """Selected block ids [n][Hkv][topk] int32, ascending, -1 padded; see msa_oracle.cpp (2).
    The comparison is made on the values given (fp32 scores are widened exactly)."""
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float64))
    n, G, nb = s.shape
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    out = np.empty((n, G, topk), dtype=np.int32)
    if _load().oracle_select_blocks(_ptr(s), _ptr(pos), n, G, nb, topk, block_size, _ptr(out)):
        raise ValueError("oracle_select_blocks: bad arguments")
    return out


def boundary_gap(scores64, pos, topk: int, block_size: int):
    """(near_tie [n][G] bool, s_a [n][G], s_b [n][G]); see msa_oracle.cpp (near-tie report)."""
    s = np.ascontiguousarray(np.asarray(scores64, dtype=np.float64))
    n, G, nb = s.shape
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    near = np.zeros((n, G), dtype=np.uint8)
    sa = np.empty((n, G))
    sb = np.empty((n, G))
    if _load().oracle_boundary_gap(_ptr(s), _ptr(pos), n, G, nb, topk, block_size, _ptr(near), _ptr(sa), _ptr(sb)):
        raise ValueError("oracle_boundary_gap: bad arguments")
    return near.astype(bool), sa, sb


# ---------------------------------------------------------------------------
# 3. Sparse GQA attention over the selected blocks
# ---------------------------------------------------------------------------

def sparse_attention(q, k, v, pos, block_idx, block_size: int,
                     scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """out [n][Hq][d] and lse [n][Hq] (float64); see msa_oracle.cpp (3).
    k, v: the sequence's keys / values in token order, array-likes slicing as
    k[a:b] -> [b-a][Hkv][d]; only the selected blocks are read.  block_idx: [n][Hkv][topk]."""
    qq = _np(q)
    n, Hq, d = qq.shape
    sel = np.ascontiguousarray(np.asarray(block_idx, dtype=np.int32))
    Hkv, topk = sel.shape[1], sel.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    blocks = sorted(set(int(b) for b in sel[sel >= 0].reshape(-1)))
    nblk = (blocks[-1] + 1) if blocks else 0
    kb = {b: _np(k[b * block_size:(b + 1) * block_size]) for b in blocks}
    vb = {b: _np(v[b * block_size:(b + 1) * block_size]) for b in blocks}
    f32, arrs = _common(qq, *kb.values(), *vb.values())
    qq = arrs[0]
    kb = dict(zip(blocks, arrs[1:1 + len(blocks)]))
    vb = dict(zip(blocks, arrs[1 + len(blocks):]))
    kptr = (ctypes.c_void_p * max(1, nblk))()
    vptr = (ctypes.c_void_p * max(1, nblk))()
    lens = np.zeros(max(1, nblk), dtype=np.int32)
    for b in blocks:
        kptr[b], vptr[b] = _ptr(kb[b]), _ptr(vb[b])
        lens[b] = min(kb[b].shape[0], vb[b].shape[0])
    out = np.empty((n, Hq, d), dtype=np.float64)
    lse = np.empty((n, Hq), dtype=np.float64)
    fn = _load().oracle_sparse_attention_f32 if f32 else _load().oracle_sparse_attention_f64
    rc = fn(_ptr(qq), _ptr(pos), n, Hq, d, ctypes.addressof(kptr), ctypes.addressof(vptr), _ptr(lens), nblk, Hkv,
            _ptr(sel), topk, block_size, float(scale), _ptr(out), _ptr(lse), _threads)
    if rc:
        raise ValueError(f"oracle_sparse_attention: bad arguments ({rc})")
    return out, lse


# ---------------------------------------------------------------------------
# 4. Two-phase forward: combine partial results by their log-sum-exp
# ---------------------------------------------------------------------------

def merge_partials(outs, lses) -> Tuple[np.ndarray, np.ndarray]:
    """outs [S][...][d], lses [S][...] -> (out [...][d], L [...]); see msa_oracle.cpp (4)."""
    o = np.ascontiguousarray(np.asarray(outs, dtype=np.float64))
    l = np.ascontiguousarray(np.asarray(lses, dtype=np.float64))
    S = l.shape[0]
    d = o.shape[-1]
    units = int(np.prod(l.shape[1:], dtype=np.int64))
    out = np.empty(l.shape[1:] + (d,), dtype=np.float64)
    lse = np.empty(l.shape[1:], dtype=np.float64)
    _load().oracle_merge_partials(_ptr(o), _ptr(l), S, units, d, _ptr(out), _ptr(lse))
    return out, lse


# ---------------------------------------------------------------------------
# Whole path for one sequence
# ---------------------------------------------------------------------------

def msa_rows(q, idx_q, k, v, idx_k, pos, num_kv_heads: int, block_size: int, topk: int,
             nb_out: int, scale: Optional[float] = None):
    """Indexer scores -> top-k (decided on fp32-rounded scores, as the kernel) -> sparse
    attention, for query rows of ONE sequence."""
    s64 = block_scores(idx_q, idx_k, pos, num_kv_heads, block_size, nb_out)
    sel = select_blocks(s64.astype(np.float32), pos, topk, block_size)
    out, lse = sparse_attention(q, k, v, pos, sel, block_size, scale)
    return s64, sel, out, lse
