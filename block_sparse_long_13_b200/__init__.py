"""MiniMax Sparse Attention (MSA) hot path for B200: Python binding of libmsa.so.

Argument marshalling only: every step runs in the CUDA library behind the C
ABI declared in include/msa.h.  Tensors must be CUDA tensors on the current
device; work is enqueued on the current torch stream (or the given one).

    import block_sparse_long_13_b200 as msa
    cfg = msa.Config(num_q_heads=64, num_kv_heads=4, idx_heads=8, topk=16)
    batch = msa.Batch.make(q_start, ctx_len, page_table, num_pages, device="cuda")
    msa.index_scores(cfg, batch, idx_q, idx_k_cache, block_scores)
    msa.topk_blocks(cfg, batch, block_scores, block_idx)
    msa.attn_prefill(cfg, batch, q, k_cache, v_cache, block_idx, out, lse, workspace)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

EXPORTS = (
    "msa_index_scores", "msa_topk_blocks", "msa_attn_prefill", "msa_attn_decode",
    "msa_prefill_workspace_bytes", "msa_decode_workspace_bytes", "msa_get_device_status",
    "msa_set_wait_limit_ns", "msa_debug_wait_timeout", "msa_status_string", "msa_last_error",
    "msa_version", "msa_attn_decode_noalloc", "msa_index_topk", "msa_set_timing_events",
    "msa_qknorm_rope_insert", "msa_merge_partials", "msa_index_scores_fp8",
)

MSA_OK, MSA_ERR_INVALID_ARG, MSA_ERR_UNSUPPORTED, MSA_ERR_CUDA, MSA_ERR_TIMEOUT, MSA_ERR_DEVICE_BOUNDS = range(6)


class MsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"msa status {status}: {msg}")
        self.status = status


class _CConfig(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("idx_heads", ctypes.c_int32),
                ("idx_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


class _CBatch(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("total_q", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("max_q_per_seq", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("q_start", ctypes.c_void_p),
                ("ctx_len", ctypes.c_void_p), ("page_table", ctypes.c_void_p)]


_lib_handle = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmsa.so (built in-tree); raises if it is missing."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m block_sparse_long_13_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    cfgp, batp = ctypes.POINTER(_CConfig), ctypes.POINTER(_CBatch)
    sigs = {
        "msa_index_scores": [cfgp, batp, P, P, P, P],
        "msa_index_scores_fp8": [cfgp, batp, P, P, ctypes.c_float, P, P],
        "msa_topk_blocks": [cfgp, batp, P, P, P],
        "msa_index_topk": [cfgp, batp, P, P, P, P],
        "msa_set_timing_events": [P, ctypes.c_int32],
        "msa_attn_prefill": [cfgp, batp, P, P, P, P, P, P, P, ctypes.c_size_t, P],
        "msa_attn_decode": [cfgp, batp, P, P, P, P, P, P, P, ctypes.c_size_t, P],
        "msa_attn_decode_noalloc": [cfgp, batp, P, P, P, P, P, P, P],
        "msa_qknorm_rope_insert": [cfgp, batp, P, P, P, P, P, P, P, ctypes.c_int32, ctypes.c_float, ctypes.c_float, P],
        "msa_merge_partials": [ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, P, P, P, P, P],
        "msa_prefill_workspace_bytes": [cfgp, batp],
        "msa_decode_workspace_bytes": [cfgp, batp],
        "msa_get_device_status": [P],
        "msa_set_wait_limit_ns": [ctypes.c_uint64],
        "msa_debug_wait_timeout": [P],
        "msa_status_string": [ctypes.c_int],
        "msa_last_error": [],
        "msa_version": [],
    }
    for name, args in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.msa_prefill_workspace_bytes.restype = ctypes.c_size_t
    lib.msa_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.msa_status_string.restype = ctypes.c_char_p
    lib.msa_last_error.restype = ctypes.c_char_p
    _lib_handle = lib
    return lib


def _check(status: int) -> None:
    if status != MSA_OK:
        lib = load_library()
        raise MsaError(status, lib.msa_last_error().decode() or lib.msa_status_string(status).decode())


@dataclass
class Config:
    num_q_heads: int = 64
    num_kv_heads: int = 4
    head_dim: int = 128
    idx_heads: int = 8
    idx_dim: int = 64
    block_size: int = 128
    topk: int = 16
    softmax_scale: float = 0.0  # <= 0: 1/sqrt(head_dim)

    def _c(self) -> _CConfig:
        return _CConfig(self.num_q_heads, self.num_kv_heads, self.head_dim, self.idx_heads,
                        self.idx_dim, self.block_size, self.topk, self.softmax_scale)


@dataclass
class Batch:
    """Varlen batch: device int32 index tensors plus their host-side sizes."""
    q_start: torch.Tensor        # [num_seqs + 1] int32
    ctx_len: torch.Tensor        # [num_seqs] int32
    page_table: torch.Tensor     # [num_seqs][max_blocks_per_seq] int32
    total_q: int
    max_q_per_seq: int
    num_pages: int

    @property
    def num_seqs(self) -> int:
        return int(self.ctx_len.numel())

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.page_table.shape[1])

    @staticmethod
    def make(q_start: Sequence[int], ctx_len: Sequence[int], page_table, num_pages: int,
             device="cuda") -> "Batch":
        qs = torch.as_tensor(list(q_start), dtype=torch.int32)
        nq = (qs[1:] - qs[:-1])
        pt = torch.as_tensor(page_table, dtype=torch.int32)
        return Batch(q_start=qs.to(device), ctx_len=torch.as_tensor(list(ctx_len), dtype=torch.int32).to(device),
                     page_table=pt.contiguous().to(device), total_q=int(qs[-1]),
                     max_q_per_seq=max(1, int(nq.max())) if nq.numel() else 1, num_pages=int(num_pages))

    def _c(self, host_only: bool = False) -> _CBatch:
        """C view; with host_only the index arrays may live anywhere (size queries)."""
        if not host_only:
            for t in (self.q_start, self.ctx_len, self.page_table):
                _need(t, torch.int32, "batch index arrays")
        return _CBatch(self.num_seqs, self.total_q, self.max_blocks_per_seq, self.max_q_per_seq,
                       self.num_pages, self.q_start.data_ptr(), self.ctx_len.data_ptr(),
                       self.page_table.data_ptr())


def _need(t: Optional[torch.Tensor], dtype, what: str) -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise MsaError(MSA_ERR_INVALID_ARG, f"{what} must be a CUDA tensor")
    if t.dtype != dtype:
        raise MsaError(MSA_ERR_INVALID_ARG, f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise MsaError(MSA_ERR_INVALID_ARG, f"{what} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def index_scores(cfg: Config, batch: Batch, idx_q, idx_k_cache, block_scores, stream=None) -> None:
    lib = load_library()
    _check(lib.msa_index_scores(ctypes.byref(cfg._c()), ctypes.byref(batch._c()),
                                _need(idx_q, torch.bfloat16, "idx_q"),
                                _need(idx_k_cache, torch.bfloat16, "idx_k_cache"),
                                _need(block_scores, torch.float32, "block_scores"), _stream(stream)))


def index_scores_fp8(cfg: Config, batch: Batch, idx_q, idx_k_cache_e4m3, k_scale: float, block_scores,
                     stream=None) -> None:
    """Indexer block scores over an e4m3 indexer-key cache (uint8 codes, value = code * k_scale);
    decode and verify calls (at most 8 queries per sequence)."""
    lib = load_library()
    _check(lib.msa_index_scores_fp8(ctypes.byref(cfg._c()), ctypes.byref(batch._c()),
                                    _need(idx_q, torch.bfloat16, "idx_q"),
                                    _need(idx_k_cache_e4m3, torch.uint8, "idx_k_cache_e4m3"), float(k_scale),
                                    _need(block_scores, torch.float32, "block_scores"), _stream(stream)))


def topk_blocks(cfg: Config, batch: Batch, block_scores, block_idx, stream=None) -> None:
    lib = load_library()
    _check(lib.msa_topk_blocks(ctypes.byref(cfg._c()), ctypes.byref(batch._c()),
                               _need(block_scores, torch.float32, "block_scores"),
                               _need(block_idx, torch.int32, "block_idx"), _stream(stream)))


def index_topk(cfg: Config, batch: Batch, idx_q, idx_k_cache, block_idx, stream=None) -> None:
    """Indexer scores and top-k selection in one pass (the scores are not materialised)."""
    lib = load_library()
    _check(lib.msa_index_topk(ctypes.byref(cfg._c()), ctypes.byref(batch._c()),
                              _need(idx_q, torch.bfloat16, "idx_q"),
                              _need(idx_k_cache, torch.bfloat16, "idx_k_cache"),
                              _need(block_idx, torch.int32, "block_idx"), _stream(stream)))


def set_timing_events(events=None) -> None:
    """Record four torch.cuda.Event (created with enable_timing=True) around the phases of the
    following msa_attn_prefill calls on this thread: schedule, block-major kernel, merge.
    None stops recording."""
    lib = load_library()
    if not events:
        _check(lib.msa_set_timing_events(None, 0))
        return
    for e in events:
        if not e.cuda_event:     # torch creates the CUDA event on its first record
            e.record()
    handles = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib.msa_set_timing_events(handles, 4))


def prefill_workspace_bytes(cfg: Config, batch: Batch) -> int:
    return int(load_library().msa_prefill_workspace_bytes(ctypes.byref(cfg._c()),
                                                          ctypes.byref(batch._c(host_only=True))))


def decode_workspace_bytes(cfg: Config, batch: Batch) -> int:
    return int(load_library().msa_decode_workspace_bytes(ctypes.byref(cfg._c()),
                                                         ctypes.byref(batch._c(host_only=True))))


def _attn(fn, cfg, batch, q, k_cache, v_cache, block_idx, out, lse, workspace, stream):
    ws = _need(workspace, torch.uint8, "workspace") if workspace is not None else 0
    nbytes = workspace.numel() if workspace is not None else 0
    _check(fn(ctypes.byref(cfg._c()), ctypes.byref(batch._c()), _need(q, torch.bfloat16, "q"),
              _need(k_cache, torch.bfloat16, "k_cache"), _need(v_cache, torch.bfloat16, "v_cache"),
              _need(block_idx, torch.int32, "block_idx"), _need(out, torch.bfloat16, "out"),
              _need(lse, torch.float32, "lse"), ws, nbytes, _stream(stream)))


def attn_prefill(cfg: Config, batch: Batch, q, k_cache, v_cache, block_idx, out, lse=None, workspace=None,
                 stream=None) -> None:
    _attn(load_library().msa_attn_prefill, cfg, batch, q, k_cache, v_cache, block_idx, out, lse, workspace, stream)


def attn_decode(cfg: Config, batch: Batch, q, k_cache, v_cache, block_idx, out, lse=None, workspace=None,
                stream=None) -> None:
    _attn(load_library().msa_attn_decode, cfg, batch, q, k_cache, v_cache, block_idx, out, lse, workspace, stream)


def qknorm_rope_insert(cfg: Config, batch: Batch, q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache,
                       rotary_dim: int = 64, rope_theta: float = 10000.0, eps: float = 1e-6, stream=None) -> None:
    """Per-head RMSNorm + partial rotary embedding of q (in place) and of the new keys, whose
    rows go with the new values into their cache page and slot (see include/msa.h)."""
    lib = load_library()
    _check(lib.msa_qknorm_rope_insert(ctypes.byref(cfg._c()), ctypes.byref(batch._c()),
                                      _need(q, torch.bfloat16, "q"), _need(k_new, torch.bfloat16, "k_new"),
                                      _need(v_new, torch.bfloat16, "v_new"), _need(q_norm_w, torch.bfloat16, "q_norm_w"),
                                      _need(k_norm_w, torch.bfloat16, "k_norm_w"),
                                      _need(k_cache, torch.bfloat16, "k_cache"), _need(v_cache, torch.bfloat16, "v_cache"),
                                      int(rotary_dim), float(rope_theta), float(eps), _stream(stream)))


def merge_partials(outs, lses, out, lse=None, stream=None) -> None:
    """Log-sum-exp merge of n partials: outs bf16 [n][..][128], lses fp32 [n][..] -> out, lse.

    The kernel trusts the sizes it is given, so every shape is checked here:
    outs must be [n, *lses.shape[1:], head_dim], out must hold units * head_dim
    elements and lse (when given) units, units = lses[0].numel()."""
    if outs.dim() < 2 or lses.dim() < 1 or int(lses.shape[0]) != int(outs.shape[0]):
        raise MsaError(MSA_ERR_INVALID_ARG, "outs must be [n][..][head_dim] and lses [n][..] with the same n")
    n = int(outs.shape[0])
    units = int(lses[0].numel())
    if tuple(outs.shape) != (n, *lses.shape[1:], int(outs.shape[-1])):
        raise MsaError(MSA_ERR_INVALID_ARG,
                       f"outs has shape {tuple(outs.shape)}, expected {(n, *lses.shape[1:], int(outs.shape[-1]))}")
    if out.numel() != units * int(outs.shape[-1]):
        raise MsaError(MSA_ERR_INVALID_ARG, f"out holds {out.numel()} elements, expected {units * int(outs.shape[-1])}")
    if lse is not None and lse.numel() != units:
        raise MsaError(MSA_ERR_INVALID_ARG, f"lse holds {lse.numel()} elements, expected {units}")
    lib = load_library()
    _check(lib.msa_merge_partials(n, units, int(outs.shape[-1]), _need(outs, torch.bfloat16, "outs"),
                                  _need(lses, torch.float32, "lses"), _need(out, torch.bfloat16, "out"),
                                  _need(lse, torch.float32, "lse"), _stream(stream)))


def attn_decode_noalloc(cfg: Config, batch: Batch, q, k_cache, v_cache, block_idx, out, lse=None,
                        stream=None) -> None:
    """msa_attn_decode without a workspace: for callers that cannot allocate,
    the scratch lives in a fixed 16 MiB device array inside the library (see
    include/msa.h).  Calls that may overlap on the GPU must be serialized."""
    lib = load_library()
    _check(lib.msa_attn_decode_noalloc(ctypes.byref(cfg._c()), ctypes.byref(batch._c()),
                                       _need(q, torch.bfloat16, "q"), _need(k_cache, torch.bfloat16, "k_cache"),
                                       _need(v_cache, torch.bfloat16, "v_cache"),
                                       _need(block_idx, torch.int32, "block_idx"), _need(out, torch.bfloat16, "out"),
                                       _need(lse, torch.float32, "lse"), _stream(stream)))


def device_status(stream=None) -> int:
    """Synchronise, then read and clear the device error word (an MSA_* status)."""
    return int(load_library().msa_get_device_status(_stream(stream)))


def set_wait_limit_ns(ns: int) -> None:
    _check(load_library().msa_set_wait_limit_ns(int(ns)))


def debug_wait_timeout(stream=None) -> None:
    _check(load_library().msa_debug_wait_timeout(_stream(stream)))


def version() -> int:
    return int(load_library().msa_version())
