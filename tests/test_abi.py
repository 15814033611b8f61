"""The C-ABI library: it builds, loads without a GPU, exports every entry
point include/msa.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import block_sparse_long_13_b200 as msa
from block_sparse_long_13_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return msa.load_library()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for need in ("msa_index_scores", "msa_topk_blocks", "msa_attn_prefill", "msa_attn_decode",
                 "msa_prefill_workspace_bytes", "msa_decode_workspace_bytes", "msa_get_device_status",
                 "msa_status_string"):
        assert need in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", msa.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (msa_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    assert set(msa.EXPORTS) == set(declared_functions())


def test_status_strings_and_version(lib):
    assert lib.msa_status_string(0) == b"ok"
    assert lib.msa_status_string(2) == b"unsupported size or layout"
    assert msa.version() == 100


def _cfg(**kw):
    c = msa.Config()
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _batch():
    return msa.Batch.make([0, 128], [256], [[0, 1]], 2, device="cpu")


@pytest.mark.parametrize("bad,status", [
    (dict(head_dim=64), msa.MSA_ERR_UNSUPPORTED),
    (dict(block_size=64), msa.MSA_ERR_UNSUPPORTED),
    (dict(idx_dim=128), msa.MSA_ERR_UNSUPPORTED),
    (dict(topk=0), msa.MSA_ERR_INVALID_ARG),
    (dict(topk=65), msa.MSA_ERR_UNSUPPORTED),
    (dict(num_q_heads=62), msa.MSA_ERR_INVALID_ARG),
    (dict(num_q_heads=32), msa.MSA_ERR_UNSUPPORTED),
    (dict(idx_heads=6), msa.MSA_ERR_INVALID_ARG),
    (dict(idx_heads=40, num_q_heads=64 * 5, num_kv_heads=20), msa.MSA_ERR_UNSUPPORTED),
])
def test_bad_config_rejected_before_launch(lib, bad, status):
    cfg = _cfg(**bad)._c()
    b = _batch()._c(host_only=True)
    p = ctypes.c_void_p(16)  # never dereferenced: the checks fail first
    st = lib.msa_index_scores(ctypes.byref(cfg), ctypes.byref(b), p, p, p, None)
    assert st == status, lib.msa_last_error()
    st = lib.msa_attn_prefill(ctypes.byref(cfg), ctypes.byref(b), p, p, p, p, p, None, p, 1 << 40, None)
    assert st == status
    assert lib.msa_prefill_workspace_bytes(ctypes.byref(cfg), ctypes.byref(b)) == 0


def test_bad_batch_and_pointers_rejected(lib):
    cfg = msa.Config()._c()
    b = _batch()._c(host_only=True)
    p = ctypes.c_void_p(16)
    assert lib.msa_index_scores(ctypes.byref(cfg), ctypes.byref(b), None, p, p, None) == msa.MSA_ERR_INVALID_ARG
    assert b"NULL" in lib.msa_last_error()
    odd = ctypes.c_void_p(18)
    assert lib.msa_index_scores(ctypes.byref(cfg), ctypes.byref(b), odd, p, p, None) == msa.MSA_ERR_INVALID_ARG
    assert b"aligned" in lib.msa_last_error()
    b2 = _batch()._c(host_only=True)
    b2.max_blocks_per_seq = 20000
    assert lib.msa_topk_blocks(ctypes.byref(cfg), ctypes.byref(b2), p, p, None) == msa.MSA_ERR_UNSUPPORTED
    b3 = _batch()._c(host_only=True)
    b3.page_table = None
    assert lib.msa_topk_blocks(ctypes.byref(cfg), ctypes.byref(b3), p, p, None) == msa.MSA_ERR_INVALID_ARG
    # workspace too small
    need = lib.msa_prefill_workspace_bytes(ctypes.byref(cfg), ctypes.byref(b))
    assert need > 0
    st = lib.msa_attn_prefill(ctypes.byref(cfg), ctypes.byref(b), p, p, p, p, p, None, p, need - 1, None)
    assert st == msa.MSA_ERR_INVALID_ARG and b"workspace" in lib.msa_last_error()
    assert lib.msa_set_wait_limit_ns(0) == msa.MSA_ERR_INVALID_ARG


def test_empty_batch_launches_nothing(lib):
    """total_q = 0 (a sequence with no new rows): every compute call checks its arguments and
    returns MSA_OK without launching; on a machine without a GPU any launch would fail."""
    cfg = msa.Config()._c()
    b = msa.Batch.make([0, 0], [300], [list(range(3))], 3, device="cpu")._c(host_only=True)
    p = ctypes.c_void_p(16)
    n = 1 << 20
    assert lib.msa_index_scores(ctypes.byref(cfg), ctypes.byref(b), p, p, p, None) == msa.MSA_OK
    assert lib.msa_topk_blocks(ctypes.byref(cfg), ctypes.byref(b), p, p, None) == msa.MSA_OK
    assert lib.msa_index_topk(ctypes.byref(cfg), ctypes.byref(b), p, p, p, None) == msa.MSA_OK
    assert lib.msa_attn_prefill(ctypes.byref(cfg), ctypes.byref(b), p, p, p, p, p, None, p, n, None) == msa.MSA_OK
    assert lib.msa_attn_decode(ctypes.byref(cfg), ctypes.byref(b), p, p, p, p, p, None, p, n, None) == msa.MSA_OK
    assert lib.msa_qknorm_rope_insert(ctypes.byref(cfg), ctypes.byref(b), *([p] * 7), 64, 10000.0, 1e-6,
                                      None) == msa.MSA_OK


def test_fused_index_topk_checks(lib):
    """The fused call validates like the two calls it replaces and keeps at most 16 blocks per row."""
    b = _batch()._c(host_only=True)
    p = ctypes.c_void_p(16)
    cfg17 = _cfg(topk=17)._c()
    assert lib.msa_index_topk(ctypes.byref(cfg17), ctypes.byref(b), p, p, p, None) == msa.MSA_ERR_UNSUPPORTED
    assert b"16" in lib.msa_last_error()
    cfg = msa.Config()._c()
    assert lib.msa_index_topk(ctypes.byref(cfg), ctypes.byref(b), p, None, p, None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_index_topk(ctypes.byref(cfg), ctypes.byref(b), p, p, ctypes.c_void_p(20), None) == \
        msa.MSA_ERR_INVALID_ARG
    bad = _cfg(head_dim=64)._c()
    assert lib.msa_index_topk(ctypes.byref(bad), ctypes.byref(b), p, p, p, None) == msa.MSA_ERR_UNSUPPORTED


def test_qknorm_rope_insert_checks(lib):
    """Argument checks of the fused norm / rotary / insert call (nothing is launched)."""
    b = _batch()._c(host_only=True)
    p = ctypes.c_void_p(16)
    cfg = msa.Config()._c()
    def call(rd=64, theta=10000.0, eps=1e-6, ptrs=None):
        a = ptrs or [p] * 7
        return lib.msa_qknorm_rope_insert(ctypes.byref(cfg), ctypes.byref(b), *a, rd, theta, eps, None)
    for rd in (0, -8, 60, 136):
        assert call(rd=rd) == msa.MSA_ERR_INVALID_ARG, rd
    assert b"rotary_dim" in lib.msa_last_error()
    assert call(theta=0.0) == msa.MSA_ERR_INVALID_ARG
    assert call(theta=float("inf")) == msa.MSA_ERR_INVALID_ARG
    assert call(eps=-1.0) == msa.MSA_ERR_INVALID_ARG
    assert call(eps=float("nan")) == msa.MSA_ERR_INVALID_ARG
    assert call(ptrs=[p] * 6 + [None]) == msa.MSA_ERR_INVALID_ARG
    assert call(ptrs=[p] * 3 + [ctypes.c_void_p(24)] + [p] * 3) == msa.MSA_ERR_INVALID_ARG
    bad = _cfg(head_dim=64)._c()
    assert lib.msa_qknorm_rope_insert(ctypes.byref(bad), ctypes.byref(b), *([p] * 7), 64, 10000.0, 1e-6, None) == \
        msa.MSA_ERR_UNSUPPORTED


def test_merge_partials_checks(lib):
    p, f = ctypes.c_void_p(16), ctypes.c_void_p(20)
    assert lib.msa_merge_partials(0, 8, 128, p, p, p, None, None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_merge_partials(2, -1, 128, p, p, p, None, None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_merge_partials(2, 8, 64, p, p, p, None, None) == msa.MSA_ERR_UNSUPPORTED
    assert lib.msa_merge_partials(2, 8, 128, None, p, p, None, None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_merge_partials(2, 8, 128, f, p, p, None, None) == msa.MSA_ERR_INVALID_ARG   # outs misaligned
    assert lib.msa_merge_partials(2, 0, 128, p, f, p, f, None) == msa.MSA_OK                  # nothing to merge


def test_timing_events_hook_checks(lib):
    assert lib.msa_set_timing_events(None, 3) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_set_timing_events(None, 4) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_set_timing_events(None, 0) == msa.MSA_OK


def test_workspace_sizes_scale_with_the_batch(lib):
    cfg = msa.Config()
    b1 = msa.Batch.make([0, 16384], [16384], [list(range(128))], 128, device="cpu")
    b2 = msa.Batch.make([0, 32768], [32768], [list(range(256))], 256, device="cpu")
    w1, w2 = msa.prefill_workspace_bytes(cfg, b1), msa.prefill_workspace_bytes(cfg, b2)
    part = 16384 * 16 * 64 * 128 * 2
    assert part < w1 < part * 1.1 and 1.9 < w2 / w1 < 2.1
    d = msa.Batch.make(list(range(65)), [131072] * 64, [list(range(1024))] * 64, 65536, device="cpu")
    wd = msa.decode_workspace_bytes(cfg, d)
    assert 0 < wd < (64 << 20)


def test_binding_refuses_cpu_tensors(lib):
    cfg = msa.Config()
    b = _batch()
    with pytest.raises(msa.MsaError):
        msa.topk_blocks(cfg, b, torch.zeros(128, 4, 2), torch.zeros(128, 4, 16, dtype=torch.int32))
