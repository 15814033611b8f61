"""Benchmark of the MSA hot path on B200: tokens/s and roofline fractions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole hot path over one batch of synthetic inputs:
the default workload `msa_128k_1m` is a 131,072-token chunked prefill (8 chunks
of 16,384 queries: indexer -> top-k -> block-major attention) followed by one
decode step of 64 sequences at 131,072 tokens and one of 8 sequences at
1,048,576 tokens (indexer -> top-k -> split-K attention), all in one layer,
M3 head configuration (64 query / 4 KV heads, head_dim 128, indexer 8 x 64,
k = 16).  `value` counts every query token of the step.

With torchrun (N > 1) every rank runs its own replica (weak scaling: the
units are independent sequences), timed between barriers; the slowest rank's
time sets `value`.  `--impl reference` times the CPU oracle on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import configs, gen  # noqa: E402

METRIC = "MSA tokens/s (prefill & decode) at 128K/1M ctx; % of HBM/tensor roofline"
WORKLOADS = ("msa_128k_1m", "chunked_prefill_128k", "prefill_32k", "decode_128k", "decode_1m", "verify_ragged",
             "tiny_prefill_2k", "prefill_8k", "prefill_128k_last_chunk")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured", **SPEC}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback", **SPEC}


# nominal B200 figures the per-workload fractions are also stated against: 8 TB/s of HBM (the
# decode target's denominator) and 2.25 PFLOP/s of dense bf16
SPEC = {"hbm_gbs_spec": 8000.0, "bf16_tflops_spec": 2250.0}


def recorded_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu record (profiles/traffic.json), or
    None when there is none or the kernel's sources changed since it was taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    h = hashlib.sha256()
    for rel in rec["sources"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return rec["dram_bytes_per_launch"] if h.hexdigest() == rec["sources_sha256"] else None


# ------------------------------------------------------------------ workload parts

class Part:
    """One batch through the three calls (indexer, top-k, attention)."""

    def __init__(self, name, wl, caches, kind, out_rows=None, fused=False):
        import block_sparse_long_13_b200 as msa
        self.msa = msa
        self.name, self.wl, self.kind = name, wl, kind
        dev = "cuda"
        self.cfg = msa.Config(num_q_heads=wl.num_q_heads, num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim,
                              idx_heads=wl.idx_heads, idx_dim=wl.idx_dim, block_size=wl.block_size,
                              topk=wl.topk)
        self.batch = msa.Batch.make(wl.q_start, wl.ctx_len, wl.page_table, wl.num_pages, device=dev)
        self.caches = caches
        self.q = gen.query_rows(wl, gen.TID_Q, device=dev)
        self.idx_q = gen.query_rows(wl, gen.TID_IDX_Q, device=dev)
        T, G, nb = wl.total_q, wl.num_kv_heads, wl.max_blocks
        self.sel = torch.empty((T, G, wl.topk), dtype=torch.int32, device=dev)
        self.out = torch.empty_like(self.q) if out_rows is None else out_rows
        self.lse = torch.empty((T, wl.num_q_heads), dtype=torch.float32, device=dev)
        wsb = (msa.prefill_workspace_bytes if kind == "prefill" else msa.decode_workspace_bytes)(self.cfg, self.batch)
        self.ws_bytes = wsb
        self.ws = None
        # prefill: indexer and top-k in one call (msa_index_topk) when asked
        self.fused = fused and kind == "prefill" and wl.topk <= 16
        self.scores = None if self.fused else torch.empty((T, G, nb), dtype=torch.float32, device=dev)
        # kernels of ours per run: indexer (+ top-k), then attention: prefill = schedule (4 kernels),
        # block-major attention, merge; decode = work-item plan + attention
        self.launches = (1 if self.fused else 2) + (6 if kind == "prefill" else 2)
        self.pos = wl.positions()

    def run(self, ws, ev=None, stream=None, stop_after="attn"):
        # NVTX ranges name each call of the part (part/index, part/topk, part/attn) for a profiler's timeline
        m = self.msa
        nvtx = torch.cuda.nvtx
        if ev is not None:
            ev[0].record(stream)
        nvtx.range_push(f"{self.name}/index")
        if self.fused:
            m.index_topk(self.cfg, self.batch, self.idx_q, self.caches["idx_k"], self.sel)
        else:
            m.index_scores(self.cfg, self.batch, self.idx_q, self.caches["idx_k"], self.scores)
        nvtx.range_pop()
        if ev is not None:
            ev[1].record(stream)
        if stop_after != "index" and not self.fused:
            nvtx.range_push(f"{self.name}/topk")
            m.topk_blocks(self.cfg, self.batch, self.scores, self.sel)
            nvtx.range_pop()
        if ev is not None:
            ev[2].record(stream)
        if stop_after == "attn":
            fn = m.attn_prefill if self.kind == "prefill" else m.attn_decode
            phases = ev is not None and self.kind == "prefill"
            if phases:
                m.set_timing_events(ev[4:8])
            nvtx.range_push(f"{self.name}/attn")
            fn(self.cfg, self.batch, self.q, self.caches["k"], self.caches["v"], self.sel, self.out, self.lse,
               ws[:self.ws_bytes])
            nvtx.range_pop()
            if phases:
                m.set_timing_events(None)
        if ev is not None:
            ev[3].record(stream)

    # ---- algorithmic work (for the roofline), from the shapes and the selection
    def index_work(self):
        wl = self.wl
        vis = (self.pos + 1).double()
        if self.kind == "prefill":
            return {"flops": float(vis.sum()) * 2 * wl.idx_dim * wl.idx_heads}
        ctx = torch.tensor(wl.ctx_len, dtype=torch.float64)
        return {"bytes": float(ctx.sum()) * wl.idx_heads * wl.idx_dim * 2}

    def attn_work(self):
        wl = self.wl
        sel = self.sel.long().cpu()
        pos = self.pos.view(-1, 1, 1)
        vis = torch.clamp(pos - sel * wl.block_size + 1, 0, wl.block_size)
        vis = torch.where(sel >= 0, vis, torch.zeros_like(vis))
        keys = float(vis.sum())  # per (row, group)
        G = wl.num_q_heads // wl.num_kv_heads
        flops = keys * G * 4 * wl.head_dim
        bytes_ = keys * 2 * wl.head_dim * 2 + self.q.numel() * 2 * 2
        return {"flops": flops, "bytes": bytes_}

    def merge_work(self):
        """Partial O (bf16) and lse of every valid slot read once; out and lse written."""
        wl = self.wl
        slots = float((self.sel >= 0).sum())
        G = wl.num_q_heads // wl.num_kv_heads
        return {"bytes": slots * G * (wl.head_dim * 2 + 4) + wl.total_q * wl.num_q_heads * (wl.head_dim * 2 + 4)}

    def topk_work(self):
        cur = (self.pos // self.wl.block_size).double()
        return {"bytes": float(cur.sum()) * self.wl.num_kv_heads * 4 + self.sel.numel() * 4}


def build_parts(name, batch=None, fused=False):
    """Device inputs of a workload: list of Part (in order).  `batch` shrinks
    a decode workload (fewer sequences, same shapes) for profiling runs;
    `fused` selects msa_index_topk for prefill (else the two calls)."""
    parts = []
    if name in ("msa_128k_1m", "chunked_prefill_128k", "prefill_128k_last_chunk"):
        chunks = configs.chunked_prefill_128k()
        full = chunks[-1]
        caches = {"k": gen.paged_cache(full, gen.TID_K, device="cuda"),
                  "v": gen.paged_cache(full, gen.TID_V, device="cuda"),
                  "idx_k": gen.paged_cache(full, gen.TID_IDX_K, device="cuda")}
        which = [7] if name == "prefill_128k_last_chunk" else list(range(8))
        out_all = torch.empty((len(which) * 16384, 64, 128), dtype=torch.bfloat16, device="cuda")
        for n, c in enumerate(which):
            parts.append(Part(f"prefill128k/c{c}", chunks[c], caches, "prefill",
                              out_all[n * 16384:(n + 1) * 16384], fused=fused))
    if name in ("msa_128k_1m", "decode_128k", "decode_1m", "verify_ragged"):
        for dn in (("decode_128k", "decode_1m") if name == "msa_128k_1m" else (name,)):
            wl = configs.ALL[dn](batch=batch) if batch else configs.ALL[dn]()
            caches = {"k": gen.paged_cache(wl, gen.TID_K, device="cuda"),
                      "v": gen.paged_cache(wl, gen.TID_V, device="cuda"),
                      "idx_k": gen.paged_cache(wl, gen.TID_IDX_K, device="cuda")}
            parts.append(Part(dn, wl, caches, "decode"))
    if name in ("prefill_32k", "tiny_prefill_2k", "prefill_8k"):
        wl = configs.prefill_8k() if name == "prefill_8k" else configs.ALL[name]()
        caches = {"k": gen.paged_cache(wl, gen.TID_K, device="cuda"),
                  "v": gen.paged_cache(wl, gen.TID_V, device="cuda"),
                  "idx_k": gen.paged_cache(wl, gen.TID_IDX_K, device="cuda")}
        parts.append(Part(name, wl, caches, "prefill", fused=fused))
    return parts


# ------------------------------------------------------------------ per-call times and per-workload fractions

def call_stats(parts, evs, steps, stop_after="attn"):
    """Per part: device time of each call (mean over the timed steps, CUDA events on the
    launching stream) and its algorithmic work."""
    calls = {}
    for i, p in enumerate(parts):
        t_idx = statistics.mean(evs[k][i][0].elapsed_time(evs[k][i][1]) for k in range(steps))
        t_top = statistics.mean(evs[k][i][1].elapsed_time(evs[k][i][2]) for k in range(steps))
        t_att = statistics.mean(evs[k][i][2].elapsed_time(evs[k][i][3]) for k in range(steps))
        phase = None
        if p.kind == "prefill" and stop_after == "attn":
            phase = {nm: statistics.mean(evs[k][i][4 + j].elapsed_time(evs[k][i][5 + j]) for k in range(steps))
                     for j, nm in enumerate(("schedule_ms", "kernel_ms", "merge_ms"))}
        calls[p.name] = {"index_ms": t_idx, "topk_ms": t_top, "attn_ms": t_att, "attn_phases": phase,
                         "index": p.index_work(), "attn": p.attn_work(), "topk": p.topk_work(), "kind": p.kind,
                         "merge": p.merge_work() if p.kind == "prefill" else None,
                         "tokens": p.wl.total_q, "fused": p.fused}
    return calls


def workload_summary(calls, pk):
    """Fractions of the roofline per workload, as the decode and prefill targets state them:
    prefill = (indexer causal FLOPs + attention FLOPs) / (indexer + top-k + attention time) over
    the dense bf16 peak (measured burst and nominal 2.25 PF; attention-only and indexer-only
    beside); decode = (indexer-key bytes + visible selected K/V + q/out) / (indexer + top-k +
    attention time) over 8 TB/s and over the measured copy bandwidth."""
    cs = list(calls.values())
    ms = sum(c["index_ms"] + c["topk_ms"] + c["attn_ms"] for c in cs)
    tokens = sum(c["tokens"] for c in cs)
    r = {"tokens": tokens, "ms": ms, "tokens_per_s": tokens / (ms / 1e3)}
    if cs[0]["kind"] == "prefill":
        fi = sum(c["index"]["flops"] for c in cs)
        fa = sum(c["attn"]["flops"] for c in cs)
        tf = (fi + fa) / ms / 1e9
        ti = sum(c["index_ms"] for c in cs)
        ta = sum(c["attn_ms"] for c in cs)
        r.update(index_tflop=fi / 1e12, attn_tflop=fa / 1e12, tflops=tf,
                 frac_dense_measured=tf / pk["bf16_tflops"], frac_dense_spec=tf / pk["bf16_tflops_spec"],
                 attn_only_frac_measured=(fa / ta / 1e9) / pk["bf16_tflops"] if ta > 0 else None,
                 index_only_frac_measured=(fi / ti / 1e9) / pk["bf16_tflops"] if ti > 0 else None)
    else:
        b = sum(c["index"]["bytes"] + c["attn"]["bytes"] for c in cs)
        gbs = b / ms / 1e6
        r.update(gbytes=b / 1e9, gbs=gbs, frac_hbm_8tbs=gbs / pk["hbm_gbs_spec"],
                 frac_hbm_measured=gbs / pk["hbm_gbs"])
    return r


def time_workload(name, workspace, steps=3, warmup=2):
    """A further workload timed on its own after the step (same calls, same timing method);
    returns its summary, or an error note."""
    parts = build_parts(name)
    need = max(p.ws_bytes for p in parts)
    ws = workspace if workspace.numel() >= need else torch.empty(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        for p in parts:
            p.run(ws, None, stream)
    torch.cuda.synchronize()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in parts] for _ in range(steps)]
    for k in range(steps):
        for i, p in enumerate(parts):
            p.run(ws, evs[k][i], stream)
    torch.cuda.synchronize()
    return parts, call_stats(parts, evs, steps)


# ------------------------------------------------------------------ next rows, timed on their own

def time_next_rows(parts, pk):
    """The fused QK-norm + partial-RoPE + KV-insert call (the step just before the path) on the
    workload's first prefill chunk, timed by itself: it is not part of the step, whose inputs are
    already normed, rotated and inserted.  Algorithmic bytes per row: q read and written in place,
    the new k and v rows read and written to the cache."""
    import block_sparse_long_13_b200 as msa
    p = next((x for x in parts if x.kind == "prefill"), None)
    if p is None:
        return None
    wl = p.wl
    T, hq, hkv, d = wl.total_q, wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    q = p.q.clone()
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    kn = torch.randn((T, hkv, d), device="cuda", generator=g).to(torch.bfloat16)
    vn = torch.randn((T, hkv, d), device="cuda", generator=g).to(torch.bfloat16)
    w = torch.ones(d, device="cuda", dtype=torch.bfloat16)
    kc, vc = p.caches["k"].clone(), p.caches["v"].clone()

    def call():
        msa.qknorm_rope_insert(p.cfg, p.batch, q, kn, vn, w, w, kc, vc)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 20
    e0.record()
    for _ in range(n):
        call()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    nbytes = T * 2 * (hq + 2 * hkv) * d * 2
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"qk_rope_insert_kernel": {"part": p.name, "rows": T, "ms_per_call": ms, "bytes_per_call": nbytes,
                                      "gbs": gbs, "frac": gbs / pk["hbm_gbs"], "status": int(msa.device_status())}}


def time_fp8_indexer(parts, pk):
    """The streaming indexer over an e4m3 copy of a decode workload's indexer keys (the FP8 cache
    path), timed by itself: the codes are written once with one scale (torch, untimed), then 20
    calls after 3 warm-ups, CUDA events.  Algorithmic bytes: every visible key's 64 codes per
    indexer head (half the bf16 bytes)."""
    import block_sparse_long_13_b200 as msa
    p = next((x for x in parts if x.name == "decode_128k"), None) or next(
        (x for x in parts if x.kind == "decode"), None)
    if p is None:
        return None
    k = p.caches["idx_k"]
    s = float(k.float().abs().max()) / 448.0
    codes = torch.empty(k.shape, dtype=torch.uint8, device="cuda")
    for i in range(0, k.shape[0], 4096):       # written in slices to bound the temporaries
        codes[i:i + 4096] = torch.clamp(k[i:i + 4096].float() / s, -448.0, 448.0).to(
            torch.float8_e4m3fn).view(torch.uint8)
    scores = torch.empty_like(p.scores)

    def call():
        msa.index_scores_fp8(p.cfg, p.batch, p.idx_q, codes, s, scores)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 20
    e0.record()
    for _ in range(n):
        call()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    wl = p.wl
    nbytes = float(sum(wl.ctx_len)) * wl.idx_heads * wl.idx_dim
    gbs = nbytes / (ms * 1e-3) / 1e9
    del codes
    return {"part": p.name, "ms_per_call": ms, "bytes_per_call": nbytes, "gbs": gbs,
            "frac": gbs / pk["hbm_gbs"], "frac_8tbs": gbs / pk["hbm_gbs_spec"], "status": int(msa.device_status())}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        load = [x for x in sm if mx and x > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ the oracle (CPU baseline / reference arm)

def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class _Blocks:
    """Token-order view of one sequence of a paged device cache: slices of whole blocks (or parts
    of one) are fetched page by page as float32 host arrays (bf16 values widened exactly)."""

    def __init__(self, cache, pages, bs=128):
        self.cache, self.pages, self.bs = cache, [int(x) for x in pages], bs

    def __getitem__(self, sl):
        b = sl.start // self.bs
        x = self.cache[self.pages[b]].permute(1, 0, 2).float().cpu().numpy()   # [bs][H][D]
        return x[sl.start - b * self.bs:sl.stop - b * self.bs]


class _HostBlocks:
    """Blocks already fetched to host arrays, sliced like the sequence they come from."""

    def __init__(self, blocks, bs):
        self.blocks, self.bs = blocks, bs

    def __getitem__(self, sl):
        b = sl.start // self.bs
        x = self.blocks[b]
        return x[sl.start - b * self.bs:sl.stop - b * self.bs]


class _GenTokens:
    """Token-order view of one sequence straight from the seeded generator: a slice generates only
    its own tokens (the attention reads just the selected blocks; the whole 1M-token K and V of a
    sequence would be 4 GB of float32 per sampled sequence)."""

    def __init__(self, wl, tid, s, dev):
        self.wl, self.tid, self.s, self.dev, self.ctx = wl, tid, s, dev, wl.ctx_len[s]

    def __getitem__(self, sl):
        idx = torch.arange(sl.start, min(sl.stop, self.ctx))
        return gen.token_tensor(self.wl, self.tid, self.s, idx, device=self.dev).float().cpu().numpy()


def _seq_tokens(wl, tid, s, cache=None, dev="cpu"):
    """float32 [ctx][H][D] of one sequence in token order: from the device cache when given
    (pages gathered), else from the seeded generator."""
    ctx = wl.ctx_len[s]
    nb = (ctx + wl.block_size - 1) // wl.block_size
    if cache is not None:
        pages = wl.page_table[s, :nb].long().to(cache.device)
        t = cache.index_select(0, pages)                      # [nb][H][bs][D]
        return t.permute(0, 2, 1, 3).reshape(nb * wl.block_size, t.shape[1], t.shape[3])[:ctx].float().cpu().numpy()
    return gen.token_tensor(wl, tid, s, torch.arange(ctx), device=dev).float().cpu().numpy()


class OracleLeg:
    """The plain C++ oracle (indexer over every visible block, top-k, sparse attention; double
    arithmetic, std::thread over independent outputs) timed on the host cores on bounded samples
    of the step's workloads; the step's oracle time is extrapolated from each workload's time per
    query row.  Inputs come from the device caches of the timed step when there are any, else
    from the seeded generator (on the GPU when there is one); preparing them is not timed."""

    GEN_POOL = 4   # decode sequences sampled per workload when inputs come from the generator

    def __init__(self, parts=None):
        from oracle import cpp as C
        self.C = C
        C.build()
        self.parts = parts or []
        self.dev = "cuda" if torch.cuda.is_available() else "cpu"
        self.chunks = configs.chunked_prefill_128k()
        self._prefill_keys = None
        self._decode = {}
        self.rng = np.random.default_rng(0)
        self.report = {"rows": 0, "near_ties": 0, "selection_mismatches": 0, "attn_rows_compared": 0,
                       "attn_max_abs": 0.0, "attn_sum_abs": 0.0, "attn_elems": 0}

    def _part(self, name):
        return next((p for p in self.parts if p.name == name), None)

    # ---- prefill: rows drawn uniformly from the 131,072-token chunked prefill
    def prefill_rows(self, n):
        full = self.chunks[-1]
        if self._prefill_keys is None:
            p0 = self._part("prefill128k/c0")
            cc = p0.caches if p0 is not None else None
            self._prefill_keys = {
                "idx_k": _seq_tokens(full, gen.TID_IDX_K, 0, cc["idx_k"] if cc else None, self.dev),
                "k": _seq_tokens(full, gen.TID_K, 0, cc["k"] if cc else None, self.dev),
                "v": _seq_tokens(full, gen.TID_V, 0, cc["v"] if cc else None, self.dev)}
        gpos = np.sort(self.rng.integers(0, full.ctx_len[0], size=n))
        q, iq = [], []
        for g in gpos:
            c, r = int(g) // 16384, int(g) % 16384
            wl = self.chunks[c]
            q.append(gen.token_tensor(wl, gen.TID_Q, 0, torch.tensor([int(g)]), device=self.dev).float().cpu())
            iq.append(gen.token_tensor(wl, gen.TID_IDX_Q, 0, torch.tensor([int(g)]), device=self.dev).float().cpu())
        q = torch.cat(q).numpy()
        iq = torch.cat(iq).numpy()
        hk = self._prefill_keys
        t0 = time.perf_counter()
        s64, sel, out, lse = self.C.msa_rows(q, iq, hk["k"], hk["v"], hk["idx_k"], gpos, full.num_kv_heads,
                                             full.block_size, full.topk, full.max_blocks)
        dt = time.perf_counter() - t0
        if self.parts:
            for i, g in enumerate(gpos):
                p = self._part(f"prefill128k/c{int(g) // 16384}")
                if p is not None:
                    self._compare(p, int(g) % 16384, s64[i:i + 1], sel[i:i + 1], out[i:i + 1], np.array([g]))
        return dt

    # ---- decode: whole sequences of the decode workloads (one query row each)
    def decode_seq(self, name, s):
        wl = configs.ALL[name]()
        p = self._part(name)
        cc = p.caches if p is not None else None
        key = (name, s)
        if key not in self._decode:
            if len(self._decode) >= (2 * self.GEN_POOL if not self.parts else 3):
                self._decode.clear()
            self._decode[key] = _seq_tokens(wl, gen.TID_IDX_K, s, cc["idx_k"] if cc else None, self.dev)
        ik = self._decode[key]
        nb = (wl.ctx_len[s] + wl.block_size - 1) // wl.block_size
        if cc is not None:
            k, v = _Blocks(cc["k"], wl.page_table[s, :nb]), _Blocks(cc["v"], wl.page_table[s, :nb])
        else:
            k, v = _GenTokens(wl, gen.TID_K, s, self.dev), _GenTokens(wl, gen.TID_V, s, self.dev)
        rows = list(range(wl.q_start[s], wl.q_start[s + 1]))
        pos = wl.positions()[rows].numpy()
        q = gen.query_rows(wl, gen.TID_Q, device=self.dev)[rows].float().cpu().numpy() if p is None else \
            p.q[rows].float().cpu().numpy()
        iq = gen.query_rows(wl, gen.TID_IDX_Q, device=self.dev)[rows].float().cpu().numpy() if p is None else \
            p.idx_q[rows].float().cpu().numpy()
        # timed: the oracle's three steps; not timed: fetching the selected K / V blocks (device cache
        # or generator) into host arrays between the selection and the attention
        t0 = time.perf_counter()
        s64 = self.C.block_scores(iq, ik, pos, wl.num_kv_heads, wl.block_size, wl.max_blocks)
        sel = self.C.select_blocks(s64.astype(np.float32), pos, wl.topk, wl.block_size)
        t1 = time.perf_counter()
        bs = wl.block_size
        blocks = sorted(set(int(b) for b in sel[sel >= 0].reshape(-1)))
        kh = _HostBlocks({b: k[b * bs:(b + 1) * bs] for b in blocks}, bs)
        vh = _HostBlocks({b: v[b * bs:(b + 1) * bs] for b in blocks}, bs)
        t2 = time.perf_counter()
        out, lse = self.C.sparse_attention(q, kh, vh, pos, sel, bs)
        dt = (t1 - t0) + (time.perf_counter() - t2)
        if p is not None:
            for i, r in enumerate(rows):
                self._compare(p, r, s64[i:i + 1], sel[i:i + 1], out[i:i + 1], pos[i:i + 1])
        return dt, len(rows)

    def _compare(self, p, r, s64, sel, out, pos):
        """Parity of the step's own results on a sampled row: selection (exact outside near-ties),
        and the attention output where the selections agree."""
        near, _, _ = self.C.boundary_gap(s64, pos, p.wl.topk, p.wl.block_size)
        got_sel = p.sel[r].cpu().numpy()
        rep = self.report
        rep["rows"] += 1
        rep["near_ties"] += int(near.sum())
        same = np.array_equal(got_sel, sel[0])
        if not same:
            rep["selection_mismatches"] += 1
            return
        err = np.abs(p.out[r].float().cpu().numpy().astype(np.float64) - out[0])
        rep["attn_rows_compared"] += 1
        rep["attn_max_abs"] = max(rep["attn_max_abs"], float(err.max()))
        rep["attn_sum_abs"] += float(err.sum())
        rep["attn_elems"] += int(err.size)

    def run(self, seconds=20.0):
        """Oracle time per query row of each workload of the default step, then the extrapolated
        step.  Budget: about half the seconds on prefill rows, the rest on decode sequences."""
        per_row, used, n_rows = {}, {}, {}
        # prefill rows in batches until the budget is spent
        t_pre, n_pre, batch = 0.0, 0, 16
        while t_pre < 0.5 * seconds:
            t_pre += self.prefill_rows(batch)
            n_pre += batch
            batch = min(256, batch * 2)
        per_row["prefill_128k"] = t_pre / n_pre
        used["prefill_128k"], n_rows["prefill_128k"] = t_pre, n_pre
        for name, share in (("decode_128k", 0.3), ("decode_1m", 0.2)):
            wl_n = configs.ALL[name]().num_seqs
            # without the step's device caches (the reference arm) every sampled sequence's indexer keys
            # are generated again: a fixed few sequences, kept between steps (all have the same length)
            pool = wl_n if self.parts else min(self.GEN_POOL, wl_n)
            t, n, s = 0.0, 0, 0
            while (t < share * seconds or n == 0) and s < pool:
                dt, k = self.decode_seq(name, int(self.rng.integers(0, pool)))
                t, n, s = t + dt, n + k, s + 1
            per_row[name] = t / n
            used[name], n_rows[name] = t, n
        tokens = {"prefill_128k": 131072, "decode_128k": 64, "decode_1m": 8}
        step_s = sum(tokens[k] * per_row[k] for k in tokens)
        rep = dict(self.report)
        if rep["attn_elems"]:
            rep["attn_mean_abs"] = rep["attn_sum_abs"] / rep["attn_elems"]
        rep.pop("attn_sum_abs")
        rep.pop("attn_elems")
        sample = ("C++ oracle (double; std::thread over independent outputs) on "
                  + ", ".join(f"{n_rows[k]} {k} rows ({used[k]:.1f} s)" for k in per_row)
                  + "; the step's time extrapolated from each workload's time per row"
                  + " (131072 prefill + 64 + 8 decode rows)")
        return {"value": sum(tokens.values()) / step_s, "unit": "tokens/s", "cores": int(self.C.threads()),
                "cpu_model": cpu_model(), "kind": "oracle", "sample": sample,
                "seconds_per_row": per_row, "extrapolated_step_s": step_s,
                "parity": rep if self.parts else None}


# ------------------------------------------------------------------ main

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        rank = int(os.environ["RANK"])
        local = int(os.environ.get("LOCAL_RANK", rank))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        return rank, ws, local
    return 0, 1, 0


def max_over_ranks(x, ws, device="cuda"):
    """Slowest rank's value (timings are taken per rank on its device)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, ws, ms_slowest):
    """Whole-job tokens/s: every rank processes its own replica (weak scaling)."""
    return tokens_per_rank * ws / (ms_slowest / 1e3)


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def run_reference(args, rank, ws):
    """The oracle as it stands, timed on the host cores: each step a bounded sample of the step's
    workloads (no GPU kernel of this repository runs)."""
    if rank != 0:
        return
    leg = OracleLeg()
    for _ in range(args.warmup):
        leg.run(seconds=1.0)
    steps = [leg.run(seconds=max(4.0, 60.0 / max(1, args.steps))) for _ in range(args.steps)]
    val = statistics.median(s["value"] for s in steps)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": steps[-1]["extrapolated_step_s"] * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded generator)",
            "config": {"workload": args.workload, "sample": steps[-1]["sample"]},
            "cpu_baseline": dict(steps[-1], value=val),
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="msa_128k_1m", choices=WORKLOADS)
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--batch", type=int, default=None, help="sequences of a decode workload (profiling)")
    ap.add_argument("--stop-after", default="attn", choices=("index", "topk", "attn"),
                    help="profiling: run the step only up to this call")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the 32K prefill and ragged verify timings")
    ap.add_argument("--fused-prefill", action="store_true",
                    help="prefill indexer and top-k in one call (msa_index_topk) instead of the two calls")
    args = ap.parse_args()
    rank, ws, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, rank, ws)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    import block_sparse_long_13_b200 as msa
    msa.load_library()  # fails loudly when the CUDA library is missing

    parts = build_parts(args.workload, args.batch, fused=args.fused_prefill)
    stream = torch.cuda.current_stream()
    ws_bytes = max(p.ws_bytes for p in parts) if args.stop_after == "attn" else 0
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    tokens = sum(p.wl.total_q for p in parts)
    nev = len(parts)

    def step(evs=None):
        for i, p in enumerate(parts):
            p.run(workspace, None if evs is None else evs[i], stream, args.stop_after)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = msa.device_status()
    if st != msa.MSA_OK:
        raise SystemExit(f"device status {st} after warm-up")

    # per step and part: 4 call boundaries, then (prefill) the 4 phase events of msa_attn_prefill
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(nev)]
           for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(args.steps):
        step(evs[k])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = max_over_ranks(ms, ws)
    value = job_throughput(tokens, ws, ms_max)

    # per-call device times (average over the timed steps) and algorithmic work
    calls = call_stats(parts, evs, args.steps, args.stop_after)
    pk = peaks()
    # per kernel: device time per step (CUDA events on the launching stream) and algorithmic work
    kern = {}

    def addk(name, ms, launches, flops=0.0, bytes_=0.0):
        k = kern.setdefault(name, {"ms": 0.0, "launches": 0, "flops": 0.0, "bytes": 0.0})
        k["ms"] += ms
        k["launches"] += launches
        k["flops"] += flops
        k["bytes"] += bytes_

    decode_attn_parts = {}
    name_of = {id(c): n for n, c in calls.items()}
    for c in calls.values():
        if c["kind"] == "prefill":
            if c["fused"]:
                addk("index_prefill_kernel (fused top-k)", c["index_ms"], 1, flops=c["index"]["flops"])
            else:
                addk("index_prefill_kernel", c["index_ms"], 1, flops=c["index"]["flops"])
                addk("topk kernel (prefill)", c["topk_ms"], 1, bytes_=c["topk"]["bytes"])
            ph = c["attn_phases"]
            if ph is not None:
                addk("schedule (4 kernels)", ph["schedule_ms"], 4)
                addk("attn_prefill_kernel", ph["kernel_ms"], 1, flops=c["attn"]["flops"])
                addk("attn_merge_kernel", ph["merge_ms"], 1, bytes_=c["merge"]["bytes"])
        else:
            addk("index_decode_kernel", c["index_ms"], 1, bytes_=c["index"]["bytes"])
            addk("topk kernel (decode)", c["topk_ms"], 1, bytes_=c["topk"]["bytes"])
            addk("attn_decode_kernel", c["attn_ms"], 1, bytes_=c["attn"]["bytes"])
            if c["attn_ms"] > 0:   # each decode workload's attention on its own (the 8 x 1M one is a few us)
                gbs = c["attn"]["bytes"] / c["attn_ms"] / 1e6
                decode_attn_parts[name_of[id(c)]] = {"ms": c["attn_ms"], "gbs": gbs}
    # every kernel is timed inside a step of tens of ms, far shorter than the seconds-long loop the
    # sustained figure comes from: the burst tensor peak is the denominator
    tensor_peak, tensor_src = pk["bf16_tflops"], pk["source"] + " burst bf16 (cuBLAS)"
    fractions = {}
    for name, k in kern.items():
        if k["ms"] <= 0:
            continue
        if k["flops"] > 0:
            ach = k["flops"] / k["ms"] / 1e9
            fractions[name] = {"ms_per_step": k["ms"], "launches_per_step": k["launches"], "tflops": ach,
                               "frac": ach / tensor_peak}
        elif k["bytes"] > 0:
            ach = k["bytes"] / k["ms"] / 1e6
            fractions[name] = {"ms_per_step": k["ms"], "launches_per_step": k["launches"], "gbs": ach,
                               "frac": ach / pk["hbm_gbs"]}
        else:
            fractions[name] = {"ms_per_step": k["ms"], "launches_per_step": k["launches"]}
    if "attn_decode_kernel" in fractions and decode_attn_parts:
        fractions["attn_decode_kernel"]["per_part"] = {
            n: dict(v, frac=v["gbs"] / pk["hbm_gbs"]) for n, v in decode_attn_parts.items()}
    dom_name, dom = max(((n, k) for n, k in kern.items() if k["flops"] > 0 or k["bytes"] > 0),
                        key=lambda nk: nk[1]["ms"])
    launch_ms = dom["ms"] / dom["launches"]
    traffic = recorded_traffic(dom_name)
    if dom["flops"] > 0:
        ach = dom["flops"] / dom["launches"] / (launch_ms / 1e3) / 1e12
        roof = {"kernel": dom_name, "bound": "tensor", "achieved": ach, "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": ach / tensor_peak, "traffic": traffic, "peak_source": tensor_src, "launch_ms": launch_ms,
                "flops_per_launch": dom["flops"] / dom["launches"]}
    else:
        ach = dom["bytes"] / dom["launches"] / (launch_ms / 1e3) / 1e9
        roof = {"kernel": dom_name, "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": ach / pk["hbm_gbs"], "traffic": traffic, "peak_source": pk["source"] + " copy",
                "launch_ms": launch_ms, "bytes_per_launch": dom["bytes"] / dom["launches"]}
    parts_summary = {}
    pre = {n: c for n, c in calls.items() if c["kind"] == "prefill"}
    if pre:
        parts_summary["prefill"] = workload_summary(pre, pk)
    for name, c in calls.items():
        if c["kind"] == "decode":
            parts_summary[name] = workload_summary({name: c}, pk)

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        host_in, host_out = [], []
        for p in parts:
            hin = {"q": p.q.cpu().pin_memory(), "idx_q": p.idx_q.cpu().pin_memory()}
            host_in.append(hin)
            host_out.append(torch.empty(p.out.shape, dtype=p.out.dtype).pin_memory())
        new_kv = None
        if parts[0].kind == "prefill":
            # the prefill's own keys / values / indexer keys are inputs of the step too
            cch = parts[0].caches
            new_kv = {k: cch[k].cpu().pin_memory() for k in ("k", "v", "idx_k")}
        h2d = sum(t.numel() * t.element_size() for h in host_in for t in h.values())
        if new_kv is not None:
            h2d += sum(t.numel() * t.element_size() for t in new_kv.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out)

        # Copies in run on s_in, the calls on the compute stream, copies out on s_out, chained per part
        # by events: part i's inputs arrive while part i-1 computes and its output leaves while part
        # i+1 computes (a chunked prefill pipelines this way).  A device buffer is rewritten only after
        # its previous use has finished: inputs after the previous step's call on them, outputs after
        # the previous step's copy out, each of the prefill's two alternating cache copies after the last
        # prefill call that read it.
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        n = len(parts)
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_done = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        last_prefill = max((i for i, p in enumerate(parts) if p.kind == "prefill"), default=-1)
        # the prefill's own caches alternate between two device copies from step to step, so the next
        # step's copy in does not wait for this step's last prefill call (a serving loop double-buffers
        # its staging the same way)
        cache_sets, cache_free = None, None
        if new_kv is not None:
            cache_sets = [parts[0].caches, {k: torch.empty_like(v) for k, v in parts[0].caches.items()}]
            cache_free = [torch.cuda.Event(), torch.cuda.Event()]
        started = [0]

        def e2e_step():
            j = started[0]
            again = j > 0
            started[0] = j + 1
            with torch.cuda.stream(s_in):
                if new_kv is not None:
                    cs = cache_sets[j % 2]
                    if j >= 2:
                        s_in.wait_event(cache_free[j % 2])      # its last reader, two steps back
                    for key, t in new_kv.items():
                        cs[key].copy_(t, non_blocking=True)
                    for p in parts:
                        if p.kind == "prefill":
                            p.caches = cs
                for i, (p, hin) in enumerate(zip(parts, host_in)):
                    if again:
                        s_in.wait_event(ev_done[i])
                    p.q.copy_(hin["q"], non_blocking=True)
                    p.idx_q.copy_(hin["idx_q"], non_blocking=True)
                    ev_in[i].record(s_in)
            for i, p in enumerate(parts):
                stream.wait_event(ev_in[i])
                if again:
                    stream.wait_event(ev_out[i])
                p.run(workspace, None, stream, args.stop_after)
                ev_done[i].record(stream)
                if i == last_prefill and cache_free is not None:
                    cache_free[j % 2].record(stream)
            with torch.cuda.stream(s_out):
                for i, (p, hout) in enumerate(zip(parts, host_out)):
                    s_out.wait_event(ev_done[i])
                    hout.copy_(p.out, non_blocking=True)
                    ev_out[i].record(s_out)
        e2e_step()
        stream.wait_stream(s_out)
        torch.cuda.synchronize()
        barrier(ws)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        s_in.wait_event(a0)
        ksteps = max(2, args.steps // 2)
        for _ in range(ksteps):
            e2e_step()
        stream.wait_stream(s_out)          # the timed region ends when the last output is on the host
        a1.record(stream)
        if cache_sets is not None:
            for p in parts:
                if p.kind == "prefill":
                    p.caches = cache_sets[0]
        torch.cuda.synchronize()
        barrier(ws)
        ems = max_over_ranks(a0.elapsed_time(a1) / ksteps, ws)
        e2e = {"value": job_throughput(tokens, ws, ems), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": ems}
    st = msa.device_status()

    # never let this extra measurement cost the line itself
    next_rows = None
    if rank == 0:
        try:
            next_rows = time_next_rows(parts, pk)
        except Exception as exc:  # noqa: BLE001
            next_rows = {"error": str(exc)[:200]}
        try:
            fp8 = time_fp8_indexer(parts, pk)
            if fp8 is not None:
                next_rows = dict(next_rows or {}, index_decode_kernel_e4m3=fp8)
        except Exception as exc:  # noqa: BLE001
            next_rows = dict(next_rows or {}, index_decode_kernel_e4m3={"error": str(exc)[:200]})

    # the other workloads of the parity set, timed on their own after the step (not in `value`)
    if rank == 0 and args.workload == "msa_128k_1m" and not args.no_extra:
        for xname in ("prefill_32k", "verify_ragged"):
            try:
                xparts, xcalls = time_workload(xname, workspace)
                parts_summary[xname] = dict(workload_summary(xcalls, pk), separate_run=True)
                del xparts
            except Exception as exc:  # noqa: BLE001
                parts_summary[xname] = {"error": str(exc)[:200]}
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        try:
            cpu = OracleLeg(parts).run(seconds=20.0) if args.workload == "msa_128k_1m" else None
        except Exception as exc:  # noqa: BLE001
            cpu = {"error": str(exc)[:300]}
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded counter-based generator)",
                "config": {"workload": args.workload, "tokens_per_step": tokens,
                           "parts": [p.name for p in parts], "l2": "inputs larger than L2 (no flush)",
                           "heads": "64q/4kv, head_dim 128, indexer 8x64, block 128, k=16",
                           "parallelism": f"replicas x{ws}"},
                "roofline": roof, "fractions": fractions, "parts": parts_summary,
                "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
                "gpu_launches": sum(p.launches for p in parts) * args.steps,
                "device_status": int(st), "next_rows": next_rows}
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
