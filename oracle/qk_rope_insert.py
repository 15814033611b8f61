"""Plain CPU oracle for the step just before the MSA path: per-head QK
normalization, partial rotary embedding and the paged K/V insert.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke check and
the benchmark's CPU-baseline / reference arm may import this module.  It shares
no code with the CUDA library and imports nothing from it.

Float64 numpy, one definition at a time, in the order the pages state them.
Sources (page title, then section):

* [inteligile] "MiniMax-M3" model page, table "Checked in its code":
  - row "QK normalization": queries and keys each go through a per-head
    RMSNorm (q_norm / k_norm) before the rotary embedding and the attention
    dot product; use_qk_norm is true, qk_norm_type is "per_head";
  - row "Partial RoPE": partial_rotary_factor = 0.5, rotary_dim = 64; only the
    first rotary_dim channels of each head are rotated, the others pass
    through unchanged;
  - row "Layers without positional encoding (NoPE)": every attention layer,
    the sparse ones included, applies the same rotary embedding.
* [daily.dev] "MiniMax M3: 1M-token multimodal reasoning model ...", section
  "Serving options": the vLLM implementation fuses QKNorm + RoPE + KV insert
  into one kernel.

Readings where the pages leave a step open:

* RMSNorm: x / sqrt(mean over the head's channels of x^2 + eps) * w, with one
  weight vector of head_dim entries per projection (q or k) shared by all
  heads; eps is a parameter (1e-6 by default);
* rotary pairing "rotate half": inside the first rotary_dim channels, channel
  i pairs with channel i + rotary_dim / 2, and the pair turns by the angle
  p * theta^(-2 i / rotary_dim) at absolute position p; theta is a parameter
  (10,000 by default: the pages do not give the base);
* the norm covers all head_dim channels, the rotation only the first
  rotary_dim of them; values are inserted as given (no norm, no rotation);
* a row's position is its absolute position in its sequence
  (ctx_len - n_q + i for the i-th of a sequence's n_q new rows) and its K/V
  rows land in page page_table[seq][p // block_size], slot p % block_size.

Parity pins: tests/test_oracle_pins_rope.py (closed forms of the norm, the
rotation as a complex exponential, position-0 identity, the relative-position
invariant, a hand-worked fixture under tests/golden/, brute force on the
cache writes).
"""
from __future__ import annotations

from typing import Tuple

import numpy as np


def _f64(x) -> np.ndarray:
    """bf16/fp32 inputs widened exactly to float64."""
    if hasattr(x, "detach"):  # a torch tensor
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# 1. Per-head RMSNorm ("QK normalization" row)
# ---------------------------------------------------------------------------

def rms_norm_heads(x, weight, eps: float = 1e-6) -> np.ndarray:
    """x: [..., head_dim]; weight: [head_dim].  Each head's channels are divided
    by their root mean square (plus eps inside the root), then scaled by weight."""
    x = _f64(x)
    w = _f64(weight)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * w


# ---------------------------------------------------------------------------
# 2. Partial rotary embedding ("Partial RoPE" row)
# ---------------------------------------------------------------------------

def rope_angles(pos, rotary_dim: int, theta: float) -> np.ndarray:
    """[len(pos)][rotary_dim / 2]: angle of pair i at position p = p * theta^(-2i / rotary_dim)."""
    pos = np.asarray(pos, dtype=np.float64)
    half = rotary_dim // 2
    inv_freq = theta ** (-2.0 * np.arange(half, dtype=np.float64) / rotary_dim)
    return pos[:, None] * inv_freq[None, :]


def rope_partial(x, pos, rotary_dim: int = 64, theta: float = 10000.0) -> np.ndarray:
    """x: [T][H][head_dim]; pos: [T].  Rotates channel pairs (i, i + rotary_dim/2),
    i < rotary_dim/2, by their angle at the row's position; channels from rotary_dim
    on are copied unchanged."""
    x = _f64(x).copy()
    half = rotary_dim // 2
    ang = rope_angles(pos, rotary_dim, theta)[:, None, :]  # [T][1][half]
    c, s = np.cos(ang), np.sin(ang)
    a = x[..., :half].copy()
    b = x[..., half:rotary_dim].copy()
    x[..., :half] = a * c - b * s
    x[..., half:rotary_dim] = b * c + a * s
    return x


# ---------------------------------------------------------------------------
# 3. Norm, rotation and paged insert for one call
# ---------------------------------------------------------------------------

def qknorm_rope_insert(q, k, v, q_weight, k_weight, pos, seq_of_row, page_table, k_cache, v_cache,
                       block_size: int = 128, rotary_dim: int = 64, theta: float = 10000.0,
                       eps: float = 1e-6) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """q: [T][H_q][D]; k, v: [T][H_kv][D] (this call's new rows); pos, seq_of_row: [T];
    page_table: [num_seqs][max_blocks]; k_cache, v_cache: [pages][H_kv][block_size][D].

    Returns (q_out, k_cache_out, v_cache_out): q_out = rope(rmsnorm(q)); row t's
    rope(rmsnorm(k)) and v go to page page_table[seq][p // block_size], slot
    p % block_size of every KV head; every other cache row is unchanged."""
    pos = np.asarray(pos, dtype=np.int64)
    q_out = rope_partial(rms_norm_heads(q, q_weight, eps), pos, rotary_dim, theta)
    k_new = rope_partial(rms_norm_heads(k, k_weight, eps), pos, rotary_dim, theta)
    v_new = _f64(v)
    kc = _f64(k_cache).copy()
    vc = _f64(v_cache).copy()
    for t in range(len(pos)):
        page = int(page_table[int(seq_of_row[t])][int(pos[t]) // block_size])
        slot = int(pos[t]) % block_size
        kc[page, :, slot, :] = k_new[t]
        vc[page, :, slot, :] = v_new[t]
    return q_out, kc, vc
