"""Plain CPU oracle for FP8 (e4m3) K/V and indexer-key caches.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke check and
the benchmark's CPU-baseline / reference arm may import this module.  It shares
no code with the CUDA library and imports nothing from it.

Source: [daily.dev] "MiniMax M3: 1M-token multimodal reasoning model ...",
section "What's coming": FP8 KV-cache paths are on the vLLM roadmap.  The pages
fix no format, so every step below is a reading:

* format e4m3 ("fn": no infinities, finite range +-448, smallest subnormal
  2^-9, 3 mantissa bits);
* one float scale per cache tensor (K, V, indexer keys), chosen by the writer:
  code = e4m3(clamp(x / scale, -448, 448)) rounded to nearest, ties to even;
  the value read back is code * scale;
* the path reads the dequantized values and computes exactly what the bf16
  path computes on them (indexer scores, selection, attention).

Parity pins: tests/test_oracle_pins_fp8.py (torch's float8_e4m3fn cast inside
the finite range, every representable code round-tripping exactly, the
saturation and relative-error bounds, and brute force on the dequantized
indexer scores).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL_EXP = -6     # smallest normal 2^-6
E4M3_MANT_BITS = 3
E4M3_SUBNORMAL_QUANTUM = 2.0 ** -9


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def round_e4m3(y) -> np.ndarray:
    """Nearest e4m3 value of each entry of y (ties to even), saturated to +-448."""
    y = np.clip(_f64(y), -E4M3_MAX, E4M3_MAX)
    a = np.abs(y)
    # binade of |y|: |y| = m * 2^e with m in [0.5, 1), so floor(log2|y|) = e - 1
    _, e = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(e - 1, E4M3_MIN_NORMAL_EXP)            # below 2^-6 the spacing stays 2^-9
    quantum = np.ldexp(1.0, e - E4M3_MANT_BITS)
    q = np.round(a / quantum) * quantum                    # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, y)


def quantize(x, scale: float) -> np.ndarray:
    """e4m3 code values (as float64) of x / scale."""
    return round_e4m3(_f64(x) / float(scale))


def decode_bits(bits) -> np.ndarray:
    """Values of e4m3 ("fn") bit patterns (uint8): sign bit 7, exponent bits 6..3 (bias 7), mantissa
    bits 2..0; exponent 0 is subnormal (m * 2^-9); the two patterns 0x7F / 0xFF are NaN."""
    b = np.asarray(bits, dtype=np.int64) & 0xFF
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64)))
    mag = np.where((b & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def dequantize(codes, scale: float) -> np.ndarray:
    return _f64(codes) * float(scale)


def roundtrip(x, scale: float) -> np.ndarray:
    """What a reader of the FP8 cache sees for the values x written with this scale."""
    return dequantize(quantize(x, scale), scale)
