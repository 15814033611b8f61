"""CPU oracle for the MSA hot path: test infrastructure, not product code.

Only the tests, the package smoke check and the benchmark's CPU-baseline /
reference arm may import it.
"""
from .msa_oracle import (block_scores, select_blocks, boundary_gap, sparse_attention,  # noqa: F401
                         merge_partials, msa_rows)
from .qk_rope_insert import rms_norm_heads, rope_partial, qknorm_rope_insert  # noqa: F401
from .fp8_cache import round_e4m3, quantize, dequantize, roundtrip  # noqa: F401
