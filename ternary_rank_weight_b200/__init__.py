"""ExTernD greedy sequential ternary ALS on B200 (sm_100a).

The factorization runs in the CUDA library ``libexternd.so`` (C ABI in
include/externd.h); this package is its Python binding plus the seeded
synthetic workload generators.
"""
from .api import (ExterndError, Factors, NOALLOC_SCRATCH_BYTES, STATUS, Trace, debug_component,  # noqa: F401
                  debug_halfstep, debug_start_trits,
                  factor, factor_batched, factor_block, factor_noalloc, factor_weighted, inference_layout, last_stats, matvec, pack_mask_sign,
                  pack_trits, rank, reconstruct, strerror, transpose_trits, trit_bytes, unpack_trits)

__all__ = [
    "ExterndError", "Factors", "NOALLOC_SCRATCH_BYTES", "STATUS", "factor_noalloc", "debug_halfstep", "debug_start_trits", "debug_component", "Trace", "factor", "factor_batched", "factor_block",
    "last_stats", "pack_trits", "rank", "reconstruct", "strerror", "trit_bytes", "unpack_trits",
    "transpose_trits", "inference_layout", "matvec", "pack_mask_sign", "factor_weighted",
]
