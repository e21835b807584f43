"""ExTernD greedy sequential ternary ALS on B200 (sm_100a).

The factorization runs in the CUDA library ``libexternd.so`` (C ABI in
include/externd.h); this package is its Python binding plus the seeded
synthetic workload generators.
"""
from .api import (ExterndError, Factors, STATUS, debug_halfstep, debug_start_trits, factor,  # noqa: F401
                  factor_batched, last_stats, pack_trits, rank, reconstruct, strerror, trit_bytes,
                  unpack_trits)

__all__ = [
    "ExterndError", "Factors", "STATUS", "debug_halfstep", "debug_start_trits", "factor", "factor_batched",
    "last_stats", "pack_trits", "rank", "reconstruct", "strerror", "trit_bytes", "unpack_trits",
]
