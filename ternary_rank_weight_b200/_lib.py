"""ctypes loader for libexternd.so (the C ABI declared in include/externd.h).

The library is built in-tree by ``ternary_rank_weight_b200.build``.  If it is
missing, every entry point raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libexternd.so")

# Every symbol declared in include/externd.h.
EXPORTS = (
    "externd_rank",
    "externd_trit_bytes",
    "externd_factor",
    "externd_factor_ex",
    "externd_factor_weighted",
    "externd_factor_noalloc",
    "externd_factor_block",
    "externd_factor_batched",
    "externd_factor_batched_ex",
    "externd_reconstruct",
    "externd_strerror",
    "externd_debug_halfstep",
    "externd_debug_start_trits",
    "externd_debug_component",
    "externd_last_stats",
    "externd_transpose_trits",
    "externd_matvec",
    "externd_pack_mask_sign",
)


class Options(ctypes.Structure):
    _fields_ = [
        ("grid", ctypes.c_int),
        ("pending", ctypes.c_int),
        ("wait_limit_s", ctypes.c_double),
        ("fault_skip_cta", ctypes.c_int),
        ("fault_inject", ctypes.c_int),
        ("d64_out", ctypes.c_void_p),
        ("sweeps", ctypes.c_int),
        ("sweep_energy_out", ctypes.c_void_p),
        ("h", ctypes.c_void_p),
        ("lambda_", ctypes.c_double),
        ("trace_first", ctypes.c_int64),
        ("trace_count", ctypes.c_int64),
        ("trace_pre_v", ctypes.c_void_p),
        ("trace_thr_v", ctypes.c_void_p),
        ("trace_trit_v", ctypes.c_void_p),
        ("trace_pre_u", ctypes.c_void_p),
        ("trace_thr_u", ctypes.c_void_p),
        ("trace_trit_u", ctypes.c_void_p),
        ("cluster", ctypes.c_int),
        ("async_status", ctypes.c_void_p),
        ("block", ctypes.c_int),
    ]


class BatchOptions(ctypes.Structure):
    _fields_ = [
        ("h", ctypes.c_void_p),
        ("lambda_", ctypes.c_void_p),
        ("sweeps", ctypes.c_int),
        ("sweep_energy_out", ctypes.c_void_p),
        ("grid", ctypes.c_int),
        ("cluster", ctypes.c_int),
        ("plan_only", ctypes.c_int),
        ("async_status", ctypes.c_void_p),
        ("block", ctypes.c_int),
    ]


class Stats(ctypes.Structure):
    _fields_ = [
        ("als_ms", ctypes.c_double),
        ("setup_ms", ctypes.c_double),
        ("init_ms", ctypes.c_double),
        ("total_ms", ctypes.c_double),
        ("alg_bytes", ctypes.c_double),
        ("read_bytes", ctypes.c_double),
        ("residual_energy", ctypes.c_double),
        ("components", ctypes.c_int64),
        ("half_steps", ctypes.c_int64),
        ("fallbacks", ctypes.c_int64),
        ("launches", ctypes.c_int),
        ("grid", ctypes.c_int),
        ("group", ctypes.c_int),
        ("block", ctypes.c_int),
        ("vec_v", ctypes.c_int),
        ("vec_u", ctypes.c_int),
        ("pending", ctypes.c_int),
        ("smem_bytes", ctypes.c_size_t),
        ("workspace_bytes", ctypes.c_size_t),
        ("sweep_kept", ctypes.c_int64),
        ("phase_cycles", ctypes.c_int64 * 11),
        ("safeguard_hits", ctypes.c_int64),
        ("cluster", ctypes.c_int),
        ("reserved", ctypes.c_int),
    ]

    def as_dict(self):
        d = {name: getattr(self, name) for name, _ in self._fields_}
        d["phase_cycles"] = list(self.phase_cycles)
        return d


_lib = None


def load():
    """Load the shared library (once) and declare argument types."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m ternary_rank_weight_b200.build` "
            "(the CUDA library is required; there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, dbl, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_int
    u64 = ctypes.c_uint64
    L.externd_rank.argtypes = [i64, i64, dbl]
    L.externd_rank.restype = i64
    L.externd_trit_bytes.argtypes = [i64]
    L.externd_trit_bytes.restype = ctypes.c_size_t
    L.externd_factor.argtypes = [vp, i64, i64, dbl, dbl, c_int, u64, vp, vp, vp, vp, vp]
    L.externd_factor.restype = c_int
    L.externd_factor_ex.argtypes = [vp, i64, i64, dbl, dbl, c_int, u64, vp, vp, vp, vp, vp,
                                    ctypes.POINTER(Options)]
    L.externd_factor_ex.restype = c_int
    L.externd_factor_weighted.argtypes = [vp, i64, i64, dbl, dbl, c_int, u64, vp, dbl, vp, vp, vp, vp, vp]
    L.externd_factor_weighted.restype = c_int
    L.externd_factor_noalloc.argtypes = [vp, i64, i64, dbl, dbl, c_int, u64, vp, vp, vp, vp, vp]
    L.externd_factor_noalloc.restype = c_int
    L.externd_factor_block.argtypes = [vp, i64, i64, dbl, dbl, c_int, u64, c_int, vp, vp, vp, vp, vp, vp]
    L.externd_factor_block.restype = c_int
    L.externd_factor_batched.argtypes = [c_int, vp, vp, vp, vp, vp, c_int, vp, vp, vp, vp, vp, vp, vp]
    L.externd_factor_batched.restype = c_int
    L.externd_factor_batched_ex.argtypes = [c_int, vp, vp, vp, vp, vp, c_int, vp, vp, vp, vp, vp, vp, vp, vp]
    L.externd_factor_batched_ex.restype = c_int
    L.externd_reconstruct.argtypes = [vp, vp, vp, i64, i64, i64, vp, vp]
    L.externd_reconstruct.restype = c_int
    L.externd_strerror.argtypes = [c_int]
    L.externd_strerror.restype = ctypes.c_char_p
    L.externd_debug_halfstep.argtypes = [vp, i64, i64, c_int, vp, dbl, vp, vp, vp, vp]
    L.externd_debug_halfstep.restype = c_int
    L.externd_debug_start_trits.argtypes = [i64, i64, dbl, u64, vp, vp]
    L.externd_debug_start_trits.restype = c_int
    L.externd_debug_component.argtypes = [vp, i64, i64, dbl, c_int, vp, c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                          vp, vp, vp, vp, c_int, vp]
    L.externd_debug_component.restype = c_int
    L.externd_last_stats.argtypes = [ctypes.POINTER(Stats)]
    L.externd_last_stats.restype = c_int
    L.externd_transpose_trits.argtypes = [vp, i64, i64, vp, vp]
    L.externd_transpose_trits.restype = c_int
    L.externd_matvec.argtypes = [vp, vp, vp, i64, i64, i64, vp, i64, vp, vp, vp]
    L.externd_matvec.restype = c_int
    L.externd_pack_mask_sign.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp]
    L.externd_pack_mask_sign.restype = c_int
    _lib = L
    return L
