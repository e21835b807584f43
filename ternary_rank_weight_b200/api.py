"""Python binding of the ExTernD C ABI (include/externd.h).

Argument marshalling only: tensors are turned into pointers, every step of the
factorization runs in the CUDA library.  PyTorch provides device memory and
streams.  Inputs may live on the GPU (device pointers) or on the host (the
library stages them through device memory inside the call).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch

from . import _lib


class ExterndError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {strerror(status)} (status {status})")


STATUS = {
    "OK": 0, "EINVAL": -1, "EZERO": -2, "ENONFINITE": -3, "ENOMEM": -4,
    "ECUDA": -5, "ELAUNCH": -6, "ETIMEOUT": -7, "ELIMIT": -8,
}


def strerror(status: int) -> str:
    return _lib.load().externd_strerror(int(status)).decode()


def rank(m: int, n: int, mu: float) -> int:
    return int(_lib.load().externd_rank(int(m), int(n), float(mu)))


def trit_bytes(length: int) -> int:
    return int(_lib.load().externd_trit_bytes(int(length)))


def last_stats() -> dict:
    st = _lib.Stats()
    _lib.load().externd_last_stats(ctypes.byref(st))
    return st.as_dict()


def _check(rc: int, what: str):
    if rc != 0:
        raise ExterndError(rc, what)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    raise TypeError(type(t))


def _stream(stream, device) -> int:
    if stream is not None:
        return int(getattr(stream, "cuda_stream", stream))
    if device is not None and device.type == "cuda":
        return torch.cuda.current_stream(device).cuda_stream
    if torch.cuda.is_available():
        return torch.cuda.current_stream().cuda_stream
    return 0


def _as_matrix(A) -> torch.Tensor:
    if isinstance(A, np.ndarray):
        A = torch.from_numpy(np.ascontiguousarray(A, dtype=np.float32))
    if not isinstance(A, torch.Tensor) or A.dim() != 2:
        raise ValueError("A must be a 2-D float32 tensor or array")
    if A.dtype != torch.float32:
        raise ValueError("A must be float32")
    return A.contiguous()


def _empty(shape, dtype, like: torch.Tensor) -> torch.Tensor:
    if like.is_cuda:
        return torch.empty(shape, dtype=dtype, device=like.device)
    return torch.empty(shape, dtype=dtype, pin_memory=like.is_pinned())


class _on_device:
    def __init__(self, t: torch.Tensor):
        self.ctx = torch.cuda.device(t.device) if t.is_cuda else None

    def __enter__(self):
        if self.ctx:
            self.ctx.__enter__()

    def __exit__(self, *a):
        if self.ctx:
            self.ctx.__exit__(*a)


@dataclass
class Factors:
    """B diag(D) C with packed ternary rows (2 bits per trit)."""
    B: torch.Tensor                 # uint8 [k, trit_bytes(m)]  row i = column i of B
    D: torch.Tensor                 # float32 [k]
    C: torch.Tensor                 # uint8 [k, trit_bytes(n)]  row i = row i of C
    energy: Optional[torch.Tensor]  # float64 [k]
    m: int
    n: int
    k: int
    mu: float
    tau: float
    d64: Optional[torch.Tensor] = None
    stats: dict = field(default_factory=dict)
    sweep_energy: Optional[torch.Tensor] = None   # float64 [sweeps]: energy after each refinement sweep
    trace: Optional["Trace"] = None               # test hook: traced half-steps (factor(..., trace=...))

    def trits(self):
        """Unpacked (B as m x k int8, C as k x n int8) on the host."""
        Bu = unpack_trits(self.B.cpu().numpy(), self.m).T.copy()
        Cu = unpack_trits(self.C.cpu().numpy(), self.n)
        return Bu, Cu


@dataclass
class Trace:
    """Half-steps of components [first, first + count) as the kernel saw them (test hook).

    pre_v[c, t] / pre_u[c, t]: the published output of the t-th V-step (x = R^T u, length n)
    and U-step (y = R v, length m) of component first + c; thr_*: the thresholds; trit_*:
    the packed trits those half-steps produced."""
    first: int
    count: int
    pre_v: torch.Tensor
    thr_v: torch.Tensor
    trit_v: torch.Tensor
    pre_u: torch.Tensor
    thr_u: torch.Tensor
    trit_u: torch.Tensor

    @staticmethod
    def alloc(first: int, count: int, iters: int, m: int, n: int, device) -> "Trace":
        """Buffers pre-filled with NaN, so half-steps a visit did not run stay recognisable."""
        nan = dict(fill_value=float("nan"), dtype=torch.float64, device=device)
        return Trace(first, count,
                     torch.full((count, iters, n), **nan), torch.full((count, iters), **nan),
                     torch.zeros((count, iters, trit_bytes(n)), dtype=torch.uint8, device=device),
                     torch.full((count, iters, m), **nan), torch.full((count, iters), **nan),
                     torch.zeros((count, iters, trit_bytes(m)), dtype=torch.uint8, device=device))


def factor(A, mu: float, tau: float, iters: int = 15, seed: int = 0, *, grid: int = 0, pending: int = 0,
           wait_limit_s: float = 0.0, fault_skip_cta: Optional[int] = None, want_d64: bool = False,
           want_energy: bool = True, sweeps: int = 0, h=None, lam: float = 0.0, trace=None, cluster: int = 0,
           block: int = 0, async_status=None, stream=None) -> Factors:
    """Factor one matrix (externd_factor_ex).  Outputs are allocated where A lives.

    sweeps: §2.4 refinement sweeps after extraction (``energy`` keeps the extraction
    energies, ``sweep_energy`` the energy after each sweep).  h, lam: §2.5 importance
    weights (per-column second moments, n float32 values), or None for the plain objective.
    trace: (first, count) -- test hook, records the half-steps of those visits: visit
    i < k extracts component i, visit (s + 1) k + i is sweep s's refit of component i
    (``Factors.trace``; A must be on the GPU).  cluster: kernel choice (0 automatic, 1 one
    CTA per residual stripe, 2/4/8/16 the clustered kernel with that cluster size).
    block: threads per CTA (0 automatic, 256, 512 or 1024); the same grid, cluster and block
    give the same bits.
    async_status: a one-element int32 CUDA tensor: the call queues its work and returns at
    once; the tensor receives the status (0 or a negative code) when the stream gets there.
    A (and h) must then be contiguous float32 CUDA tensors, which the queued work reads until
    the stream reaches its end: keep them alive and unchanged until then (the outputs are the
    returned tensors).  ``stats`` then holds the launch plan only."""
    if async_status is not None:
        _check_async_inputs([A], h, async_status)
    A = _as_matrix(A)
    m, n = A.shape
    if h is not None:
        h = _weights(h, n)
    k = rank(m, n, mu)
    if k < 1:
        raise ExterndError(STATUS["EINVAL"], "externd_rank")
    B = _empty((k, trit_bytes(m)), torch.uint8, A)
    C = _empty((k, trit_bytes(n)), torch.uint8, A)
    D = _empty((k,), torch.float32, A)
    E = _empty((k,), torch.float64, A) if want_energy else None
    d64 = _empty((k,), torch.float64, A) if want_d64 else None
    opt = _lib.Options()
    opt.grid = int(grid)
    opt.pending = int(pending)
    opt.wait_limit_s = float(wait_limit_s)
    opt.fault_inject = 1 if fault_skip_cta is not None else 0
    opt.fault_skip_cta = int(fault_skip_cta) if fault_skip_cta is not None else -1
    opt.d64_out = _ptr(d64)
    SE = _empty((int(sweeps),), torch.float64, A) if sweeps > 0 else None
    opt.sweeps = int(sweeps)
    opt.sweep_energy_out = _ptr(SE)
    opt.h = _ptr(h)
    opt.lambda_ = float(lam)
    opt.cluster = int(cluster)
    opt.block = int(block)
    if async_status is not None:
        opt.async_status = _ptr(async_status)
    tr = None
    if trace is not None:
        if not A.is_cuda:
            raise ValueError("trace needs A on the GPU")
        tr = Trace.alloc(int(trace[0]), int(trace[1]), int(iters), m, n, A.device)
        opt.trace_first, opt.trace_count = tr.first, tr.count
        opt.trace_pre_v, opt.trace_thr_v, opt.trace_trit_v = _ptr(tr.pre_v), _ptr(tr.thr_v), _ptr(tr.trit_v)
        opt.trace_pre_u, opt.trace_thr_u, opt.trace_trit_u = _ptr(tr.pre_u), _ptr(tr.thr_u), _ptr(tr.trit_u)
    with _on_device(A):
        rc = _lib.load().externd_factor_ex(_ptr(A), m, n, float(mu), float(tau), int(iters), int(seed),
                                           _ptr(B), _ptr(D), _ptr(C), _ptr(E),
                                           _stream(stream, A.device), ctypes.byref(opt))
    _check(rc, "externd_factor")
    return Factors(B=B, D=D, C=C, energy=E, m=m, n=n, k=k, mu=float(mu), tau=float(tau), d64=d64,
                   stats=last_stats(), sweep_energy=SE, trace=tr)


def _check_async_inputs(As, h, async_status, hs=None):
    """An asynchronous call reads its inputs after it returns: they must be the caller's own
    tensors (contiguous float32 on the GPU, so no temporary copy is made) and the status an
    int32 CUDA tensor."""
    if not (isinstance(async_status, torch.Tensor) and async_status.is_cuda and async_status.dtype == torch.int32
            and async_status.numel() >= 1):
        raise ValueError("async_status must be an int32 CUDA tensor")
    ins = list(As) + ([h] if h is not None else []) + (list(hs) if hs is not None else [])
    for t in ins:
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()):
            raise ValueError("an asynchronous call needs contiguous float32 CUDA tensors as inputs")


def _weights(h, n: int) -> torch.Tensor:
    if isinstance(h, np.ndarray):
        h = torch.from_numpy(np.ascontiguousarray(h, dtype=np.float32))
    if not isinstance(h, torch.Tensor) or h.dtype != torch.float32 or h.numel() != n:
        raise ValueError("h must hold n float32 values")
    return h.contiguous()


def factor_weighted(A, h, mu: float, tau: float, lam: float = 0.0, iters: int = 15, seed: int = 0, *,
                    stream=None) -> Factors:
    """Importance-weighted factorization (externd_factor_weighted, §2.5).

    h: per-column second moments (n,), float32, on the host or the GPU.  The returned
    energy is the weighted energy.  (Refinement sweeps with weights: ``factor(..., h=h, sweeps=S)``.)"""
    A = _as_matrix(A)
    m, n = A.shape
    h = _weights(h, n)
    k = rank(m, n, mu)
    if k < 1:
        raise ExterndError(STATUS["EINVAL"], "externd_rank")
    B = _empty((k, trit_bytes(m)), torch.uint8, A)
    C = _empty((k, trit_bytes(n)), torch.uint8, A)
    D = _empty((k,), torch.float32, A)
    E = _empty((k,), torch.float64, A)
    with _on_device(A):
        rc = _lib.load().externd_factor_weighted(_ptr(A), m, n, float(mu), float(tau), int(iters), int(seed), _ptr(h),
                                                 float(lam), _ptr(B), _ptr(D), _ptr(C), _ptr(E),
                                                 _stream(stream, A.device))
    _check(rc, "externd_factor_weighted")
    return Factors(B=B, D=D, C=C, energy=E, m=m, n=n, k=k, mu=float(mu), tau=float(tau), stats=last_stats())


def factor_noalloc(A: torch.Tensor, mu: float, tau: float, iters: int = 15, seed: int = 0, *, out=None,
                   stream=None) -> Factors:
    """externd_factor_noalloc: the same factorization with no device allocation inside the call.

    For callers that cannot allocate device memory while the factorization runs
    (e.g. a service whose pool already reserved the GPU).  The library's scratch is
    a fixed static device array (``NOALLOC_SCRATCH_BYTES``); larger shapes are
    rejected (ELIMIT).  A and the outputs must live on the GPU; pass preallocated
    outputs as ``out=(B, D, C, energy)`` to keep this call allocation-free on the
    Python side too.  Calls share the scratch and must not overlap on the GPU."""
    if not (isinstance(A, torch.Tensor) and A.is_cuda and A.dtype == torch.float32 and A.dim() == 2):
        raise ValueError("A must be a 2-D float32 CUDA tensor")
    if not A.is_contiguous():
        # a contiguous copy would be an allocation on the caller's side
        raise ValueError("A must be contiguous (row-major): factor_noalloc makes no copies")
    m, n = A.shape
    k = rank(m, n, mu)
    if k < 1:
        raise ExterndError(STATUS["EINVAL"], "externd_rank")
    if out is None:
        out = (torch.empty((k, trit_bytes(m)), dtype=torch.uint8, device=A.device),
               torch.empty((k,), dtype=torch.float32, device=A.device),
               torch.empty((k, trit_bytes(n)), dtype=torch.uint8, device=A.device),
               torch.empty((k,), dtype=torch.float64, device=A.device))
    B, D, C, E = out
    with _on_device(A):
        rc = _lib.load().externd_factor_noalloc(_ptr(A), m, n, float(mu), float(tau), int(iters), int(seed),
                                                _ptr(B), _ptr(D), _ptr(C), _ptr(E), _stream(stream, A.device))
    _check(rc, "externd_factor_noalloc")
    return Factors(B=B, D=D, C=C, energy=E, m=m, n=n, k=k, mu=float(mu), tau=float(tau))


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def factor_block(A: torch.Tensor, mu: float, tau: float, iters: int = 15, seed: int = 0, *, b: int = 0,
                 want_d64: bool = False, stream=None) -> Factors:
    """§2.4 batched block ALS with decorrelated targets (externd_factor_block); b = 0 takes the
    pages' default width (256 capped at min(m, n) / 8).  A must be a float32 CUDA tensor."""
    if not (isinstance(A, torch.Tensor) and A.is_cuda and A.dtype == torch.float32 and A.dim() == 2):
        raise ValueError("A must be a 2-D float32 CUDA tensor")
    A = A.contiguous()
    m, n = A.shape
    k = rank(m, n, mu)
    if k < 1:
        raise ExterndError(STATUS["EINVAL"], "externd_rank")
    B = torch.empty((k, trit_bytes(m)), dtype=torch.uint8, device=A.device)
    C = torch.empty((k, trit_bytes(n)), dtype=torch.uint8, device=A.device)
    D = torch.empty((k,), dtype=torch.float32, device=A.device)
    E = torch.empty((k,), dtype=torch.float64, device=A.device)
    d64 = torch.empty((k,), dtype=torch.float64, device=A.device) if want_d64 else None
    with _on_device(A):
        rc = _lib.load().externd_factor_block(_ptr(A), m, n, float(mu), float(tau), int(iters), int(seed), int(b),
                                              _ptr(B), _ptr(D), _ptr(C), _ptr(E), _ptr(d64), _stream(stream, A.device))
    _check(rc, "externd_factor_block")
    return Factors(B=B, D=D, C=C, energy=E, m=m, n=n, k=k, mu=float(mu), tau=float(tau), d64=d64, stats=last_stats())


def factor_batched(As: Sequence, mus: Sequence[float], taus: Sequence[float], iters: int = 15,
                   seeds: Optional[Sequence[int]] = None, *, hs: Optional[Sequence] = None,
                   lams: Optional[Sequence[float]] = None, sweeps: int = 0, grid: int = 0, cluster: int = 0,
                   block: int = 0, plan_only: bool = False, async_status=None, stream=None):
    """Factor independent matrices in one launch (externd_factor_batched_ex).

    hs: per-matrix importance weights (§2.5; every matrix or none), lams their lambdas;
    sweeps: refinement sweeps (§2.4) for every matrix; grid, cluster, block: the launch (0:
    automatic; a matrix gets the same bits from any launch with the same three).  plan_only: return (None, stats of the plan) without device work.
    async_status: a one-element int32 CUDA tensor: queue the work and return at once; the
    tensor receives the batch's status when the stream gets there.  Every matrix (and weight
    vector) must then be a contiguous float32 CUDA tensor, kept alive and unchanged until then.
    Returns (list of Factors, list of per-matrix status codes)."""
    if async_status is not None:
        _check_async_inputs(As, None, async_status, hs)
    mats = [_as_matrix(a) for a in As]
    cnt = len(mats)
    if seeds is None:
        seeds = list(range(cnt))
    outs = []
    for A, mu, tau in zip(mats, mus, taus):
        m, n = A.shape
        k = rank(m, n, mu)
        if k < 1:
            raise ExterndError(STATUS["EINVAL"], "externd_rank")
        outs.append((_empty((k, trit_bytes(m)), torch.uint8, A), _empty((k,), torch.float32, A),
                     _empty((k, trit_bytes(n)), torch.uint8, A), _empty((k,), torch.float64, A), k))
    P = ctypes.c_void_p * cnt
    a_ptrs = P(*[_ptr(a) for a in mats])
    b_ptrs = P(*[_ptr(o[0]) for o in outs])
    d_ptrs = P(*[_ptr(o[1]) for o in outs])
    c_ptrs = P(*[_ptr(o[2]) for o in outs])
    e_ptrs = P(*[_ptr(o[3]) for o in outs])
    ms = (ctypes.c_int64 * cnt)(*[a.shape[0] for a in mats])
    ns = (ctypes.c_int64 * cnt)(*[a.shape[1] for a in mats])
    mu_a = (ctypes.c_double * cnt)(*[float(x) for x in mus])
    tau_a = (ctypes.c_double * cnt)(*[float(x) for x in taus])
    seed_a = (ctypes.c_uint64 * cnt)(*[int(s) for s in seeds])
    st = (ctypes.c_int * cnt)()
    opt = _lib.BatchOptions()
    keep = []   # ctypes arrays and tensors that must outlive the call
    if hs is not None:
        hts = [_weights(h, A.shape[1]) for h, A in zip(hs, mats)]
        harr = P(*[_ptr(h) for h in hts])
        keep += [hts, harr]
        opt.h = ctypes.cast(harr, ctypes.c_void_p)
        if lams is not None:
            larr = (ctypes.c_double * cnt)(*[float(x) for x in lams])
            keep.append(larr)
            opt.lambda_ = ctypes.cast(larr, ctypes.c_void_p)
    SEs = [_empty((int(sweeps),), torch.float64, A) if sweeps > 0 else None for A in mats]
    opt.sweeps = int(sweeps)
    opt.grid = int(grid)
    opt.cluster = int(cluster)
    opt.block = int(block)
    opt.plan_only = 1 if plan_only else 0
    if async_status is not None:
        opt.async_status = _ptr(async_status)
    if sweeps > 0:
        sarr = P(*[_ptr(x) for x in SEs])
        keep.append(sarr)
        opt.sweep_energy_out = ctypes.cast(sarr, ctypes.c_void_p)
    with _on_device(mats[0]):
        rc = _lib.load().externd_factor_batched_ex(cnt, a_ptrs, ms, ns, mu_a, tau_a, int(iters), seed_a,
                                                   b_ptrs, d_ptrs, c_ptrs, e_ptrs, st,
                                                   _stream(stream, mats[0].device), ctypes.byref(opt))
    stats = last_stats()
    if plan_only:
        _check(rc, "externd_factor_batched_ex")
        return None, stats
    res = []
    for A, mu, tau, o, se in zip(mats, mus, taus, outs, SEs):
        res.append(Factors(B=o[0], D=o[1], C=o[2], energy=o[3], m=A.shape[0], n=A.shape[1], k=o[4],
                           mu=float(mu), tau=float(tau), stats=stats, sweep_energy=se))
    statuses = list(st)
    if rc != 0 and all(s == 0 for s in statuses):
        _check(rc, "externd_factor_batched_ex")
    return res, statuses


def reconstruct(B: torch.Tensor, D: torch.Tensor, C: torch.Tensor, m: int, n: int, *, stream=None) -> torch.Tensor:
    """Ahat = B diag(D) C as an m x n float32 tensor on B's device."""
    k = D.shape[0]
    out = _empty((m, n), torch.float32, B)
    with _on_device(B):
        rc = _lib.load().externd_reconstruct(_ptr(B), _ptr(D), _ptr(C), int(m), int(n), int(k), _ptr(out),
                                             _stream(stream, B.device))
    _check(rc, "externd_reconstruct")
    return out


def debug_halfstep(R, trits_in: torch.Tensor, tau: float, transpose: bool, *, stream=None):
    """One V-step (transpose=True: x = R^T u) or U-step (y = R v) through the ALS kernel.

    Returns (pre-threshold fp64 vector, threshold, packed output trits)."""
    R = _as_matrix(R)
    m, n = R.shape
    lout = n if transpose else m
    pre = _empty((lout,), torch.float64, R)
    thr = _empty((1,), torch.float64, R)
    out = _empty((trit_bytes(lout),), torch.uint8, R)
    with _on_device(R):
        rc = _lib.load().externd_debug_halfstep(_ptr(R), m, n, 1 if transpose else 0, _ptr(trits_in), float(tau),
                                                _ptr(pre), _ptr(thr), _ptr(out), _stream(stream, R.device))
    _check(rc, "externd_debug_halfstep")
    return pre, float(thr[0].item()), out


def debug_component(R, u0: torch.Tensor, tau: float, iters: int = 15, *, pend_d=None, pend_u=None, pend_v=None,
                    grid: int = 0, stream=None):
    """One component of §2.3 on a given residual state (externd_debug_component, test hook).

    R: m x n float32 (GPU); u0: packed start trits (GPU); pend_d / pend_u / pend_v: pending
    rank-1 terms (fp64 scales, packed u rows, packed v rows, all on the GPU) that the kernel
    applies as lazy-deflation corrections.  Returns (Trace with count 1, d64, packed u, packed v)."""
    R = _as_matrix(R)
    m, n = R.shape
    dev = R.device
    tr = Trace.alloc(0, 1, int(iters), m, n, dev)
    D = torch.empty((1,), dtype=torch.float32, device=dev)
    d64 = torch.empty((1,), dtype=torch.float64, device=dev)
    uo = torch.empty((1, trit_bytes(m)), dtype=torch.uint8, device=dev)
    vo = torch.empty((1, trit_bytes(n)), dtype=torch.uint8, device=dev)
    npend = 0 if pend_d is None else int(pend_d.shape[0])
    with _on_device(R):
        rc = _lib.load().externd_debug_component(
            _ptr(R), m, n, float(tau), int(iters), _ptr(u0), npend, _ptr(pend_d), _ptr(pend_u), _ptr(pend_v),
            _ptr(tr.pre_v), _ptr(tr.thr_v), _ptr(tr.trit_v), _ptr(tr.pre_u), _ptr(tr.thr_u), _ptr(tr.trit_u),
            _ptr(D), _ptr(d64), _ptr(uo), _ptr(vo), int(grid), _stream(stream, dev))
    _check(rc, "externd_debug_component")
    return tr, float(d64[0].item()), uo[0], vo[0]


def debug_start_trits(m: int, k: int, tau: float, seed: int, device="cuda", *, stream=None) -> torch.Tensor:
    """Packed start trits of components 0..k-1 (k x trit_bytes(m)), generated on the GPU."""
    out = torch.empty((k, trit_bytes(m)), dtype=torch.uint8, device=device)
    with _on_device(out):
        rc = _lib.load().externd_debug_start_trits(int(m), int(k), float(tau), int(seed), _ptr(out),
                                                   _stream(stream, out.device))
    _check(rc, "externd_debug_start_trits")
    return out


# ---------------------------------------------------------------------------
# host codecs of the packed 2-bit format: 00 = 0, 01 = +1, 11 = -1
# ---------------------------------------------------------------------------

def unpack_trits(packed: np.ndarray, length: int) -> np.ndarray:
    """uint8 rows (..., nbytes) -> int8 (..., length)."""
    p = np.asarray(packed, dtype=np.uint8)
    shifts = np.array([0, 2, 4, 6], dtype=np.uint8)
    codes = (p[..., :, None] >> shifts) & 3
    codes = codes.reshape(*p.shape[:-1], p.shape[-1] * 4)[..., :length]
    out = np.zeros(codes.shape, dtype=np.int8)
    out[codes == 1] = 1
    out[codes == 3] = -1
    return out


def pack_trits(t: np.ndarray) -> np.ndarray:
    """int8 (..., length) in {-1, 0, 1} -> uint8 (..., trit_bytes(length))."""
    t = np.asarray(t, dtype=np.int8)
    length = t.shape[-1]
    nb = trit_bytes(length)
    codes = np.zeros((*t.shape[:-1], nb * 4), dtype=np.uint8)
    codes[..., :length][t == 1] = 1
    codes[..., :length][t == -1] = 3
    codes = codes.reshape(*t.shape[:-1], nb, 4)
    return (codes[..., 0] | (codes[..., 1] << 2) | (codes[..., 2] << 4) | (codes[..., 3] << 6)).astype(np.uint8)


# ---------------------------------------------------------------------------
# inference with the factors and mask+sign storage (§2.6)
# ---------------------------------------------------------------------------

def transpose_trits(T: torch.Tensor, rows: int, length: int, *, stream=None) -> torch.Tensor:
    """(rows x length) packed trits -> (length x rows) packed trits, on T's device."""
    out = torch.empty((length, trit_bytes(rows)), dtype=torch.uint8, device=T.device)
    with _on_device(T):
        rc = _lib.load().externd_transpose_trits(_ptr(T), int(rows), int(length), _ptr(out), _stream(stream, T.device))
    _check(rc, "externd_transpose_trits")
    return out


def inference_layout(f: "Factors") -> torch.Tensor:
    """B laid out for inference: m rows x trit_bytes(k), row r = B[r, 0..k)."""
    return transpose_trits(f.B, f.k, f.m)


def matvec(Bt: torch.Tensor, D: torch.Tensor, C: torch.Tensor, m: int, n: int, X: torch.Tensor, *,
           out: Optional[torch.Tensor] = None, z_work: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y = B diag(D) C X for X of shape (batch, n) or (n,), fp32 on the GPU (externd_matvec)."""
    k = D.shape[0]
    squeeze = X.dim() == 1
    X2 = X.reshape(1, -1) if squeeze else X
    if X2.dtype != torch.float32 or not X2.is_cuda:
        raise ValueError("X must be a float32 CUDA tensor")
    X2 = X2.contiguous()
    batch = X2.shape[0]
    Y = out if out is not None else torch.empty((batch, m), dtype=torch.float32, device=X2.device)
    Z = z_work if z_work is not None else torch.empty((min(batch, 8), k), dtype=torch.float32, device=X2.device)
    with _on_device(X2):
        rc = _lib.load().externd_matvec(_ptr(Bt), _ptr(D), _ptr(C), int(m), int(n), int(k), _ptr(X2), int(batch),
                                        _ptr(Y), _ptr(Z), _stream(stream, X2.device))
    _check(rc, "externd_matvec")
    return Y.reshape(-1) if squeeze else Y


def pack_mask_sign(T: torch.Tensor, rows: int, length: int, *, stream=None):
    """Mask+sign storage of packed trit rows: (mask bytes rows x ceil(length/8),
    sign bit stream as int32 words, bit offsets per row (rows + 1))."""
    mask = torch.empty((rows, (length + 7) // 8), dtype=torch.uint8, device=T.device)
    words = max(1, (rows * length + 31) // 32)
    signs = torch.empty((words,), dtype=torch.int32, device=T.device)
    offs = torch.empty((rows + 1,), dtype=torch.int64, device=T.device)
    with _on_device(T):
        rc = _lib.load().externd_pack_mask_sign(_ptr(T), int(rows), int(length), _ptr(mask), _ptr(signs), int(words),
                                                _ptr(offs), _stream(stream, T.device))
    _check(rc, "externd_pack_mask_sign")
    total = int(offs[-1].item())
    return mask, signs[: (total + 31) // 32], offs
