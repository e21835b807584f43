"""Half-step parity between a kernel trace and the fp64 oracle (shared by the GPU tests).

The acceptance bar ("ExTernD: Expanded-Rank Ternary Decomposition", §2.2 T_tau and §2.3
step 1): on the same residual, every ternarization is reproduced exactly except where
|x| lies within TIE (1e-5) relative of the threshold.  A trace holds, for every V-step
and U-step of a component, the output vector the kernel thresholded, the threshold and
the trits; the oracle replays the half-steps from the same start trits with its own
``half_step``.  The replay stops at the first half-step whose trits differ (the two
trajectories then legitimately part): every differing entry of that half-step must be a
near-tie on the oracle's side.
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass, field

import numpy as np

import ternary_rank_weight_b200 as ext
from oracle import externd_oracle as ora

TIE = 1e-5

_REPORT: list = []


def record(entry: dict) -> None:
    """Add one divergence (or a summary line) to the session report."""
    _REPORT.append(entry)


def write_report(path: str) -> None:
    with open(path, "w") as f:
        json.dump(_REPORT, f, indent=1)
        f.write("\n")


def report_path():
    return os.environ.get("EXTERND_DIVERGENCE_REPORT")


@dataclass
class Replay:
    steps: int = 0                       # half-steps compared (trits equal)
    diverged: bool = False
    half_step: int = -1                  # index of the first differing half-step (0 = first V-step)
    entries: list = field(default_factory=list)    # (index, gpu trit, oracle trit, relative margin)
    max_pre_err: float = 0.0             # largest |pre_gpu - pre_oracle| / thr_oracle before the divergence


def own_trits_consistent(pre: np.ndarray, thr: float, trits: np.ndarray) -> bool:
    """The traced trits are T_tau of the traced vector at the traced threshold (§2.2, incl. the
    all-zero fallback: lowest index of largest magnitude, +1 for an all-zero vector)."""
    want = np.where(np.abs(pre) > thr, np.where(pre < 0, -1, 1), 0).astype(np.int8)
    if not want.any():
        j = int(np.argmax(np.abs(pre)))
        want[j] = -1 if pre[j] < 0 else 1
    return bool(np.array_equal(want, trits))


def replay(tr, c: int, R_eff: np.ndarray, u0: np.ndarray, tau: float, iters: int, pre_tol=None,
           hw=None) -> Replay:
    """Replay component c of trace ``tr`` with the oracle on the fp64 residual ``R_eff``.

    pre_tol(kind, t_in, pre_oracle) -> per-entry bound on |pre_gpu - pre_oracle|; None
    skips the check (the residuals then agree only up to the kernel's fp32 rounding).
    hw: the normalized importance weights of §2.5 (U-steps on R diag(h~)), or None."""
    m, n = R_eff.shape
    pv = tr.pre_v[c].cpu().numpy()
    tv = tr.thr_v[c].cpu().numpy()
    rv = ext.unpack_trits(tr.trit_v[c].cpu().numpy(), n)
    pu = tr.pre_u[c].cpu().numpy()
    tu = tr.thr_u[c].cpu().numpy()
    ru = ext.unpack_trits(tr.trit_u[c].cpu().numpy(), m)
    out = Replay()
    t_in = np.asarray(u0, dtype=np.int8)
    for it in range(iters):
        for kind in ("V", "U"):
            transpose = kind == "V"
            pre_g, thr_g, tri_g = (pv[it], tv[it], rv[it]) if transpose else (pu[it], tu[it], ru[it])
            if np.isnan(thr_g):
                # not run: a refinement refit stops at a fixed point (a U-step that changed no
                # trit), and every later iteration would repeat it; the oracle's replay does
                return out
            if hw is None:
                pre_o, thr_o, tri_o, _ = ora.half_step(R_eff, t_in, tau, transpose)
            else:
                pre_o, thr_o, tri_o, _ = ora.half_step_weighted(R_eff, t_in, tau, transpose, hw)
            assert own_trits_consistent(pre_g, thr_g, tri_g), (kind, it)
            if thr_o > 0:
                out.max_pre_err = max(out.max_pre_err, float(np.max(np.abs(pre_g - pre_o))) / thr_o)
            if pre_tol is not None:
                tol = pre_tol(kind, t_in, pre_o)
                assert np.all(np.abs(pre_g - pre_o) <= tol), (kind, it, float(np.max(np.abs(pre_g - pre_o) - tol)))
                assert abs(thr_g - thr_o) <= tau / pre_o.shape[0] * float(np.sum(tol)) + 1e-12 * thr_o, (kind, it)
            bad = np.nonzero(tri_g != tri_o)[0]
            h = 2 * it + (0 if transpose else 1)
            if bad.size:
                out.diverged = True
                out.half_step = h
                for j in bad:
                    marg = abs(abs(pre_o[j]) - thr_o) / thr_o if thr_o > 0 else float("inf")
                    out.entries.append((int(j), int(tri_g[j]), int(tri_o[j]), float(marg)))
                return out
            out.steps += 1
            t_in = tri_o
    return out


def assert_tie_only(rep: Replay, what) -> None:
    """A divergence must start at a near-tie: every differing entry within TIE of the threshold."""
    if rep.diverged:
        worst = max(e[3] for e in rep.entries)
        assert worst <= TIE, (what, rep.half_step, rep.entries[:8])


def first_divergence(Bg, Cg, Bo, Co, k) -> int:
    for i in range(k):
        if not (np.array_equal(Bg[:, i], Bo[:, i]) and np.array_equal(Cg[i], Co[i])):
            return i
    return k


def localize(A, f, seed: int, tau: float, comp: int, iters: int = 15, **factor_kw):
    """Re-run the factorization with a trace of component ``comp`` (the kernel is deterministic:
    the factors must repeat bit for bit), rebuild the residual that the GPU's own earlier
    components leave (teacher forcing, fp64) and replay the component with the oracle."""
    import torch
    Ag = torch.from_numpy(A).cuda() if isinstance(A, np.ndarray) else A
    g = ext.factor(Ag, f.mu, tau, iters=iters, seed=seed, want_d64=True, trace=(comp, 1), **factor_kw)
    assert torch.equal(g.B.cpu(), f.B.cpu()) and torch.equal(g.C.cpu(), f.C.cpu()) and torch.equal(g.D.cpu(), f.D.cpu())
    Bg, Cg = f.trits()
    d64 = f.d64.cpu().numpy()
    Ah = A if isinstance(A, np.ndarray) else A.cpu().numpy()
    R = ora.residual_after(Ah, Bg, d64, Cg, comp)
    u0, _, _ = ora.ternarize(ora.start_normals(seed, comp, Ah.shape[0]), tau)
    rep = replay(g.trace, 0, R, u0, tau, iters)
    return rep


def teacher_forced(A, f, seed: int, tau: float, samples, what, iters: int = 15, hw=None, **factor_kw) -> int:
    """Trace each sampled component of factorization ``f`` (re-run, deterministic), rebuild the
    residual the GPU's own earlier components leave (fp64) and replay it with the oracle.  Every
    divergence must start at a near-tie; a component without one must end in the same trits
    with d within 1e-4 relative.  The kernel's residual is fp32 (one rounding per entry and
    fold), so the replay records, but does not bound, the difference of the output vectors.
    Returns the number of sampled components that diverged."""
    import torch
    Ah = A if isinstance(A, np.ndarray) else A.cpu().numpy()
    Ag = torch.from_numpy(Ah).cuda()
    Bg, Cg = f.trits()
    d64 = f.d64.cpu().numpy()
    m = Ah.shape[0]
    ndiv = 0
    for i in samples:
        g = ext.factor(Ag, f.mu, tau, iters=iters, seed=seed, want_d64=True, trace=(int(i), 1), **factor_kw)
        assert torch.equal(g.B.cpu(), f.B.cpu()) and torch.equal(g.C.cpu(), f.C.cpu()), (what, i)
        R = ora.residual_after(Ah, Bg, d64, Cg, int(i))
        u0, _, _ = ora.ternarize(ora.start_normals(seed, int(i), m), tau)
        rep = replay(g.trace, 0, R, u0, tau, iters, hw=hw)
        record({"test": str(what), "component": int(i), "diverged": rep.diverged, "half_step": rep.half_step,
                "half_steps_equal": rep.steps, "entries": rep.entries[:16], "max_pre_err_rel_thr": rep.max_pre_err})
        assert_tie_only(rep, (what, int(i)))
        if rep.diverged:
            ndiv += 1
        else:
            d_o = ora.ls_scale(R, Bg[:, i], Cg[i]) if hw is None else ora.weighted_ls_scale(R, Bg[:, i], Cg[i], hw)
            assert abs(d64[i] - d_o) <= 1e-4 * abs(d_o), (what, int(i), d64[i], d_o)
    return ndiv
