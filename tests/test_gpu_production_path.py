"""Half-step parity of the production ALS kernel on a given residual state.

``externd_debug_component`` runs one component of §2.3 ("ExTernD: Expanded-Rank Ternary
Decomposition") through the kernel that every factorization and the benchmark run: the
incremental GEMVs over the trits that changed since the previous half-step of the same kind
(coefficients +-1 and +-2), the corrections of up to 31 pending rank-1 terms (deflations not
yet folded into R), the tagged-word exchange of 44-bit values and the threshold pass every
CTA runs.  The caller fixes the state -- an fp32 residual R, the pending terms d_j u_j v_j^T
and the start trits -- so the oracle can replay the component on exactly the residual the
kernel fits, R_eff = R - sum_j d_j u_j v_j^T, in fp64.

Tolerances, from the kernel's arithmetic:
* output vectors: |x_gpu - x| <= 2^-43 |x| + 1e-8 S, S = the sum of |terms| of the direct
  evaluation (|R|^T |t| plus sum_j |d_j| |t_j . t| |v_j|).  The kernel adds every term
  exactly to an fp64 sum (error (N - 1) 2^-53 times the sum of |terms| over the
  component's incremental history, which is at most 2 iters / density times S) and
  exchanges values rounded to 44 significant bits;
* thresholds: tau / len times the summed bound, plus 1e-12 relative (fp64 sums);
* trits: identical except entries within 1e-5 relative of the oracle's threshold (a tie);
  the replay stops at the first half-step with such a tie;
* scale d (when no tie occurred): 1e-9 relative.
"""
import numpy as np
import pytest
import torch

import ternary_rank_weight_b200 as ext
from oracle import externd_oracle as ora

import _parity

pytestmark = pytest.mark.gpu


def _state(m, n, tau, n_pend, seed):
    rng = np.random.default_rng(seed)
    R = (0.02 * rng.standard_normal((m, n))).astype(np.float32)
    pu = rng.choice(np.array([-1, 0, 1], dtype=np.int8), size=(n_pend, m), p=[0.28, 0.44, 0.28])
    pv = rng.choice(np.array([-1, 0, 1], dtype=np.int8), size=(n_pend, n), p=[0.28, 0.44, 0.28])
    pd = 0.004 * rng.standard_normal(n_pend)
    u0, _, _ = ora.ternarize(rng.standard_normal(m), tau)
    R_eff = R.astype(np.float64)
    for j in range(n_pend):
        R_eff -= pd[j] * np.outer(pu[j].astype(np.float64), pv[j].astype(np.float64))
    return R, pu, pv, pd, u0, R_eff


def _run(m, n, tau, n_pend, grid, seed, iters=15):
    R, pu, pv, pd, u0, R_eff = _state(m, n, tau, n_pend, seed)
    kw = {}
    if n_pend:
        kw = dict(pend_d=torch.from_numpy(pd).cuda(), pend_u=torch.from_numpy(ext.pack_trits(pu)).cuda(),
                  pend_v=torch.from_numpy(ext.pack_trits(pv)).cuda())
    tr, d64, uo, vo = ext.debug_component(torch.from_numpy(R).cuda(), torch.from_numpy(ext.pack_trits(u0)).cuda(),
                                          tau, iters, grid=grid, **kw)
    aR = np.abs(R).astype(np.float64)
    apu, apv, apd = np.abs(pu).astype(np.float64), np.abs(pv).astype(np.float64), np.abs(pd)

    def pre_tol(kind, t_in, pre_o):
        t = t_in.astype(np.float64)
        if kind == "V":
            S = aR.T @ np.abs(t) + (apd * np.abs(pu.astype(np.float64) @ t)) @ apv if n_pend else aR.T @ np.abs(t)
        else:
            S = aR @ np.abs(t) + (apd * np.abs(pv.astype(np.float64) @ t)) @ apu if n_pend else aR @ np.abs(t)
        return 2.0 ** -43 * np.abs(pre_o) + 1e-8 * S

    rep = _parity.replay(tr, 0, R_eff, u0, tau, iters, pre_tol=pre_tol)
    _parity.record({"test": "component", "m": m, "n": n, "tau": tau, "pending": n_pend, "grid": grid, "seed": seed,
                    "half_steps_equal": rep.steps, "diverged": rep.diverged, "half_step": rep.half_step,
                    "entries": rep.entries[:16], "max_pre_err_rel_thr": rep.max_pre_err})
    _parity.assert_tie_only(rep, (m, n, tau, n_pend, grid))
    if not rep.diverged:
        fit = ora.fit_component(R_eff, u0, tau, iters)
        assert np.array_equal(ext.unpack_trits(uo.cpu().numpy(), m), fit.u)
        assert np.array_equal(ext.unpack_trits(vo.cpu().numpy(), n), fit.v)
        assert d64 == pytest.approx(fit.d, rel=1e-9, abs=0)
    return rep


@pytest.mark.parametrize("m,n,tau,n_pend,grid", [
    (1, 1, 0.7, 0, 0), (7, 5, 0.7, 0, 1), (7, 5, 1.0, 3, 2), (33, 65, 1.0, 3, 3), (64, 48, 0.0, 3, 2),
    (300, 517, 0.7, 7, 0), (300, 517, 2.0, 5, 5), (256, 256, 0.7, 31, 1), (1024, 1024, 0.7, 31, 0),
    (1536, 1536, 2.0, 16, 9)])
def test_component_matches_oracle_on_given_state(m, n, tau, n_pend, grid):
    _run(m, n, tau, n_pend, grid, seed=m * 7 + n + n_pend)


@pytest.mark.parametrize("n_pend", [0, 31])
def test_component_full_size_in_the_bench_launch_configuration(n_pend):
    """2560 x 6912, tau = 1.0, the automatic grid (148 CTAs on a B200) and depth 32: the
    configuration the headline benchmark times, at an empty and a full pending list."""
    _run(2560, 6912, 1.0, n_pend, 0, seed=20 + n_pend)


def test_component_at_the_largest_shape_the_pages_tested():
    """~9216 x 2560 ("Limitations": the largest matrix the pages factor)."""
    _run(9216, 2560, 1.0, 31, 0, seed=9)


def test_pending_terms_beyond_the_depth_are_refused():
    """The pending list holds the caller's terms plus the component itself, at most 32."""
    m, n = 64, 48
    R, pu, pv, pd, u0, _ = _state(m, n, 0.7, 32, 1)
    Rg, ug = torch.from_numpy(R).cuda(), torch.from_numpy(ext.pack_trits(u0)).cuda()
    kw = dict(pend_d=torch.from_numpy(pd).cuda(), pend_u=torch.from_numpy(ext.pack_trits(pu)).cuda(),
              pend_v=torch.from_numpy(ext.pack_trits(pv)).cuda())
    with pytest.raises(ext.ExterndError) as e:
        ext.debug_component(Rg, ug, 0.7, **kw)
    assert e.value.status == ext.STATUS["ELIMIT"]
    kw31 = {k: v[:31] for k, v in kw.items()}
    tr, _, _, _ = ext.debug_component(Rg, ug, 0.7, **kw31)
    assert tr.pre_v.shape == (1, 15, n)


def test_trace_of_a_factorization_repeats_its_factors_and_follows_its_own_rule():
    """The trace option records what the run computed without changing it."""
    A = torch.from_numpy(np.random.default_rng(4).standard_normal((200, 300)).astype(np.float32) * 0.02).cuda()
    f = ext.factor(A, 1.0, 0.7, seed=2, want_d64=True)
    g = ext.factor(A, 1.0, 0.7, seed=2, want_d64=True, trace=(37, 5))
    assert torch.equal(f.B, g.B) and torch.equal(f.C, g.C) and torch.equal(f.d64, g.d64)
    Bg, Cg = g.trits()
    for c in range(5):
        last_v = ext.unpack_trits(g.trace.trit_v[c, -1].cpu().numpy(), 300)
        last_u = ext.unpack_trits(g.trace.trit_u[c, -1].cpu().numpy(), 200)
        assert np.array_equal(last_v, Cg[37 + c]) and np.array_equal(last_u, Bg[:, 37 + c])
        for it in range(15):
            assert _parity.own_trits_consistent(g.trace.pre_v[c, it].cpu().numpy(), g.trace.thr_v[c, it].item(),
                                                ext.unpack_trits(g.trace.trit_v[c, it].cpu().numpy(), 300))
