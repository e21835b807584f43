"""Parity of the refinement sweeps (§2.4, blocks of one component) with the oracle.

Teacher forcing: the kernel is deterministic, so the extraction inside a run with
sweeps equals a run without them (checked); the oracle's sweeps start from those
GPU factors (fp64 scales).  A component is compared as a rank-1 term, so (u, v, d)
and (u, -v, -d) are the same.  Tolerances are the extraction's: trits equal and d
within 1e-4 relative until the first visit that differs.  That visit is traced and
its refit replayed by the oracle on the added-back residual the GPU's own other
components leave: the first half-step whose trits differ may differ only at entries
within 1e-5 relative of the threshold; if no half-step differs, the refit/stored
decision must have been a tie (decreases within 1e-6 relative).  Energies within
2e-3 (1e-5 before any divergence).
"""
import numpy as np
import pytest
import torch

import ternary_rank_weight_b200 as ext
from oracle import externd_oracle as ora
from ternary_rank_weight_b200.workloads import WORKLOADS, importance_weights, llm_matrix

import _parity

pytestmark = pytest.mark.gpu


def _canonical(B, D, C):
    """Flip (u, v, d) with d < 0 to (u, -v, -d)."""
    sgn = np.where(np.asarray(D) < 0, -1, 1)
    return B.copy(), np.abs(np.asarray(D, dtype=np.float64)), (C * sgn[:, None].astype(np.int8))


def _run(A, mu, tau, seed, sweeps, h=None):
    """The factorization with sweeps (ref) and without (base).  Bits depend on the block size, and
    the automatic choice gives plans with sweeps 512 threads where it gives extraction alone 256,
    so base runs at ref's block size: its extraction is then ref's, bit for bit."""
    Ag = torch.from_numpy(A).cuda()
    ref = ext.factor(Ag, mu, tau, seed=seed, want_d64=True, sweeps=sweeps, h=h)
    base = ext.factor(Ag, mu, tau, seed=seed, want_d64=True, h=h, block=ref.stats["block"])
    ref.run_seed = seed
    return base, ref


def _visit_replay(A, base, ref, i, tau, h=None, what="sweep visit"):
    """Trace sweep 1's visit of component i (a deterministic re-run) and replay its refit with
    the oracle on the added-back residual: A minus the GPU's refined components before i and
    its extracted components after i.  Returns the replay (its divergence must be a tie)."""
    k = base.k
    m = A.shape[0]
    kw = {} if h is None else {"h": np.asarray(h, dtype=np.float32)}   # the weights were fp32 (exact round trip)
    g = ext.factor(torch.from_numpy(A).cuda(), base.mu, tau, seed=ref.run_seed, want_d64=True, sweeps=1,
                   trace=(k + i, 1), **kw)
    assert torch.equal(g.B, ref.B) and torch.equal(g.C, ref.C) and torch.equal(g.D, ref.D)
    B0, C0 = base.trits()
    B1, C1 = ref.trits()
    D0, D1 = base.d64.cpu().numpy(), ref.d64.cpu().numpy()
    Bm = np.concatenate([B1[:, :i], B0[:, i + 1:]], axis=1).astype(np.float64)
    Cm = np.concatenate([C1[:i], C0[i + 1:]], axis=0).astype(np.float64)
    Dm = np.concatenate([D1[:i], D0[i + 1:]])
    R = A.astype(np.float64) - (Bm * Dm) @ Cm
    hwn = None if h is None else ora.normalized_weights(np.asarray(h, dtype=np.float64), 0.0).astype(np.float64)
    rep = _parity.replay(g.trace, 0, R, B0[:, i], tau, 15, hw=hwn)
    _parity.record({"test": what, "visit_of": int(i), "diverged": rep.diverged, "half_step": rep.half_step,
                    "half_steps_equal": rep.steps, "entries": rep.entries[:16], "max_pre_err_rel_thr": rep.max_pre_err})
    _parity.assert_tie_only(rep, (what, i))
    return rep


def _check_one_sweep(A, base, ref, tau, h=None):
    B0, C0 = base.trits()
    D0 = base.d64.cpu().numpy()
    want = ora.refine_sweeps(A, B0, D0, C0, sweeps=1, tau=tau, h=h)
    B1, C1 = ref.trits()
    gb, gd, gc = _canonical(B1, ref.d64.cpu().numpy(), C1)
    ob, od, oc = _canonical(want.B, want.D, want.C)
    k = base.k
    div = k
    for i in range(k):
        if not (np.array_equal(gb[:, i], ob[:, i]) and np.array_equal(gc[i], oc[i])):
            div = i
            break
    if div > 0:
        assert np.allclose(gd[:div], od[:div], rtol=1e-4, atol=1e-12)
    if div < k:
        rep = _visit_replay(A, base, ref, div, tau, h=h, what=("first differing sweep visit", A.shape))
        if not rep.diverged:
            assert want.decision_margins[0, div] < 1e-6, (div, want.decision_margins[0, div])
        assert abs(ref.sweep_energy[0].item() - want.sweep_energy[0]) < 2e-3
    else:
        assert abs(ref.sweep_energy[0].item() - want.sweep_energy[0]) < 1e-5
    return want, div


@pytest.mark.parametrize("m,n,mu,tau", [(7, 5, 2.0, 0.7), (33, 65, 1.5, 1.0), (96, 160, 2.0, 1.0),
                                        (160, 96, 1.0, 0.7), (256, 256, 2.0, 0.7)])
def test_one_sweep_matches_oracle(m, n, mu, tau):
    A = llm_matrix(m, n, seed=m * 3 + n, outliers=min(2, n))
    base, ref = _run(A, mu, tau, seed=5, sweeps=1)
    # the extraction inside the refined run is the plain one, bit for bit
    assert torch.equal(base.energy, ref.energy)
    _, div = _check_one_sweep(A, base, ref, tau)
    assert ref.sweep_energy[0].item() >= base.energy[-1].item() - 1e-9
    # the refined factors reproduce the reported energy
    Ah = ext.reconstruct(ref.B, ref.D, ref.C, m, n).cpu().numpy()
    assert ora.energy(A, Ah) == pytest.approx(ref.sweep_energy[-1].item(), abs=1e-4)
    assert ref.stats["residual_energy"] == pytest.approx(ref.sweep_energy[-1].item(), abs=1e-5)


def test_weighted_sweep_matches_oracle():
    m, n = 128, 192
    A = llm_matrix(m, n, seed=21, outliers=2)
    h = importance_weights(n, seed=22)
    base, ref = _run(A, 1.5, 1.0, seed=3, sweeps=1, h=h)
    assert torch.equal(base.energy, ref.energy)
    _check_one_sweep(A, base, ref, 1.0, h=h.astype(np.float64))
    hw = ora.normalized_weights(h.astype(np.float64), 0.0)
    Ah = ext.reconstruct(ref.B, ref.D, ref.C, m, n).cpu().numpy()
    assert ora.weighted_energy(A, Ah, hw) == pytest.approx(ref.sweep_energy[-1].item(), abs=1e-4)


@pytest.mark.parametrize("m,n", [(4, 4), (1, 9), (40, 3)])
def test_single_component_sweeps(m, n):
    """k = 1: every visit re-reads the component written by the previous one."""
    A = llm_matrix(m, n, seed=m + 7 * n, outliers=0)
    mu = 1.0 / min(m, n)
    base, ref = _run(A, mu, 1.0, seed=1, sweeps=3)
    assert base.k == 1
    B0, C0 = base.trits()
    want = ora.refine_sweeps(A, B0, base.d64.cpu().numpy(), C0, sweeps=3, tau=1.0)
    np.testing.assert_allclose(ref.sweep_energy.cpu().numpy(), want.sweep_energy, atol=1e-6)
    B1, C1 = ref.trits()
    gb, gd, gc = _canonical(B1, ref.d64.cpu().numpy(), C1)
    ob, od, oc = _canonical(want.B, want.D, want.C)
    assert np.array_equal(gb, ob) and np.array_equal(gc, oc)
    assert np.allclose(gd, od, rtol=1e-6)


def test_several_sweeps_are_monotone_and_track_the_oracle():
    m, n = 192, 256
    A = llm_matrix(m, n, seed=31, outliers=2)
    base, ref = _run(A, 1.5, 1.0, seed=2, sweeps=4)
    se = ref.sweep_energy.cpu().numpy()
    assert np.all(np.diff(np.concatenate([[base.energy[-1].item()], se])) >= -1e-9)
    B0, C0 = base.trits()
    want = ora.refine_sweeps(A, B0, base.d64.cpu().numpy(), C0, sweeps=4, tau=1.0)
    assert np.max(np.abs(se - want.sweep_energy)) < 2e-3
    assert ref.stats["sweep_kept"] >= 0
    Ah = ext.reconstruct(ref.B, ref.D, ref.C, m, n).cpu().numpy()
    assert ora.energy(A, Ah) == pytest.approx(se[-1], abs=1e-4)


def test_sweeps_with_small_pending_depth_and_host_buffers():
    """Depth 2 folds after every visit; host (pinned) inputs stage through the call."""
    A = llm_matrix(64, 80, seed=41, outliers=1)
    Ah = torch.from_numpy(A).pin_memory()
    f2 = ext.factor(Ah, 1.5, 0.7, seed=4, sweeps=2, pending=2, want_d64=True)
    fd = ext.factor(torch.from_numpy(A).cuda(), 1.5, 0.7, seed=4, sweeps=2, want_d64=True)
    assert f2.sweep_energy is not None and not f2.sweep_energy.is_cuda
    # a different fold schedule changes fp32 rounding only
    assert np.max(np.abs(f2.sweep_energy.numpy() - fd.sweep_energy.cpu().numpy())) < 2e-3
    with pytest.raises(ext.ExterndError) as e:
        ext.factor(Ah, 1.5, 0.7, sweeps=1, pending=1)
    assert e.value.status == ext.STATUS["ELIMIT"]
    for bad in (-1, 1001):
        with pytest.raises(ext.ExterndError) as e:
            ext.factor(Ah, 1.5, 0.7, sweeps=bad)
        assert e.value.status == ext.STATUS["EINVAL"]


def test_refinement_headline_workload_full_size_sampled():
    """2560 x 6912 (k = 7680), one sweep: sampled visits teacher-forced.  Visit i sees
    A minus the refined components before i and the extracted ones after it (component
    i added back); the oracle's visit on that residual must give the GPU's term."""
    w = WORKLOADS["mlp_2560x6912_bf16_mu3_tau1.0_sweep1"]
    A = w.matrix(0)
    base, ref = _run(A, w.mu[0], w.tau[0], seed=w.seeds[0], sweeps=1)
    assert base.k == 7680 and torch.equal(base.energy, ref.energy)
    assert ref.sweep_energy[0].item() >= base.energy[-1].item() - 1e-9
    assert ref.stats["residual_energy"] == pytest.approx(ref.sweep_energy[0].item(), abs=1e-4)
    B0, C0 = base.trits()
    B1, C1 = ref.trits()
    D0 = base.d64.cpu().numpy()
    D1 = ref.d64.cpu().numpy()
    hw = np.ones(A.shape[1])
    mism = 0
    for i in (0, 1, 700, 7679):
        Bm = np.concatenate([B1[:, :i], B0[:, i + 1:]], axis=1).astype(np.float64)
        Cm = np.concatenate([C1[:i], C0[i + 1:]], axis=0).astype(np.float64)
        Dm = np.concatenate([D1[:i], D0[i + 1:]])
        R = A.astype(np.float64) - (Bm * Dm) @ Cm
        vis = ora.refine_visit(R, B0[:, i], C0[i], w.tau[0], 15, hw)
        gb, gd, gc = _canonical(B1[:, i:i + 1], D1[i:i + 1], C1[i:i + 1])
        ob, od, oc = _canonical(vis.u[:, None], np.array([vis.d]), vis.v[None, :])
        rep = _visit_replay(A, base, ref, i, w.tau[0], what="mlp 2560x6912 sweep visit")
        if np.array_equal(gb, ob) and np.array_equal(gc, oc):
            assert gd[0] == pytest.approx(od[0], rel=1e-4)
        else:
            if not rep.diverged:
                assert vis.decision_margin < 1e-6, (i, vis.decision_margin)
            mism += 1
    assert mism <= 1


@pytest.mark.parametrize("weighted", [False, True])
def test_batched_sweeps_equal_single_calls(weighted):
    """The batched entry point with per-matrix weights and sweeps gives each matrix what a
    single call with the same group size gives, bit for bit."""
    mats = [llm_matrix(200, 150, seed=30), llm_matrix(96, 300, seed=31), llm_matrix(250, 250, seed=32)]
    hs = [importance_weights(A.shape[1], seed=40 + i) for i, A in enumerate(mats)] if weighted else None
    lams = [0.0, 0.1, 0.0] if weighted else None
    mus, taus, seeds = [1.5, 1.0, 2.0], [0.7, 1.0, 2.0], [5, 6, 7]
    res, st = ext.factor_batched([torch.from_numpy(a).cuda() for a in mats], mus, taus, seeds=seeds,
                                 hs=hs, lams=lams, sweeps=2)
    assert st == [0, 0, 0]
    G, nt = res[0].stats["group"], res[0].stats["block"]
    for i, (A, mu, tau, sd, r) in enumerate(zip(mats, mus, taus, seeds, res)):
        kw = {"h": hs[i], "lam": lams[i]} if weighted else {}
        f = ext.factor(torch.from_numpy(A).cuda(), mu, tau, seed=sd, grid=G, block=nt, sweeps=2, **kw)
        assert torch.equal(f.B, r.B) and torch.equal(f.C, r.C) and torch.equal(f.D, r.D)
        assert torch.equal(f.energy, r.energy) and torch.equal(f.sweep_energy, r.sweep_energy)
        assert r.sweep_energy[-1].item() >= r.energy[-1].item() - 1e-9
