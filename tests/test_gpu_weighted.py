"""Parity of the importance-weighted factorization (§2.5) with the oracle.

Same tolerances as the plain path (the arithmetic is the same plus one fp32
weight per U-step term, whose product with an fp32 residual entry is exact in
fp64): trits equal away from threshold ties (1e-5 relative), d within 1e-4
relative until the first divergence; the first divergent component is traced
and replayed by the oracle, and its first differing half-step may differ only at
entries within 1e-5 relative of the threshold; weighted energy within 2e-3.
"""
import numpy as np
import pytest
import torch

import ternary_rank_weight_b200 as ext
from oracle import externd_oracle as ora
from ternary_rank_weight_b200.workloads import WORKLOADS, importance_weights, llm_matrix

import _parity

pytestmark = pytest.mark.gpu


def _first_divergence(B, C, ref):
    for i in range(ref.k):
        if not (np.array_equal(B[:, i], ref.B[:, i]) and np.array_equal(C[i], ref.C[i])):
            return i
    return ref.k


def test_uniform_weights_reproduce_the_plain_factorization_bit_for_bit():
    A = torch.from_numpy(llm_matrix(192, 256, seed=5)).cuda()
    f = ext.factor(A, 1.5, 1.0, seed=4)
    fw = ext.factor_weighted(A, np.full(256, 3.0, dtype=np.float32), 1.5, 1.0, lam=0.0, seed=4)
    assert torch.equal(f.B, fw.B) and torch.equal(f.C, fw.C) and torch.equal(f.D, fw.D)
    assert torch.allclose(f.energy, fw.energy, rtol=0, atol=1e-12)


@pytest.mark.parametrize("m,n,mu,tau,lam", [(7, 5, 2.0, 0.7, 0.0), (33, 65, 1.5, 1.0, 0.0), (96, 160, 2.0, 1.0, 0.0),
                                            (160, 96, 1.0, 0.7, 0.1), (256, 256, 2.0, 0.7, 0.0)])
def test_weighted_matches_oracle(m, n, mu, tau, lam):
    A = llm_matrix(m, n, seed=m + n, outliers=min(2, n))
    h = importance_weights(n, seed=n)
    fw = ext.factor(torch.from_numpy(A).cuda(), mu, tau, seed=3, h=h, lam=lam, want_d64=True)
    Bg, Cg = fw.trits()
    ref = ora.greedy_als_weighted(A, h.astype(np.float64), lam, k=fw.k, tau=tau, seed=3)
    e = fw.energy.cpu().numpy()
    assert np.all(np.diff(e) >= -1e-12)
    assert np.max(np.abs(e - ref.energy)) < 2e-3
    div = _first_divergence(Bg, Cg, ref)
    D = fw.D.cpu().numpy().astype(np.float64)
    if div > 0:
        assert np.allclose(D[:div], ref.D[:div].astype(np.float32), rtol=1e-4, atol=0)
    if div < ref.k:
        hwn = ora.normalized_weights(h.astype(np.float64), lam).astype(np.float64)
        nd = _parity.teacher_forced(A, fw, 3, tau, [div], ("weighted first divergence", m, n), hw=hwn, h=h, lam=lam)
        assert nd == 1
    # the weighted energy of the reconstruction agrees with the incremental one
    hw = ora.normalized_weights(h.astype(np.float64), lam)
    Ah = ext.reconstruct(fw.B, fw.D, fw.C, m, n).cpu().numpy()
    assert ora.weighted_energy(A, Ah, hw) == pytest.approx(e[-1], abs=1e-4)
    assert fw.stats["residual_energy"] == pytest.approx(e[-1], abs=1e-5)


def test_weighting_improves_the_weighted_energy():
    A = llm_matrix(256, 384, seed=12)
    h = importance_weights(384, seed=13)
    hw = ora.normalized_weights(h.astype(np.float64), 0.0)
    Ag = torch.from_numpy(A).cuda()
    f = ext.factor(Ag, 1.5, 1.0, seed=1)
    fw = ext.factor_weighted(Ag, h, 1.5, 1.0, lam=0.0, seed=1)
    e_plain = ora.weighted_energy(A, ext.reconstruct(f.B, f.D, f.C, 256, 384).cpu().numpy(), hw)
    assert fw.energy[-1].item() > e_plain


def test_invalid_weights_are_rejected():
    A = torch.from_numpy(llm_matrix(32, 48, seed=1)).cuda()
    for bad in (np.zeros(48, dtype=np.float32), -np.ones(48, dtype=np.float32),
                np.where(np.arange(48) == 5, np.nan, 1.0).astype(np.float32)):
        with pytest.raises(ext.ExterndError) as e:
            ext.factor_weighted(A, bad, 1.0, 0.7)
        assert e.value.status == ext.STATUS["EINVAL"]
    with pytest.raises(ext.ExterndError):
        ext.factor_weighted(A, np.ones(48, dtype=np.float32), 1.0, 0.7, lam=-1.0)
    # the context is still usable
    f = ext.factor_weighted(A, np.ones(48, dtype=np.float32), 1.0, 0.7)
    assert f.energy[-1].item() > 0.5


def test_weighted_headline_workload_full_size_sampled():
    """2560 x 6912 (k = 7680) with synthetic importance weights: teacher-forced samples."""
    w = WORKLOADS["mlp_2560x6912_bf16_mu3_tau1.0"]
    A = w.matrix(0)
    h = importance_weights(6912, seed=2)
    fw = ext.factor(torch.from_numpy(A).cuda(), w.mu[0], w.tau[0], seed=w.seeds[0], h=h, lam=0.0, want_d64=True)
    e = fw.energy.cpu().numpy()
    assert fw.k == 7680 and np.all(np.diff(e) >= -1e-12) and 0.5 < e[-1] < 1.0
    assert fw.stats["residual_energy"] == pytest.approx(e[-1], abs=1e-4)
    hw = ora.normalized_weights(h.astype(np.float64), 0.0).astype(np.float64)
    ndiv = _parity.teacher_forced(A, fw, w.seeds[0], w.tau[0], (0, 1, 700, 7679), "weighted mlp 2560x6912 samples",
                                  hw=hw, h=h, lam=0.0)
    assert ndiv <= 1
