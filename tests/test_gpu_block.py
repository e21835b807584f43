"""§2.4 batched block ALS with decorrelated targets on the GPU (externd_factor_block) against the
fp64 oracle's block_als ("ExTernD: Expanded-Rank Ternary Decomposition", §2.4).

Both sides work in fp64 (residual, GEMMs, Cholesky solves), so their values agree to rounding
(~1e-13 relative): the trits of each block agree exactly up to the first block that differs (a
difference needs a target within that rounding of a threshold), the scales within 1e-9 relative
and the energies within 1e-9 before it, and the final energy within 2e-3.  b = 1 is the
sequential method (the oracle's greedy_als).  At full size the energies are compared block by
block with the oracle's stored run (tests/golden/oracle_block_mlp_2560x6912.json).
"""
import numpy as np
import pytest
import torch

import ternary_rank_weight_b200 as ext
from oracle import externd_oracle as ora
from ternary_rank_weight_b200.workloads import WORKLOADS, llm_matrix

pytestmark = pytest.mark.gpu


def _first_diff_block(Bg, Cg, ref, bw):
    k = ref.k
    for s0 in range(0, k, bw):
        s1 = min(k, s0 + bw)
        if not (np.array_equal(Bg[:, s0:s1], ref.B[:, s0:s1]) and np.array_equal(Cg[s0:s1], ref.C[s0:s1])):
            return s0
    return k


@pytest.mark.parametrize("m,n,mu,tau,b", [(48, 40, 0.5, 0.7, 1), (96, 160, 1.0, 1.0, 8), (256, 256, 2.0, 0.7, 0),
                                          (192, 320, 1.5, 1.0, 24), (129, 250, 1.0, 2.0, 16), (300, 517, 1.0, 0.7, 0)])
def test_block_als_matches_oracle(m, n, mu, tau, b):
    A = llm_matrix(m, n, seed=m + n, outliers=min(2, n))
    f = ext.factor_block(torch.from_numpy(A).cuda(), mu, tau, seed=3, b=b, want_d64=True)
    bw = b if b > 0 else ora.block_width(m, n)
    assert f.stats["group"] == min(bw, f.k)
    ref = ora.block_als(A, k=f.k, tau=tau, seed=3, b=bw)
    Bg, Cg = f.trits()
    div = _first_diff_block(Bg, Cg, ref, bw)
    d64 = f.d64.cpu().numpy()
    e = f.energy.cpu().numpy()
    if div > 0:
        assert np.allclose(d64[:div], ref.D[:div], rtol=1e-9, atol=1e-15)
        assert np.allclose(e[:div], ref.energy[:div], rtol=0, atol=1e-9)
    assert abs(e[-1] - ref.energy_final) < 2e-3
    assert np.all(np.diff(e) >= -1e-12)
    # the reconstruction's energy is the reported one
    Ah = ext.reconstruct(f.B, f.D, f.C, m, n).cpu().numpy()
    assert ora.energy(A, Ah) == pytest.approx(e[-1], abs=1e-5)


def test_block_of_one_is_the_sequential_method():
    A = llm_matrix(64, 48, seed=5, outliers=2)
    f = ext.factor_block(torch.from_numpy(A).cuda(), 1.0, 0.7, seed=2, b=1, want_d64=True)
    seq = ora.greedy_als(A, k=f.k, tau=0.7, seed=2)
    Bg, Cg = f.trits()
    div = _first_diff_block(Bg, Cg, seq, 1)
    assert div >= 16
    assert np.allclose(f.d64.cpu().numpy()[:div], seq.D[:div], rtol=1e-9, atol=0)


def test_block_als_headline_matrix_against_the_oracle_run():
    """2560 x 6912 (k = 7680) at the pages' default width (256): energy after every block within
    2e-3 of the oracle's block run, the first block's trits identical, and the block energy within
    0.2 points of the sequential method's (the pages' claim, §1 and the Table 1 caption)."""
    import json
    import os
    from golden.make_oracle_goldens import trit_digest
    w = WORKLOADS["mlp_2560x6912_bf16_mu3_tau1.0"]
    A = w.matrix(0)
    f = ext.factor_block(torch.from_numpy(A).cuda(), w.mu[0], w.tau[0], seed=w.seeds[0], want_d64=True)
    assert f.k == 7680 and f.stats["group"] == 256
    e = f.energy.cpu().numpy()
    assert np.all(np.diff(e) >= -1e-12)
    gdir = os.path.join(os.path.dirname(__file__), "golden")
    with open(os.path.join(gdir, "oracle_block_mlp_2560x6912.json")) as fh:
        gb = json.load(fh)
    with open(os.path.join(gdir, "oracle_mlp_2560x6912.json")) as fh:
        gs = json.load(fh)
    idx = np.asarray(gb["energy_index"])
    assert np.max(np.abs(e[idx] - np.asarray(gb["energy"]))) < 2e-3
    Bg, Cg = f.trits()
    assert [trit_digest(Bg[:, i], Cg[i]) for i in range(256)] == gb["prefix_digest"][:256]
    assert np.allclose(f.d64.cpu().numpy()[:256], gb["prefix_d"][:256], rtol=1e-9, atol=0)
    assert abs(e[-1] - gs["energy"][-1]) < 0.002


def test_block_als_errors():
    A = torch.zeros((16, 16), device="cuda")
    with pytest.raises(ext.ExterndError) as er:
        ext.factor_block(A, 1.0, 0.7)
    assert er.value.status == ext.STATUS["EZERO"]
    A[0, 0] = float("nan")
    with pytest.raises(ext.ExterndError) as er:
        ext.factor_block(A, 1.0, 0.7)
    assert er.value.status == ext.STATUS["ENONFINITE"]
    with pytest.raises(ValueError):
        ext.factor_block(A.cpu(), 1.0, 0.7)
