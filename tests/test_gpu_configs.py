"""Full-size parity for the remaining workload configurations.

* 1024 x 1024, mu = 2, tau = 0.7 (k = 2048): end to end against the oracle's whole
  run, with the extraction's tolerances (energy within 2e-3, zero fraction within 0.5
  points, trits equal until the first divergence, d within 1e-4 relative before it; the
  first divergent component is traced and its first differing half-step may differ
  only at entries within 1e-5 relative of the oracle's threshold).
* 16 x 1536 x 1536, mu = 2.5, tau cycling (the batched entry point): every matrix
  succeeds, two matrices equal single calls with the same group size bit for bit,
  and sampled components of matrix 0 are traced and replayed by the oracle on the
  residual the GPU's own earlier components leave (teacher forcing).
* 4096 x 4096, mu = 3.5, tau = 0.7 (k = 14336): the prefix property (the start vector
  of component i depends only on the seed and i, so the first k components of a run
  at larger mu are the run at smaller mu, bit for bit) and teacher-forced samples up
  to the last component.
"""
import numpy as np
import pytest
import torch

import ternary_rank_weight_b200 as ext
from oracle import externd_oracle as ora
from ternary_rank_weight_b200.workloads import WORKLOADS, llm_matrix

import _parity

pytestmark = pytest.mark.gpu


def _zero_fraction(B, C):
    return (np.count_nonzero(B == 0) + np.count_nonzero(C == 0)) / (B.size + C.size)


def test_llm_1024_end_to_end_matches_oracle():
    w = WORKLOADS["llm_1024x1024_mu2_tau0.7"]
    A = w.matrix(0)
    f = ext.factor(torch.from_numpy(A).cuda(), w.mu[0], w.tau[0], seed=w.seeds[0], want_d64=True)
    assert f.k == 2048
    ref = ora.greedy_als(A, k=f.k, tau=w.tau[0], seed=w.seeds[0])
    Bg, Cg = f.trits()
    e = f.energy.cpu().numpy()
    assert np.max(np.abs(e - ref.energy)) < 2e-3
    assert abs(_zero_fraction(Bg, Cg) - ref.zero_fraction()) < 0.005
    assert f.stats["safeguard_hits"] == ref.safeguard_hits == 0
    div = f.k
    for i in range(f.k):
        if not (np.array_equal(Bg[:, i], ref.B[:, i]) and np.array_equal(Cg[i], ref.C[i])):
            div = i
            break
    d64 = f.d64.cpu().numpy()
    if div > 0:
        assert np.allclose(d64[:div], ref.D[:div], rtol=1e-4, atol=0)
    if div < f.k:
        # the first divergence must start at a near-tie (traced, replayed by the oracle)
        assert _parity.teacher_forced(A, f, w.seeds[0], w.tau[0], [div], "llm 1024 first divergence") == 1
    assert div >= 16, div


def test_batched_attention_workload_full_size():
    w = WORKLOADS["attn_16x1536x1536_mu2.5_tau_cycle"]
    mats = [w.matrix(b) for b in range(w.count)]
    res, st = ext.factor_batched([torch.from_numpy(a).cuda() for a in mats], list(w.mu), list(w.tau),
                                 seeds=list(w.seeds))
    assert st == [0] * w.count
    G = res[0].stats["group"]
    for r in res:
        assert r.k == 3840
        e = r.energy.cpu().numpy()
        assert np.all(np.diff(e) >= -1e-12) and 0.5 < e[-1] < 1.0
    for b in (0, 7):
        f = ext.factor(torch.from_numpy(mats[b]).cuda(), w.mu[b], w.tau[b], seed=w.seeds[b], grid=G, cluster=res[0].stats["cluster"], block=res[0].stats["block"])
        assert torch.equal(f.B, res[b].B) and torch.equal(f.C, res[b].C) and torch.equal(f.D, res[b].D)
        assert torch.equal(f.energy, res[b].energy)
    f0 = ext.factor(torch.from_numpy(mats[0]).cuda(), w.mu[0], w.tau[0], seed=w.seeds[0], grid=G, cluster=res[0].stats["cluster"], block=res[0].stats["block"], want_d64=True)
    ndiv = _parity.teacher_forced(mats[0], f0, w.seeds[0], w.tau[0], (0, 1, 1919, 3839), "attn 1536 matrix 0", grid=G, cluster=res[0].stats["cluster"], block=res[0].stats["block"])
    assert ndiv <= 1


def test_llm_4096_prefix_property_and_sampled_parity():
    w = WORKLOADS["llm_4096x4096_mu3.5_tau0.7"]
    A = w.matrix(0)
    Ag = torch.from_numpy(A).cuda()
    big = ext.factor(Ag, w.mu[0], w.tau[0], seed=w.seeds[0], want_d64=True)
    small = ext.factor(Ag, 1.0, w.tau[0], seed=w.seeds[0])
    assert big.k == 14336 and small.k == 4096
    k = small.k
    assert torch.equal(big.B[:k], small.B) and torch.equal(big.C[:k], small.C) and torch.equal(big.D[:k], small.D)
    assert torch.equal(big.energy[:k], small.energy)
    e = big.energy.cpu().numpy()
    assert np.all(np.diff(e) >= -1e-12)
    assert big.stats["residual_energy"] == pytest.approx(e[-1], abs=1e-4)
    ndiv = _parity.teacher_forced(A, big, w.seeds[0], w.tau[0], (0, 4096, 14335), "llm 4096 samples")
    assert ndiv <= 1


def test_batch_slices_run_with_the_batch_plan_equal_the_whole_batch():
    """Strong scaling of a batch over GPUs: each rank runs a contiguous slice of the same matrices
    with the plan of the whole batch (CTAs per matrix, cluster size), so every matrix gets the
    bits of the single-GPU batched call.  Checked here on one GPU, slice by slice."""
    from ternary_rank_weight_b200 import dist
    w = WORKLOADS["attn_16x1536x1536_mu2.5_tau_cycle"]
    mats = [torch.from_numpy(w.matrix(b)).cuda() for b in range(w.count)]
    res, st = ext.factor_batched(mats, list(w.mu), list(w.tau), seeds=list(w.seeds))
    assert st == [0] * w.count
    _, plan = ext.factor_batched(mats, list(w.mu), list(w.tau), seeds=list(w.seeds), plan_only=True)
    G, cl, nt = res[0].stats["group"], res[0].stats["cluster"], res[0].stats["block"]
    assert (plan["group"], plan["cluster"], plan["pending"], plan["block"]) == (G, cl, res[0].stats["pending"], nt)
    for world in (2, 3):
        for rank in range(world):
            ws, idx = dist.slice_workload(w, world, rank)
            part, st2 = ext.factor_batched([mats[i] for i in idx], list(ws.mu), list(ws.tau), seeds=list(ws.seeds),
                                           grid=G, cluster=cl, block=nt)
            assert st2 == [0] * len(idx)
            for j, i in enumerate(idx):
                assert torch.equal(part[j].B, res[i].B) and torch.equal(part[j].C, res[i].C), (world, rank, i)
                assert torch.equal(part[j].D, res[i].D) and torch.equal(part[j].energy, res[i].energy)


def test_block_size_follows_the_work_per_cta():
    """The ALS kernel runs at 256, 512 or 1024 threads per CTA.  The automatic choice follows the
    work of one CTA per half-step, W = m n / G + 8 (m + n) for G CTAs per matrix: 256 below
    170000 (512 with refinement sweeps), 512 below 230000, 1024 above; an explicit block size
    overrides it, and a batch and a single call with the same grid choose alike."""
    A = torch.zeros((1536, 1536), device="cuda")
    want = {148: 256, 64: 256, 16: 512, 12: 512, 11: 1024, 9: 1024}   # W: 40k 61k 172k 221k 239k 287k
    for grid, nt in want.items():
        _, st = ext.factor_batched([A], [1.0], [0.7], grid=grid, plan_only=True)
        assert (st["group"], st["block"]) == (grid, nt), grid
    _, st = ext.factor_batched([A, A], [1.0, 1.0], [0.7, 0.7], grid=9, plan_only=True)
    assert (st["group"], st["block"]) == (9, 1024)
    for nt in (256, 512, 1024):
        _, st = ext.factor_batched([A], [1.0], [0.7], grid=148, block=nt, plan_only=True)
        assert st["block"] == nt
    # refinement sweeps take 512 where the extraction alone would take 256
    for grid, nt in ((148, 512), (16, 512), (9, 1024)):
        _, st = ext.factor_batched([A], [1.0], [0.7], grid=grid, sweeps=1, plan_only=True)
        assert st["block"] == nt, grid
    # the workloads: 256^2 and 1024^2 on 256 threads (1024^2 with ten sweeps on 512), 2560 x 6912
    # on 512, the 1536^2 batch on 1024
    for name, nt in (("iid_256x256_mu2_tau0.7", 256), ("llm_1024x1024_mu2_tau0.7", 256),
                     ("llm_1024x1024_mu2_tau0.7_sweep10", 512), ("mlp_2560x6912_bf16_mu3_tau1.0", 512),
                     ("attn_16x1536x1536_mu2.5_tau_cycle", 1024)):
        w = WORKLOADS[name]
        mats = [torch.zeros(shape, device="cuda") for shape in w.shapes]
        _, st = ext.factor_batched(mats, list(w.mu), list(w.tau), sweeps=w.sweeps, plan_only=True)
        assert st["block"] == nt, name
    # where the 1024-thread layout would leave a lazy-deflation depth below 8, 512 is kept: every
    # shape the 512-thread build can plan stays plannable
    big = torch.empty((12288, 12288), device="cuda")
    _, st = ext.factor_batched([big], [3.0], [1.0], plan_only=True)
    assert st["block"] == 1024 and st["pending"] >= 8
    _, st = ext.factor_batched([big], [3.0], [1.0], hs=[torch.ones(12288, device="cuda")], plan_only=True)
    assert st["block"] == 512 and st["pending"] >= 1
    del big
    big = torch.empty((20480, 20480), device="cuda")
    _, st = ext.factor_batched([big], [3.0], [1.0], plan_only=True)
    assert st["block"] == 512 and st["pending"] >= 1
    del big
    torch.cuda.empty_cache()
    # other sizes, and anything but 512 with the clustered kernel, are refused
    for kw in (dict(block=300), dict(block=128), dict(block=256, cluster=2), dict(block=1024, cluster=4)):
        with pytest.raises(ext.ExterndError) as e:
            ext.factor_batched([A], [1.0], [0.7], plan_only=True, **kw)
        assert e.value.status == ext.STATUS["EINVAL"], kw
        with pytest.raises(ext.ExterndError) as e:
            ext.factor(A[:64, :64].contiguous() + 1.0, 1.0, 0.7, **kw)
        assert e.value.status == ext.STATUS["EINVAL"], kw
