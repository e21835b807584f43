"""Multi-rank host logic on CPU: two gloo ranks, no GPU.

The factorization shards into independent matrices (one process per GPU, no
collective on the data path).  These tests run the rank plumbing that
bench.py uses for N > 1 -- per-rank matrices, barrier, max-over-ranks time,
whole-job throughput -- as real gloo process groups, and check that each rank's
share of the work is what a single process computes for the same matrices (the
per-matrix work is done by the fp64 oracle here, standing in for the GPU).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp

from ternary_rank_weight_b200 import dist
from ternary_rank_weight_b200.workloads import Workload, WORKLOADS


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    tdist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from oracle import externd_oracle as ora
        info = dist.rank_info()
        assert (info.world, info.rank) == (world, rank)
        base = Workload("tiny", ((24, 40), (32, 16)), (7, 8), (1.0, 1.5), (0.7, 1.0))
        w = dist.rank_workload(base, rank)
        energies = []
        for b in range(w.count):
            A = w.matrix(b)
            f = ora.greedy_als(A, k=ora.rank(*A.shape, w.mu[b]), tau=w.tau[b], iters=15, seed=w.seeds[b])
            energies.append(f.energy_final)
        dist.barrier()
        t_local = 10.0 * (rank + 1)                     # a made-up per-rank time (ms)
        t_max = dist.max_over_ranks(t_local)
        units = dist.sum_over_ranks(sum(ora.rank(*s, mu) for s, mu in zip(w.shapes, w.mu)))
        rate = dist.throughput(units, t_max)
        sl = dist.partition(16, world, rank)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([t_max, units, rate, sl.start, sl.stop] + list(w.seeds) + energies, dtype=np.float64))
    finally:
        tdist.destroy_process_group()


def test_two_gloo_ranks_shard_independent_matrices(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    r0 = np.load(tmp_path / "rank0.npy")
    r1 = np.load(tmp_path / "rank1.npy")
    # max over ranks and the whole-job rate agree on both ranks
    assert r0[0] == r1[0] == 20.0
    k_rank = 24 + 24          # rank(24, 40, 1.0) + rank(32, 16, 1.5)
    assert r0[1] == r1[1] == world * k_rank
    assert r0[2] == r1[2] == pytest.approx(world * k_rank / 0.020)
    # contiguous partition of a 16-matrix batch: disjoint, covering, balanced
    assert (r0[3], r0[4], r1[3], r1[4]) == (0, 8, 8, 16)
    # each rank factors its own matrices (distinct seeds) ...
    assert list(r0[5:7]) == [7, 8] and list(r1[5:7]) == [7 + dist.SEED_STRIDE, 8 + dist.SEED_STRIDE]
    # ... and gets what one process gets for the same matrices
    from oracle import externd_oracle as ora
    base = Workload("tiny", ((24, 40), (32, 16)), (7, 8), (1.0, 1.5), (0.7, 1.0))
    for rank, rec in ((0, r0), (1, r1)):
        w = dist.rank_workload(base, rank)
        for b in range(2):
            A = w.matrix(b)
            f = ora.greedy_als(A, k=ora.rank(*A.shape, w.mu[b]), tau=w.tau[b], iters=15, seed=w.seeds[b])
            assert rec[7 + b] == f.energy_final


def test_partition_and_rank_workload_host_logic():
    for count in (0, 1, 5, 16, 17):
        for world in (1, 2, 3, 8):
            parts = [dist.partition(count, world, r) for r in range(world)]
            covered = [i for p in parts for i in p]
            assert covered == list(range(count))
            sizes = [len(p) for p in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        dist.partition(4, 2, 2)
    w = WORKLOADS["attn_16x1536x1536_mu2.5_tau_cycle"]
    w3 = dist.rank_workload(w, 3)
    assert w3.shapes == w.shapes and w3.mu == w.mu and w3.tau == w.tau
    assert w3.seeds == tuple(s + 3 * dist.SEED_STRIDE for s in w.seeds)
    assert dist.rank_workload(w, 0) == w
    # not distributed: the collectives return the rank's own values
    assert dist.max_over_ranks(3.5) == 3.5 and dist.sum_over_ranks(2.0) == 2.0
    assert dist.throughput(100, 500.0) == pytest.approx(200.0)
    with pytest.raises(ValueError):
        dist.throughput(1, 0.0)


def _strong_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    tdist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from oracle import externd_oracle as ora
        base = Workload("tiny batch", ((24, 40), (32, 16), (20, 20), (16, 48), (40, 24)), (7, 8, 9, 10, 11),
                        (1.0, 1.5, 1.0, 2.0, 1.0), (0.7, 1.0, 2.0, 0.7, 1.0))
        w, idx = dist.slice_workload(base, world, rank)
        energies = []
        for b in range(w.count):
            A = w.matrix(b)
            f = ora.greedy_als(A, k=ora.rank(*A.shape, w.mu[b]), tau=w.tau[b], iters=15, seed=w.seeds[b])
            energies.append(f.energy_final)
        units = dist.sum_over_ranks(sum(ora.rank(*sh, mu) for sh, mu in zip(w.shapes, w.mu)))
        t_max = dist.max_over_ranks(5.0 * (rank + 1))
        np.save(os.path.join(out_dir, f"strong{rank}.npy"),
                np.array([idx.start, idx.stop, units, t_max] + energies, dtype=np.float64))
    finally:
        tdist.destroy_process_group()


def test_two_gloo_ranks_split_one_batch():
    """Strong scaling of a batch: contiguous slices of the SAME matrices; together the ranks
    process the whole batch once, and each matrix gets what a single process gets."""
    import tempfile
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_strong_worker, args=(world, _free_port(), d), nprocs=world, start_method="spawn")
        recs = [np.load(os.path.join(d, f"strong{r}.npy")) for r in range(world)]
    from oracle import externd_oracle as ora
    base = Workload("tiny batch", ((24, 40), (32, 16), (20, 20), (16, 48), (40, 24)), (7, 8, 9, 10, 11),
                    (1.0, 1.5, 1.0, 2.0, 1.0), (0.7, 1.0, 2.0, 0.7, 1.0))
    assert [(int(r[0]), int(r[1])) for r in recs] == [(0, 2), (2, 5)]
    total = sum(ora.rank(*sh, mu) for sh, mu in zip(base.shapes, base.mu))
    assert all(r[2] == total for r in recs) and all(r[3] == 10.0 for r in recs)
    got = [e for r in recs for e in r[4:]]
    for b in range(base.count):
        A = base.matrix(b)
        f = ora.greedy_als(A, k=ora.rank(*A.shape, base.mu[b]), tau=base.tau[b], iters=15, seed=base.seeds[b])
        assert got[b] == f.energy_final
