"""Benchmark: ternary components fitted per second by greedy sequential ALS.

Default workload: one 2560 x 6912 MLP-shaped matrix (LLM-like synthetic weights
rounded to bf16, held as fp32), mu = 3 (k = 7680 components), tau = 1.0,
15 alternating fits per component.  A "step" factors the whole matrix.

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]
                    [--workload NAME | --all]

N > 1 is launched by torch.distributed.run: each rank factors its own matrix
(seed + rank), no data-path collective (weak scaling); the barrier and the
max-over-ranks time use NCCL.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (test infrastructure) on the host
cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "ternary components fitted/s at 2560×6912 μ=3; achieved GB/s vs HBM peak"
UNIT = "components/s"
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _kernel_source_hash() -> str:
    """Hash of the ALS kernel's device code: externd_kernels.cuh and externd.cu up to its host half
    (which starts at `struct ProbIn`), line comments, blank lines and #include lines removed, so
    editing a comment, the host entry points or another kernel's header does not invalidate the
    recorded ncu traffic."""
    h = hashlib.sha256()
    for name in ("externd.cu", "externd_kernels.cuh"):
        with open(os.path.join(ROOT, "ternary_rank_weight_b200", "csrc", name), encoding="utf-8") as f:
            for line in f:
                if line.startswith("struct ProbIn"):
                    break
                code = line.split("//", 1)[0].rstrip()
                if code and not code.startswith("#include"):
                    h.update(code.encode() + b"\n")
    return h.hexdigest()


def _ncu_traffic(workload: str):
    """DRAM bytes per ALS launch from the committed ncu summary, if it was taken on this kernel source."""
    path = os.path.join(ROOT, "profiles", "als_kernel_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_sha256") != _kernel_source_hash():
        return None
    per = rec.get("dram_bytes_per_launch_scaled", {}).get(workload)
    return float(per) if per is not None else None


class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm.append(float(f[1]))
                    mx.append(float(f[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, f[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist():
    from ternary_rank_weight_b200.dist import rank_info
    r = rank_info()
    return r.world, r.rank, r.local


def _init_nccl(ws: int, local: int):
    """One process per GPU: bind the device and, for N > 1, join the NCCL group (barriers, max and
    sums over ranks).  Returns the device."""
    import torch
    torch.cuda.set_device(local)
    if ws > 1:
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=120))
    return torch.device("cuda", local)


def _fini_nccl(ws: int):
    import torch
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def _workload_arrays(name: str, rank: int, mu=None):
    """This rank's workload (weak scaling: same shapes and recipe, seeds offset by rank) and matrices."""
    import dataclasses
    from ternary_rank_weight_b200.dist import rank_workload
    from ternary_rank_weight_b200.workloads import WORKLOADS
    w = WORKLOADS[name]
    if mu is not None:
        w = dataclasses.replace(w, mu=tuple(mu for _ in w.mu))
    w = rank_workload(w, rank)
    return w, w.matrices()


def _config(w, extra=None):
    shapes = sorted(set(w.shapes))
    cfg = {"workload": w.name, "matrices": w.count,
           "shape": list(shapes[0]) if len(shapes) == 1 else [list(s) for s in shapes],
           "mu": w.mu[0] if len(set(w.mu)) == 1 else list(w.mu),
           "tau": w.tau[0] if len(set(w.tau)) == 1 else list(w.tau),
           "iters": w.iters, "recipe": w.recipe + ("+bf16" if w.bf16 else "") + ("+importance weights" if w.weighted else ""),
           "l2": "inputs larger than L2 (A + two residual copies exceed 126 MB); no flush"}
    if extra:
        cfg.update(extra)
    return cfg


# ---------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

def _oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def time_oracle(w, mats, budget_s: float = 15.0):
    """Time the fp64 oracle on a bounded prefix of components of matrix 0 of the workload."""
    from oracle import externd_oracle as ora
    A = mats[0]
    m, n = A.shape
    k_full = ora.rank(m, n, w.mu[0])
    # calibrate with 2 components, then size the sample to the budget
    t0 = time.perf_counter()
    ora.greedy_als(A, k=2, tau=w.tau[0], iters=w.iters, seed=w.seeds[0])
    per = (time.perf_counter() - t0) / 2
    kk = int(max(2, min(k_full, budget_s / max(per, 1e-6))))
    t0 = time.perf_counter()
    ora.greedy_als(A, k=kk, tau=w.tau[0], iters=w.iters, seed=w.seeds[0])
    dt = time.perf_counter() - t0
    return {"value": kk / dt, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"first {kk} of {k_full} components of matrix 0 ({m}x{n}, mu={w.mu[0]}, tau={w.tau[0]}), "
                      f"{dt:.1f} s, numpy fp64"}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    w, mats = _workload_arrays(args.workload, 0, args.mu)
    for _ in range(args.warmup):
        pass   # the oracle has nothing to warm up beyond the calibration inside time_oracle
    vals = []
    last = None
    t_all = time.perf_counter()
    for _ in range(args.steps):
        last = time_oracle(w, mats, budget_s=args.ref_budget)
        vals.append(last["value"])
    wall = time.perf_counter() - t_all
    value = statistics.mean(vals)
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": wall * 1000 / max(args.steps, 1), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": _config(w), "cpu_baseline": dict(last, value=value),
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


# ---------------------------------------------------------------------------
# CUDA path
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch
    import ternary_rank_weight_b200 as ext

    ws, rank, local = _dist()
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    from ternary_rank_weight_b200 import dist

    strong = args.scaling == "strong"
    plan = {"grid": args.grid, "cluster": args.cluster, "block": args.block}
    if strong:
        # one fixed batch split over the ranks: every rank takes a contiguous slice of the SAME
        # matrices and runs it with the plan of the whole batch on one GPU, so each matrix gets
        # the bits a single-GPU batched call gives
        w_full, mats_full = _workload_arrays(args.workload, 0, args.mu)
        if w_full.count < 2:
            raise SystemExit("--scaling strong needs a batched workload")
        _, pst = ext.factor_batched([torch.from_numpy(a) for a in mats_full], list(w_full.mu), list(w_full.tau),
                                    iters=w_full.iters, seeds=list(w_full.seeds), sweeps=w_full.sweeps,
                                    hs=[w_full.weights(b) for b in range(w_full.count)] if w_full.weighted else None,
                                    grid=args.grid, cluster=args.cluster, block=args.block, plan_only=True)
        plan = {"grid": pst["group"], "cluster": pst["cluster"], "block": pst["block"]}
        w, idx = dist.slice_workload(w_full, ws, rank)
        mats = [mats_full[i] for i in idx]
    else:
        w, mats = _workload_arrays(args.workload, rank, args.mu)
    As = [torch.from_numpy(a).to(dev) for a in mats]
    host_As = [torch.from_numpy(a).pin_memory() for a in mats]
    k_total = sum(ext.rank(a.shape[0], a.shape[1], mu) for a, mu in zip(mats, w.mu))
    stream = torch.cuda.current_stream(dev)

    hw = [torch.from_numpy(w.weights(b)).to(dev) for b in range(w.count)] if w.weighted else None

    # units of one step: component fits, i.e. extraction components plus refinement visits
    fits = k_total * (1 + w.sweeps)

    def step(inputs):
        if strong:
            res, st = ext.factor_batched(inputs, w.mu, w.tau, iters=w.iters, seeds=list(w.seeds), hs=hw,
                                         lams=[w.lam] * w.count if w.weighted else None, sweeps=w.sweeps,
                                         grid=plan["grid"], cluster=plan["cluster"], block=plan["block"])
            assert all(x == 0 for x in st), st
            return res, res[0].stats
        if w.weighted and not w.sweeps and w.count == 1:
            f = ext.factor_weighted(inputs[0], hw[0], w.mu[0], w.tau[0], lam=w.lam, iters=w.iters, seed=w.seeds[0])
            return [f], f.stats
        if w.count == 1:
            f = ext.factor(inputs[0], w.mu[0], w.tau[0], iters=w.iters, seed=w.seeds[0],
                           grid=args.grid, pending=args.pending, sweeps=w.sweeps,
                           h=hw[0] if w.weighted else None, lam=w.lam, cluster=args.cluster, block=args.block)
            return [f], f.stats
        res, st = ext.factor_batched(inputs, w.mu, w.tau, iters=w.iters, seeds=list(w.seeds), hs=hw,
                                     lams=[w.lam] * w.count if w.weighted else None, sweeps=w.sweeps,
                                     grid=args.grid, cluster=args.cluster, block=args.block)
        assert all(s == 0 for s in st), st
        return res, res[0].stats

    def barrier():
        dist.barrier(dev)

    def max_over_ranks(x: float) -> float:
        return dist.max_over_ranks(x, dev)

    for _ in range(args.warmup):
        step(As)

    # ---- device-resident inputs
    als_ms, alg_bytes, read_bytes, launches = [], [], [], 0
    barrier()
    with ClockSampler(dev.index) as clk:
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            res, st = step(As)
            als_ms.append(st["als_ms"])
            alg_bytes.append(st["alg_bytes"])
            read_bytes.append(st["read_bytes"])
            launches += st["launches"]
        ev1.record(stream)
        barrier()
    t_ms = max_over_ranks(ev0.elapsed_time(ev1))
    clocks = clk.summary()
    value = dist.throughput(dist.sum_over_ranks(fits * args.steps, dev), t_ms)

    # ---- end to end through the public API with pinned host buffers
    step(host_As)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d = d2h = 0
    for _ in range(args.steps):
        res, _ = step(host_As)
        h2d = sum(a.numel() * 4 for a in host_As)
        d2h = sum(r.B.numel() + r.C.numel() + r.D.numel() * 4 + (r.energy.numel() * 8 if r.energy is not None else 0)
                  + (r.sweep_energy.numel() * 8 if r.sweep_energy is not None else 0) for r in res)
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = dist.throughput(dist.sum_over_ranks(fits * args.steps, dev), e2e_ms)

    peak, peak_kind = _peaks()
    mean_als = statistics.mean(als_ms)
    mean_bytes = statistics.mean(alg_bytes)
    achieved = mean_bytes / (mean_als / 1000.0) / 1e9
    traffic = _ncu_traffic(w.name)
    energy_final = float(res[0].energy[-1].item()) if res[0].energy is not None else None
    if res[0].sweep_energy is not None:
        energy_final = float(res[0].sweep_energy[-1].item())
    energy_curve = None
    if w.mu_sweep and res[0].energy is not None:
        # the start vector of component i depends only on (seed, i), so the first k
        # components of the largest-mu run are the run at smaller mu (prefix property)
        e = res[0].energy.cpu()
        m0, n0 = w.shapes[0]
        energy_curve = {str(mu): float(e[ext.rank(m0, n0, mu) - 1].item()) for mu in w.mu_sweep}
    if st.get("cluster", 1) > 1:
        kernel = "externd::als2_kernel (clusters of %d)" % st["cluster"]
    else:   # the build of the ALS machinery the plan's block size selects
        space = {256: "externd_nt256", 1024: "externd_nt1024"}.get(st["block"], "externd")
        kernel = f"{space}::als_kernel ({st['block']} threads per CTA)"
    parallelism = (f"batch split over {ws} GPUs (contiguous slices, plan of the whole batch: {plan['grid']} CTAs per "
                   f"matrix, clusters of {plan['cluster']}, {plan['block'] or 'automatic'} threads per CTA)" if strong
                   else f"replicas x{ws} (independent matrices per rank)")
    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": t_ms / args.steps, "higher_is_better": True,
           "scaling": "strong" if strong else "weak",
           "vs_baseline": None, "dtype": "f32", "data": "synthetic",
           "config": _config(w_full if strong else w,
                             {"k": k_total, "sweeps": w.sweeps, "grid": st["grid"], "group": st["group"],
                              "block": st["block"], "cluster": st.get("cluster", 1),
                              "pending": st["pending"], "vec": [st["vec_v"], st["vec_u"]],
                              "parallelism": parallelism}),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak, "traffic": traffic,
                        "kernel": kernel, "peak_kind": f"{peak_kind} copy bandwidth",
                        "alg_bytes_per_launch": mean_bytes, "kernel_ms": mean_als,
                        "bytes_read_per_launch": statistics.mean(read_bytes),
                        "note": "alg bytes: direct-evaluation count per component; the kernel reads only "
                                "the rows/columns of changed trits (bytes_read_per_launch)"},
           "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
           "gpu_launches": launches,
           "clocks": clocks,
           "energy": energy_final,
           "energy_vs_mu": energy_curve,
           "components_per_step": dist.sum_over_ranks(k_total, dev),
           "fits_per_step": dist.sum_over_ranks(fits, dev),
           "wall_s_per_matrix": (t_ms / 1000.0) / args.steps / w.count}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = time_oracle(w, mats, budget_s=args.ref_budget)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# Inference with the factors (§2.6): y = B diag(D) C x on the headline's factors
# ---------------------------------------------------------------------------

def run_matvec(args):
    """Time externd_matvec on the factors of the workload's matrix 0 (factorization untimed).

    Before every timed call a 1 GiB buffer is overwritten (L2 is 126 MB), so every call
    streams the packed factors from HBM; each call is timed alone with CUDA events."""
    import torch
    import ternary_rank_weight_b200 as ext
    from ternary_rank_weight_b200 import dist

    ws, rank, local = _dist()
    dev = _init_nccl(ws, local)
    w, mats = _workload_arrays(args.workload, rank, args.mu)
    f = ext.factor(torch.from_numpy(mats[0]).to(dev), w.mu[0], w.tau[0], iters=w.iters, seed=w.seeds[0])
    Bt = ext.inference_layout(f)
    batch = args.batch
    X = torch.randn((batch, f.n), device=dev, dtype=torch.float32, generator=torch.Generator(device=dev).manual_seed(7))
    Y = torch.empty((batch, f.m), device=dev, dtype=torch.float32)
    Z = torch.empty((min(batch, 8), f.k), device=dev, dtype=torch.float32)
    # 1 GiB overwritten before every call: longer on the device (~160 us) than the host
    # needs to enqueue the next call, so the events bracket device work only
    flush = torch.empty(1024 * 1024 * 1024 // 4, device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        ext.matvec(Bt, f.D, f.C, f.m, f.n, X, out=Y, z_work=Z)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(dev.index) as clk:
        for e0, e1 in ev:
            flush.fill_(1.0)
            e0.record(stream)
            ext.matvec(Bt, f.D, f.C, f.m, f.n, X, out=Y, z_work=Z)
            e1.record(stream)
        torch.cuda.synchronize(dev)
    times = [e0.elapsed_time(e1) for e0, e1 in ev]
    dist.barrier(dev)
    t_ms = dist.max_over_ranks(statistics.median(times), dev)
    factor_bytes = Bt.numel() + f.C.numel() + 4 * f.k
    vec_bytes = 4 * batch * (f.n + f.m) + 2 * 4 * min(batch, 8) * f.k * ((batch + 7) // 8)
    alg = factor_bytes + vec_bytes
    peak, peak_kind = _peaks()
    achieved = alg / (t_ms / 1000.0) / 1e9
    # the dense fp16 weight the factors replace, for context: m n 2 bytes at the same peak
    dense_us = 2.0 * f.m * f.n / (peak * 1e9) * 1e6
    out = {"op": "matvec", "metric": "factored ternary matvec y = B diag(D) C x (2-bit trits)",
           "value": 1000.0 / t_ms * dist.sum_over_ranks(1, dev), "unit": "matvec/s", "n_gpus": ws,
           "steps": args.steps, "warmup": args.warmup, "us_per_call": t_ms * 1000.0, "higher_is_better": True,
           "dtype": "f32", "data": "synthetic",
           "config": {"workload": w.name, "m": f.m, "n": f.n, "k": f.k, "batch": batch,
                      "l2": "1 GiB buffer overwritten before every timed call"},
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                        "bytes_per_call": alg, "factor_bytes": factor_bytes, "peak_kind": f"{peak_kind} copy bandwidth"},
           "dense_fp16_floor_us": dense_us, "gpu_launches_per_call": 2 * ((batch + 7) // 8),
           "clocks": clk.summary()}
    if rank == 0 and not args.no_cpu_baseline:
        from oracle import externd_oracle as ora
        Bh, Ch = f.trits()
        Dh = f.D.cpu().numpy().astype(np.float64)
        Xh = X.cpu().numpy().astype(np.float64).T
        t0 = time.perf_counter()
        reps = 0
        while time.perf_counter() - t0 < 5.0:
            ora.factored_matvec(Bh, Dh, Ch, Xh)
            reps += 1
        dt = (time.perf_counter() - t0) / reps
        out["cpu_baseline"] = {"value": 1.0 / dt, "unit": "matvec/s", "cores": _oracle_threads(), "kind": "oracle",
                               "sample": f"{reps} calls of numpy fp64 B (D (C X)) on dense int8 trits, batch {batch}"}
    if rank == 0:
        print(json.dumps(out), flush=True)
    _fini_nccl(ws)
    return 0


# ---------------------------------------------------------------------------
# Batched block ALS (§2.4) on the workload's matrix 0
# ---------------------------------------------------------------------------

FP64_NOMINAL_TFLOPS = 37.0       # B200 fp64 (CUDA cores and DMMA), NVIDIA's published per-GPU figure
BF16_NOMINAL_TFLOPS = 2250.0     # dense bf16, the recipe's nominal figure


def _fp64_peak():
    """fp64 roofline denominator: the measured bf16 GEMM peak times the nominal fp64 / bf16 ratio."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]) * FP64_NOMINAL_TFLOPS / BF16_NOMINAL_TFLOPS, "measured bf16 x nominal fp64/bf16"
    except Exception:
        return 1590.0 * FP64_NOMINAL_TFLOPS / BF16_NOMINAL_TFLOPS, "fallback bf16 x nominal fp64/bf16"


def run_block(args):
    """Time externd_factor_block (device-resident A) and, end to end, with A uploaded from pinned
    host memory and the factors downloaded inside the timed region."""
    import torch
    import ternary_rank_weight_b200 as ext
    from ternary_rank_weight_b200 import dist

    ws, rank, local = _dist()
    dev = _init_nccl(ws, local)
    w, mats = _workload_arrays(args.workload, rank, args.mu)
    A = torch.from_numpy(mats[0]).to(dev)
    Ah = torch.from_numpy(mats[0]).pin_memory()
    mu, tau, seed = w.mu[0], w.tau[0], w.seeds[0]
    m, n = mats[0].shape
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        f = ext.factor_block(A, mu, tau, iters=w.iters, seed=seed)
    dist.barrier(dev)
    # one event pair per call: the call issues thousands of small launches, so a host stall shows up as
    # device idle time in that call alone; the median over the steps is reported (the mean beside it)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(dev.index) as clk:
        for e0, e1 in evs:
            e0.record(stream)
            f = ext.factor_block(A, mu, tau, iters=w.iters, seed=seed)
            e1.record(stream)
        dist.barrier(dev)
    per = [a.elapsed_time(b) for a, b in evs]
    t_ms = dist.max_over_ranks(statistics.median(per), dev)
    t_mean = dist.max_over_ranks(statistics.mean(per), dev)
    k, b = f.k, f.stats["group"]
    # end to end: upload, factor, download
    h2d = Ah.numel() * 4
    d2h = f.B.numel() + f.C.numel() + f.D.numel() * 4 + f.energy.numel() * 8
    per_e2e = []
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g = ext.factor_block(Ah.to(dev, non_blocking=True), mu, tau, iters=w.iters, seed=seed)
        for t in (g.B, g.C, g.D, g.energy):
            t.cpu()
        e1.record(stream)
        e1.synchronize()
        per_e2e.append(e0.elapsed_time(e1))
    dist.barrier(dev)
    e2e_ms = dist.max_over_ranks(statistics.median(per_e2e), dev)
    # fp64 GEMM flops per call: per block and iteration U^T U, R^T U, V^T V, R V; per block the
    # final U^T U and the deflation
    flops = 0.0
    for s0 in range(0, k, b):
        nb = min(b, k - s0)
        flops += w.iters * 2.0 * nb * (nb * m + n * m + nb * n + m * n) + 2.0 * nb * (nb * m + m * n)
    peak, peak_kind = _fp64_peak()
    achieved = flops / (t_ms / 1000.0) / 1e12
    out = {"op": "block", "metric": "ternary components fitted/s, batched block ALS (§2.4)",
           "value": dist.sum_over_ranks(k, dev) / (t_ms / 1000.0), "unit": "components/s", "n_gpus": ws,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms, "ms_per_step_mean": t_mean,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": _config(w, {"k": k, "block": b, "timing": "median of the per-call CUDA-event times",
                                 "l2": "inputs larger than L2 (A and the fp64 residual); no flush"}),
           "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                        "frac": achieved / peak, "traffic": None, "kernel": "fp64 GEMMs (cuBLAS DGEMM)",
                        "peak_kind": peak_kind, "gemm_flops_per_call": flops,
                        "note": "achieved = the GEMMs' flops / the whole call's time (a lower bound for the GEMMs)"},
           "e2e": {"value": dist.sum_over_ranks(k, dev) / (e2e_ms / 1000.0), "unit": "components/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
           "gpu_launches": f.stats["launches"],
           "clocks": clk.summary(),
           "energy": float(f.energy[-1].item())}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        # the oracle's block_als on the first blocks of the same matrix (per-block cost is constant)
        from oracle import externd_oracle as ora
        t0 = time.perf_counter()
        nblk = 0
        while True:
            nblk += 1
            ora.block_als(mats[0], k=min(k, nblk * b), tau=tau, iters=w.iters, seed=seed)
            dt = time.perf_counter() - t0
            if dt > args.ref_budget / 2 or nblk * b >= k:
                break
            t0 = time.perf_counter()
        out["cpu_baseline"] = {"value": min(k, nblk * b) / dt, "unit": "components/s", "cores": _oracle_threads(),
                               "kind": "oracle",
                               "sample": f"first {min(k, nblk * b)} of {k} components ({nblk} block(s) of {b}) of "
                                         f"the {m}x{n} matrix, {dt:.1f} s, numpy fp64"}
    if rank == 0:
        print(json.dumps(out), flush=True)
    _fini_nccl(ws)
    return 0


def main():
    from ternary_rank_weight_b200.workloads import HEADLINE, WORKLOADS
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--all", action="store_true", help="one line per workload (reporting, not the driver's line)")
    ap.add_argument("--grid", type=int, default=0)
    ap.add_argument("--block", type=int, default=0,
                    help="threads per CTA of the one-CTA-per-stripe ALS kernel: 0 automatic, 256, 512 or 1024")
    ap.add_argument("--cluster", type=int, default=0,
                    help="ALS kernel: 0 automatic, 1 one CTA per stripe, 2/4/8/16 clustered with that cluster size")
    ap.add_argument("--scaling", choices=("weak", "strong"), default="weak",
                    help="N > 1: weak = each rank its own matrices; strong = one batch split over the ranks")
    ap.add_argument("--pending", type=int, default=0)
    ap.add_argument("--ref-budget", type=float, default=15.0, help="seconds of oracle work per sample")
    ap.add_argument("--mu", type=float, default=None, help="override mu (short runs for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", choices=("factor", "matvec", "block"), default="factor",
                    help="factor: the factorization (default); matvec: inference with the factors; "
                         "block: the batched block ALS of §2.4")
    ap.add_argument("--batch", type=int, default=1, help="input vectors per matvec call (--op matvec)")
    args = ap.parse_args()
    args.ref_budget = min(args.ref_budget, 150.0 / max(args.steps, 1))
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "matvec":
        return run_matvec(args)
    if args.op == "block":
        return run_block(args)
    if args.all:
        for name in WORKLOADS:
            args.workload = name
            run_ours(args)
        return 0
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
