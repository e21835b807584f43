"""Write the oracle's expected values for the full-size workloads (tests/golden/oracle_*.json).

This script calls only ``oracle/`` (the fp64 CPU implementation of greedy sequential
ALS, "ExTernD: Expanded-Rank Ternary Decomposition" §2.1-§2.3) and the seeded input
generators; no value comes from the CUDA library.  The full runs take tens of minutes
on a few host cores, which is why their results are stored instead of recomputed by
the GPU tests.

For every workload matrix it stores
* the energy E_i of §2.1 after component i, at i = 0, 64, 128, ... and the last i;
* the zero fraction of the factors (for the 4096 x 4096 run also at the prefixes
  k = mu * 4096 for mu = 1, 2, 3, 3.5: the first components of a run do not depend
  on k, so one run gives every mu);
* the explicit final energy, the number of components where the single-entry
  safeguard condition held (§7: the pages say the safeguard never activates);
* for the first PREFIX components: the scale d_i (fp64) and an 8-byte BLAKE2b digest
  of the int8 trits (u_i then v_i), which locate the first component where another
  implementation's trits differ.

The job "block_mlp_2560x6912" runs the §2.4 batched block ALS (oracle block_als at the
pages' default width) on the same matrix; its energy_index holds every 64th component,
i.e. the energy after each block of 256 is sampled several times.

Usage: python tests/golden/make_oracle_goldens.py [NAME ...]   (default: all)
"""
from __future__ import annotations

import hashlib
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import externd_oracle as ora  # noqa: E402
from ternary_rank_weight_b200.workloads import WORKLOADS  # noqa: E402

PREFIX = 512
EVERY = 64

# (golden name, workload name, matrix index in the workload)
JOBS = {
    "mlp_2560x6912": ("mlp_2560x6912_bf16_mu3_tau1.0", 0),
    "block_mlp_2560x6912": ("mlp_2560x6912_bf16_mu3_tau1.0", 0),   # §2.4 block ALS at the default width
    "llm_4096x4096": ("llm_4096x4096_mu3.5_tau0.7", 0),
    "attn_1536_b0_tau0.7": ("attn_16x1536x1536_mu2.5_tau_cycle", 0),
    "attn_1536_b1_tau1.0": ("attn_16x1536x1536_mu2.5_tau_cycle", 1),
    "attn_1536_b2_tau2.0": ("attn_16x1536x1536_mu2.5_tau_cycle", 2),
}


def trit_digest(u: np.ndarray, v: np.ndarray) -> str:
    """8-byte BLAKE2b digest of the component's int8 trits, u then v."""
    h = hashlib.blake2b(digest_size=8)
    h.update(np.ascontiguousarray(u, dtype=np.int8).tobytes())
    h.update(np.ascontiguousarray(v, dtype=np.int8).tobytes())
    return h.hexdigest()


def make(name: str) -> dict:
    wname, b = JOBS[name]
    w = WORKLOADS[wname]
    A = w.matrix(b)
    m, n = A.shape
    mu, tau, seed = w.mu[b], w.tau[b], w.seeds[b]
    k = ora.rank(m, n, mu)
    t0 = time.time()
    if name.startswith("block_"):
        ref = ora.block_als(A, k=k, tau=tau, iters=w.iters, seed=seed)
    else:
        ref = ora.greedy_als(A, k=k, tau=tau, iters=w.iters, seed=seed)
    secs = time.time() - t0
    idx = sorted(set(range(0, k, EVERY)) | {k - 1})
    out = {
        "_source": ("fp64 oracle (oracle/externd_oracle.py " + ("block_als" if name.startswith("block_") else "greedy_als")
                    + ") of 'ExTernD: Expanded-Rank Ternary Decomposition' " + ("§2.4 batched block ALS"
                    if name.startswith("block_") else "§2.1-§2.3 greedy sequential ALS")
                    + "; written by tests/golden/make_oracle_goldens.py"),
        "workload": wname, "matrix": b, "m": m, "n": n, "mu": mu, "tau": tau, "seed": seed, "iters": w.iters,
        "k": k,
        "energy_index": idx,
        "energy": [float(ref.energy[i]) for i in idx],
        "energy_final_explicit": float(ref.energy_final),
        "zero_fraction": float(ref.zero_fraction()),
        "safeguard_hits": int(ref.safeguard_hits),
        "prefix_d": [float(x) for x in ref.D[:PREFIX]],
        "prefix_digest": [trit_digest(ref.B[:, i], ref.C[i]) for i in range(min(PREFIX, k))],
        "oracle_seconds": round(secs, 1),
    }
    if w.mu_sweep:
        pts = []
        for mu2 in w.mu_sweep:
            k2 = ora.rank(m, n, mu2)
            pts.append({"mu": mu2, "k": k2, "energy": float(ref.energy[k2 - 1]),
                        "zero_fraction": float(ref.zero_fraction(k2))})
        out["mu_sweep"] = pts
    return out


def main(names):
    for name in names:
        path = os.path.join(HERE, f"oracle_{name}.json")
        res = make(name)
        with open(path, "w") as f:
            json.dump(res, f, indent=1)
            f.write("\n")
        print(f"{name}: k={res['k']} E={res['energy'][-1]:.6f} zf={res['zero_fraction']:.4f} "
              f"safeguard={res['safeguard_hits']} {res['oracle_seconds']} s", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:] or list(JOBS))
