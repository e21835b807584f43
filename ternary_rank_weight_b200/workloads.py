"""Seeded synthetic weight matrices shaped like the pages' LLM workloads.

This module only draws inputs.  It holds none of the factorization's arithmetic,
so both the CUDA path and the fp64 oracle can be fed from it without sharing any
method code.

ExTernD (Expanded-Rank Ternary Decomposition), §3 "Results": the pages factor
trained weight matrices of Gemma-4-E2B, Qwen3.5-4B and Granite-4.0-h-tiny, none
of which are available here.  These generators stand in for them:

* ``iid``      : A_rc = 0.02 * z_rc, z ~ N(0, 1).
* ``llm``      : A_rc = 0.02 * exp(0.5 * g_r) * z_rc (per-row log-normal scale,
                 sigma = 0.5), then ``outliers`` distinct columns (chosen without
                 replacement) are replaced by 10 * 0.02 * t_rc with t ~ Student-t
                 (nu = 4) and no row scale.
* ``bf16=True``: the fp32 matrix is rounded to bfloat16 (round to nearest, ties
                 to even) and held again as fp32.

All draws come from ``numpy.random.default_rng(seed)`` (PCG64) in a fixed order,
so a (recipe, shape, seed) triple always yields the same matrix.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bfloat16 (ties to even), returned as fp32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    # NaN/Inf keep their bits (none are produced by these generators).
    special = (bits & 0x7F800000) == 0x7F800000
    rounded = np.where(special, bits, rounded)
    return rounded.astype(np.uint32).view(np.float32).reshape(a.shape)


def iid_matrix(m: int, n: int, seed: int, std: float = 0.02) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (std * rng.standard_normal((m, n))).astype(np.float32)


def llm_matrix(m: int, n: int, seed: int, outliers: int = 8, std: float = 0.02,
               row_sigma: float = 0.5, outlier_scale: float = 10.0, nu: float = 4.0,
               bf16: bool = False) -> np.ndarray:
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((m, n))
    g = rng.standard_normal(m)
    a = std * np.exp(row_sigma * g)[:, None] * z
    n_out = min(outliers, n)
    if n_out > 0:
        cols = rng.choice(n, size=n_out, replace=False)
        t = rng.standard_t(nu, size=(m, n_out))
        a[:, cols] = outlier_scale * std * t
    a = a.astype(np.float32)
    if bf16:
        a = round_to_bf16(a)
    return a


def importance_weights(n: int, seed: int, sigma: float = 1.5, hot: int = 8, hot_scale: float = 30.0) -> np.ndarray:
    """Per-input-channel second moments standing in for a llama.cpp importance matrix
    (the pages' §2.5 input, not available here): log-normal with spread ``sigma`` and
    ``hot`` distinct channels scaled by ``hot_scale`` (activation outlier channels)."""
    rng = np.random.default_rng(seed)
    h = np.exp(sigma * rng.standard_normal(n))
    k = min(hot, n)
    if k > 0:
        h[rng.choice(n, size=k, replace=False)] *= hot_scale
    return h.astype(np.float32)


@dataclass(frozen=True)
class Workload:
    """One named factorization job: matrices plus the method's parameters."""
    name: str
    shapes: tuple            # ((m, n), ...) one entry per matrix
    seeds: tuple
    mu: tuple                # per matrix
    tau: tuple               # per matrix
    recipe: str = "llm"
    outliers: int = 8
    bf16: bool = False
    iters: int = 15
    mu_sweep: tuple = field(default=())   # extra mu read off one run (prefix property)
    weighted: bool = False                # §2.5 objective with importance_weights(n, seed)
    lam: float = 0.0
    sweeps: int = 0                       # §2.4 refinement sweeps after extraction

    def weights(self, b: int) -> np.ndarray:
        return importance_weights(self.shapes[b][1], self.seeds[b])

    def matrix(self, b: int) -> np.ndarray:
        m, n = self.shapes[b]
        if self.recipe == "iid":
            return iid_matrix(m, n, self.seeds[b])
        return llm_matrix(m, n, self.seeds[b], outliers=self.outliers, bf16=self.bf16)

    def matrices(self):
        return [self.matrix(b) for b in range(len(self.shapes))]

    @property
    def count(self) -> int:
        return len(self.shapes)


# The five workloads.  Names state what they are.
WORKLOADS = {
    "iid_256x256_mu2_tau0.7": Workload(
        "iid_256x256_mu2_tau0.7", ((256, 256),), (0,), (2.0,), (0.7,), recipe="iid"),
    "llm_1024x1024_mu2_tau0.7": Workload(
        "llm_1024x1024_mu2_tau0.7", ((1024, 1024),), (1,), (2.0,), (0.7,)),
    "mlp_2560x6912_bf16_mu3_tau1.0": Workload(
        "mlp_2560x6912_bf16_mu3_tau1.0", ((2560, 6912),), (2,), (3.0,), (1.0,), bf16=True),
    "attn_16x1536x1536_mu2.5_tau_cycle": Workload(
        "attn_16x1536x1536_mu2.5_tau_cycle", tuple((1536, 1536) for _ in range(16)),
        tuple(range(100, 116)), tuple(2.5 for _ in range(16)),
        tuple((0.7, 1.0, 2.0)[b % 3] for b in range(16))),
    "attn_16x1536x1536_mu2.5_tau_cycle_weighted_sweep1": Workload(
        "attn_16x1536x1536_mu2.5_tau_cycle_weighted_sweep1", tuple((1536, 1536) for _ in range(16)),
        tuple(range(100, 116)), tuple(2.5 for _ in range(16)),
        tuple((0.7, 1.0, 2.0)[b % 3] for b in range(16)), weighted=True, sweeps=1),
    "mlp_2560x6912_bf16_mu3_tau1.0_weighted": Workload(
        "mlp_2560x6912_bf16_mu3_tau1.0_weighted", ((2560, 6912),), (2,), (3.0,), (1.0,), bf16=True, weighted=True),
    "mlp_2560x6912_bf16_mu3_tau1.0_sweep1": Workload(
        "mlp_2560x6912_bf16_mu3_tau1.0_sweep1", ((2560, 6912),), (2,), (3.0,), (1.0,), bf16=True, sweeps=1),
    "llm_1024x1024_mu2_tau0.7_sweep10": Workload(
        "llm_1024x1024_mu2_tau0.7_sweep10", ((1024, 1024),), (1,), (2.0,), (0.7,), sweeps=10),
    "llm_4096x4096_mu3.5_tau0.7": Workload(
        "llm_4096x4096_mu3.5_tau0.7", ((4096, 4096),), (4,), (3.5,), (0.7,), outliers=32,
        mu_sweep=(1.0, 2.0, 3.0, 3.5)),
}

HEADLINE = "mlp_2560x6912_bf16_mu3_tau1.0"
SMALL = "iid_256x256_mu2_tau0.7"
