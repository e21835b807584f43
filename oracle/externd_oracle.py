"""fp64 CPU oracle for ExTernD greedy sequential ternary ALS.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, links or runs
this module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` do.  It shares no code with the CUDA library.

Source: "ExTernD: Expanded-Rank Ternary Decomposition" (academ.us HTML of
arXiv 2607.13511), cited below by section and display equation:

* §2.1 display equation: A ~ B diag(D) C with B in {-1,0,1}^{m x k},
  C in {-1,0,1}^{k x n}, D in R^k; energy E = 1 - ||A - Ahat||_F^2 / ||A||_F^2.
* §2.2 display equation: T_tau(u)_i = sign(u_i) * 1[|u_i| > tau * (1/m) sum_j |u_j|],
  keeping the single largest entry when the result would be all-zero; and the
  optimal ternary projection (sort |u|, keep the prefix s* maximizing
  (1/sqrt(s)) sum_{i<=s} |u|_(i)).
* §2.3 steps 1-3: R <- A; for each component: 15 alternating fits
  v <- T_tau(R^T u), u <- T_tau(R v); scale d = u^T R v / (||u||^2 ||v||^2);
  deflate R <- R - d u v^T; store B[:, i] = u, C[i, :] = v^T.
* §2.5: importance-weighted ALS minimizes sum_ij h~_j (A - Ahat)^2_ij with
  h~ = h / max(h) + lambda; the U-step targets W = R diag(h~), the V-step the plain
  residual R (h~ cancels there), the scale solves the weighted normal equation.
* §2.4 "Refinement sweeps": after extraction, revisit each block (add its
  contribution back to R, re-run the fit, re-deflate); here blocks of one
  component.  Readings: the refit starts from the stored u and runs the same
  alternation as extraction; it replaces the stored component only if its
  least-squares decrease of the added-back residual is at least that of the
  stored pair with its own least-squares scale (otherwise the stored pair stays,
  rescaled), which makes every visit non-increasing in the residual, as the
  pages report the sweeps to be.
* §2.4 "Batched block ALS": blocks of b components (default 256, capped at
  floor(min(m, n)/8)); V <- T_tau([(U^T U + eps I)^-1 U^T R]^T),
  U <- T_tau(R V (V^T V + eps I)^-1) column-wise, then the scales solve
  [(U^T U) o (V^T V)] d = diag(U^T R V) and R <- R - U diag(d) V^T.  Readings: eps
  (unspecified) = 1e-6 x the Gram matrix's mean diagonal; the start block holds the
  sequential method's start vectors of its components; the alternation runs `iters`
  times like the sequential fit.
* §2.6 Cost model: inference computes y = B (diag(D) (C x)); mask+sign packing
  stores one zero/nonzero mask bit per element plus one sign bit per nonzero,
  and Eq. (1): bpw_eff = mu (m + n) / max(m, n) * (2 - sparsity).

Everything is plain numpy in float64, written in the pages' order.  Readings
where the pages are silent (each one is listed with its reason in the design
notes of the repository):

* start vector: the pages start the alternation from some u without saying
  which; here u^(0) = T_tau(z) with z ~ N(0, 1)^m drawn per component from the
  counter-based generator Philox4x32-10 (Salmon et al., "Parallel random
  numbers: as easy as 1, 2, 3", SC'11) keyed by the seed, followed by the
  Box-Muller transform (cosine branch).
* "15 iterations" = 15 (V-step, U-step) pairs; the scale uses the final u and
  the v of the same pair.
* the mean inside T_tau runs over the vector's own length (n for the V-step,
  m for the U-step); the comparison is strict.
* all-zero fallback: the lowest index among the entries of largest magnitude
  keeps its sign; an identically zero vector yields +1 at index 0.
* k = round-half-away-from-zero(mu * min(m, n)).
* if u^T R v = 0 the component gets d = 0 and R is unchanged.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ----------------------------------------------------------------------------
# Inner rank (§2.1: k = mu * min(m, n))
# ----------------------------------------------------------------------------


def rank(m: int, n: int, mu: float) -> int:
    """k = mu * min(m, n) rounded half away from zero; -1 if that is below 1."""
    if m < 1 or n < 1 or not math.isfinite(mu):
        return -1
    x = mu * min(m, n)
    k = int(math.floor(abs(x) + 0.5)) * (1 if x >= 0 else -1)
    return k if k >= 1 else -1


# ----------------------------------------------------------------------------
# Start vectors: Philox4x32-10 + Box-Muller (reading of §2.3, which is silent)
# ----------------------------------------------------------------------------

_MASK32 = np.uint64(0xFFFFFFFF)
_PHILOX_M0 = np.uint64(0xD2511F53)
_PHILOX_M1 = np.uint64(0xCD9E8D57)
_PHILOX_W0 = np.uint64(0x9E3779B9)
_PHILOX_W1 = np.uint64(0xBB67AE85)
INIT_STREAM = 1            # third counter word for start vectors
TWO_PI = 6.283185307179586  # nearest double to 2*pi


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds, as defined by Salmon et al. (SC'11).

    Each round multiplies counter words 0 and 2 by the two Philox multipliers,
    splits the 64-bit products into high and low halves and mixes them with the
    other two words and the key; the key is bumped by the Weyl constants before
    every round but the first.  Inputs are integer arrays holding 32-bit values.
    """
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK32 for c in (c0, c1, c2, c3))
    k0 = np.asarray(k0, dtype=np.uint64) & _MASK32
    k1 = np.asarray(k1, dtype=np.uint64) & _MASK32
    for r in range(10):
        if r > 0:
            k0 = (k0 + _PHILOX_W0) & _MASK32
            k1 = (k1 + _PHILOX_W1) & _MASK32
        p0 = _PHILOX_M0 * c0
        p1 = _PHILOX_M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0), lo1, (hi0 ^ c3 ^ k1), lo0
    return c0, c1, c2, c3


def _uniform53(hi, lo):
    """(hi:lo) 64-bit word -> double in (0, 1): top 53 bits, offset by half a step."""
    w = (hi << np.uint64(32)) | lo
    return ((w >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def start_normals(seed: int, comp: int, m: int) -> np.ndarray:
    """z_j ~ N(0, 1), j < m, for component ``comp``: counter (j, comp, 1, 0), key = seed."""
    j = np.arange(m, dtype=np.uint64)
    x0, x1, x2, x3 = philox4x32_10(j, np.uint64(comp), np.uint64(INIT_STREAM), np.uint64(0),
                                   np.uint64(seed & 0xFFFFFFFF), np.uint64(seed >> 32))
    u1 = _uniform53(x1, x0)
    u2 = _uniform53(x3, x2)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(TWO_PI * u2)


# ----------------------------------------------------------------------------
# §2.2 ternarization operator and optimal ternary projection
# ----------------------------------------------------------------------------


def ternarize(x: np.ndarray, tau: float):
    """T_tau(x) of §2.2.  Returns (trits int8, threshold, fallback_used)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    thr = tau * a.sum() / x.shape[0]
    out = np.where(a > thr, np.where(x < 0, -1, 1), 0).astype(np.int8)
    fallback = False
    if not out.any():
        fallback = True
        j = int(np.argmax(a))              # first index among the largest magnitudes
        out[j] = -1 if x[j] < 0 else 1     # x == 0 everywhere -> +1 at index 0
    return out, thr, fallback


def relative_margin(x: np.ndarray, thr: float) -> float:
    """min_c | |x_c| - thr | / thr : how close the vector came to a threshold tie."""
    if thr <= 0:
        return math.inf
    return float(np.min(np.abs(np.abs(np.asarray(x, dtype=np.float64)) - thr)) / thr)


def optimal_ternary_projection(u: np.ndarray):
    """argmin_{t, alpha} ||u - alpha t||_2 over ternary t (§2.2 closed form).

    Sort |u| descending, keep the prefix length s* that maximizes
    (1/sqrt(s)) * sum_{i<=s} |u|_(i); t = sign(u) on that prefix, alpha = mean of
    the kept magnitudes.  Returns (t int8, alpha, s*).
    """
    u = np.asarray(u, dtype=np.float64)
    order = np.argsort(-np.abs(u), kind="stable")
    csum = np.cumsum(np.abs(u)[order])
    s_range = np.arange(1, u.shape[0] + 1, dtype=np.float64)
    score = csum / np.sqrt(s_range)
    s_star = int(np.argmax(score)) + 1
    t = np.zeros(u.shape[0], dtype=np.int8)
    keep = order[:s_star]
    t[keep] = np.where(u[keep] < 0, -1, 1)
    alpha = csum[s_star - 1] / s_star
    return t, alpha, s_star


# ----------------------------------------------------------------------------
# §2.3 greedy sequential ALS
# ----------------------------------------------------------------------------


def ls_scale(R: np.ndarray, u: np.ndarray, v: np.ndarray) -> float:
    """§2.3 step 2: d = u^T R v / (||u||^2 ||v||^2); 0 when u^T R v = 0."""
    u = np.asarray(u, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    p = float(u @ (R @ v))
    if p == 0.0:
        return 0.0
    return p / (float(u @ u) * float(v @ v))


def half_step(R: np.ndarray, trits_in: np.ndarray, tau: float, transpose: bool):
    """One half of §2.3 step 1 on a given residual.

    transpose=True : x = R^T u, v = T_tau(x)   (V-step, input length m, output n)
    transpose=False: y = R v,   u = T_tau(y)   (U-step, input length n, output m)
    Returns (pre-threshold vector, threshold, output trits, fallback_used).
    """
    R = np.asarray(R, dtype=np.float64)
    w = np.asarray(trits_in, dtype=np.float64)
    pre = R.T @ w if transpose else R @ w
    out, thr, fb = ternarize(pre, tau)
    return pre, thr, out, fb


@dataclass
class ComponentFit:
    u: np.ndarray          # int8, m
    v: np.ndarray          # int8, n
    d: float
    p: float               # u^T R v
    decrease: float        # ||R||^2 - ||R - d u v^T||^2 = p^2 / (nnz u * nnz v)
    min_margin: float      # closest approach of any half-step to a threshold tie
    u_first: np.ndarray    # start trits


def fit_component(R: np.ndarray, u0: np.ndarray, tau: float, iters: int) -> ComponentFit:
    """§2.3 steps 1-2 for one component, from start trits u0, on residual R (fp64)."""
    u = np.asarray(u0, dtype=np.int8)
    v = None
    y = None
    margin = math.inf
    for _ in range(iters):
        x = R.T @ u.astype(np.float64)               # V-step: x = R^T u
        v, tv, _ = ternarize(x, tau)
        margin = min(margin, relative_margin(x, tv))
        y = R @ v.astype(np.float64)                 # U-step: y = R v
        u, tu, _ = ternarize(y, tau)
        margin = min(margin, relative_margin(y, tu))
    p = float(u.astype(np.float64) @ y)              # u^T R v with the final pair
    nu = int(np.count_nonzero(u))
    nv = int(np.count_nonzero(v))
    d = 0.0 if p == 0.0 else p / (nu * nv)
    return ComponentFit(u=u, v=v, d=d, p=p, decrease=(p * p) / (nu * nv), min_margin=margin,
                        u_first=np.asarray(u0, dtype=np.int8))


@dataclass
class Factorization:
    B: np.ndarray              # m x k int8
    C: np.ndarray              # k x n int8
    D: np.ndarray              # k float64
    energy: np.ndarray         # k float64, incremental: 1 - ||R_i||^2 / ||A||^2
    energy_final: float        # explicit 1 - ||A - Ahat||^2 / ||A||^2 at the end
    norm_a2: float
    margins: np.ndarray        # per component min relative threshold margin
    safeguard_hits: int        # components whose decrease fell below the single-entry bound ||R||^2 / (m n)
    residual_norms: np.ndarray = field(default=None)  # ||R_i||^2 explicit, per component

    @property
    def k(self) -> int:
        return self.D.shape[0]

    def zero_fraction(self, upto: int | None = None) -> float:
        kk = self.k if upto is None else upto
        zb = np.count_nonzero(self.B[:, :kk] == 0)
        zc = np.count_nonzero(self.C[:kk, :] == 0)
        return (zb + zc) / ((self.B.shape[0] + self.C.shape[1]) * kk)


def greedy_als(A: np.ndarray, k: int, tau: float, iters: int = 15, seed: int = 0,
               track_residual: bool = False) -> Factorization:
    """§2.3: greedy sequential ALS with deflation, in fp64."""
    R = np.array(A, dtype=np.float64, copy=True)       # R <- A
    m, n = R.shape
    norm_a2 = float(np.sum(R * R))
    if norm_a2 == 0.0:
        raise ValueError("||A||_F = 0: energy is undefined")
    B = np.zeros((m, k), dtype=np.int8)
    C = np.zeros((k, n), dtype=np.int8)
    D = np.zeros(k, dtype=np.float64)
    energy = np.zeros(k, dtype=np.float64)
    margins = np.zeros(k, dtype=np.float64)
    res = np.zeros(k, dtype=np.float64) if track_residual else None
    r2 = norm_a2
    hits = 0
    for i in range(k):
        u0, _, _ = ternarize(start_normals(seed, i, m), tau)
        fit = fit_component(R, u0, tau, iters)
        # §7 "Monotone residual decrease and convergence": a single-entry component
        # (u = e_r, v = e_c at the largest |R_rc|) removes max R_rc^2 >= ||R||^2 / (m n),
        # the single-entry bound behind the geometric rate in m n; the safeguard steps in
        # when the ALS decrease falls below that bound.  Count those components (the
        # pages say it never happens in practice); no substitution is made.
        if fit.decrease < float(np.sum(R * R)) / (m * n):
            hits += 1
        if fit.d != 0.0:
            R -= fit.d * np.outer(fit.u.astype(np.float64), fit.v.astype(np.float64))
        r2 -= fit.decrease
        B[:, i] = fit.u
        C[i, :] = fit.v
        D[i] = fit.d
        energy[i] = 1.0 - r2 / norm_a2
        margins[i] = fit.min_margin
        if track_residual:
            res[i] = float(np.sum(R * R))
    e_final = 1.0 - float(np.sum(R * R)) / norm_a2
    return Factorization(B=B, C=C, D=D, energy=energy, energy_final=e_final, norm_a2=norm_a2,
                         margins=margins, safeguard_hits=hits, residual_norms=res)


# ----------------------------------------------------------------------------
# §2.4 batched block ALS with decorrelated targets
# ----------------------------------------------------------------------------

BLOCK_EPS_REL = 1e-6   # reading: the ridge epsilon, unspecified on the pages, is 1e-6 x the mean
                       # diagonal of the Gram matrix it regularizes (nnz of the block's vectors)


def block_width(m: int, n: int, b: int = 256) -> int:
    """§2.4: blocks of b components (default 256), capped at floor(min(m, n) / 8), at least 1."""
    return max(1, min(int(b), min(m, n) // 8))


def ternarize_columns(X: np.ndarray, tau: float) -> np.ndarray:
    """T_tau of §2.2 applied to every column of X on its own (mean and fallback per column)."""
    X = np.asarray(X, dtype=np.float64)
    out = np.zeros(X.shape, dtype=np.int8)
    for j in range(X.shape[1]):
        out[:, j], _, _ = ternarize(X[:, j], tau)
    return out


def _ridge(G: np.ndarray) -> np.ndarray:
    eps = BLOCK_EPS_REL * float(np.mean(np.diag(G)))
    return G + eps * np.eye(G.shape[0])


def block_scales(R: np.ndarray, U: np.ndarray, V: np.ndarray) -> np.ndarray:
    """§2.4 joint scale solve: [(U^T U) o (V^T V)] d = diag(U^T R V) (the least-squares scales
    of the block for fixed trits).  A singular system (repeated components) takes the
    minimum-norm solution (reading: the pages say "solved jointly and exactly")."""
    U = np.asarray(U, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    H = (U.T @ U) * (V.T @ V)
    rhs = np.einsum("rj,rc,cj->j", U, np.asarray(R, dtype=np.float64), V)
    d, *_ = np.linalg.lstsq(H, rhs, rcond=None)
    return d


def block_fit(R: np.ndarray, U0: np.ndarray, tau: float, iters: int):
    """§2.4 block fit from start trits U0 (m x b): `iters` times
    V <- T_tau([(U^T U + eps I)^-1 U^T R]^T), U <- T_tau(R V (V^T V + eps I)^-1), column-wise,
    then the joint scales.  Returns (U int8 m x b, V int8 n x b, d)."""
    R = np.asarray(R, dtype=np.float64)
    U = np.asarray(U0, dtype=np.float64)
    V = None
    for _ in range(iters):
        Gu = U.T @ U
        V = ternarize_columns(np.linalg.solve(_ridge(Gu), U.T @ R).T, tau).astype(np.float64)
        Gv = V.T @ V
        U = ternarize_columns(np.linalg.solve(_ridge(Gv), (R @ V).T).T, tau).astype(np.float64)
    d = block_scales(R, U, V)
    return U.astype(np.int8), V.astype(np.int8), d


def block_als(A: np.ndarray, k: int, tau: float, iters: int = 15, seed: int = 0, b: int | None = None) -> Factorization:
    """§2.4 batched block ALS: components in blocks of b (the last one shorter), each block
    fitted by block_fit from the start vectors of its components (those of greedy_als, so
    that b = 1 is the sequential method), then R <- R - U diag(d) V^T; deflation across
    blocks is sequential.  energy[i] is the energy after the block holding component i."""
    R = np.array(A, dtype=np.float64, copy=True)
    m, n = R.shape
    norm_a2 = float(np.sum(R * R))
    if norm_a2 == 0.0:
        raise ValueError("||A||_F = 0: energy is undefined")
    bw = block_width(m, n) if b is None else int(b)
    B = np.zeros((m, k), dtype=np.int8)
    C = np.zeros((k, n), dtype=np.int8)
    D = np.zeros(k, dtype=np.float64)
    energy = np.zeros(k, dtype=np.float64)
    for s0 in range(0, k, bw):
        nb = min(bw, k - s0)
        U0 = np.stack([ternarize(start_normals(seed, s0 + j, m), tau)[0] for j in range(nb)], axis=1)
        U, V, d = block_fit(R, U0, tau, iters)
        R -= (U.astype(np.float64) * d) @ V.astype(np.float64).T
        B[:, s0:s0 + nb] = U
        C[s0:s0 + nb, :] = V.T
        D[s0:s0 + nb] = d
        energy[s0:s0 + nb] = 1.0 - float(np.sum(R * R)) / norm_a2
    e_final = 1.0 - float(np.sum(R * R)) / norm_a2
    return Factorization(B=B, C=C, D=D, energy=energy, energy_final=e_final, norm_a2=norm_a2,
                         margins=np.full(k, np.inf), safeguard_hits=0, residual_norms=None)


def residual_after(A: np.ndarray, B: np.ndarray, D: np.ndarray, C: np.ndarray, upto: int) -> np.ndarray:
    """R_i = A - sum_{j < upto} d_j b_j c_j^T in fp64 (teacher forcing from given factors)."""
    Bf = np.asarray(B[:, :upto], dtype=np.float64)
    Cf = np.asarray(C[:upto, :], dtype=np.float64)
    return np.asarray(A, dtype=np.float64) - (Bf * np.asarray(D[:upto], dtype=np.float64)) @ Cf


# ----------------------------------------------------------------------------
# §2.1 reconstruction / energy, §2.6 Eq. (1)
# ----------------------------------------------------------------------------


def reconstruct(B: np.ndarray, D: np.ndarray, C: np.ndarray) -> np.ndarray:
    """Ahat = B diag(D) C in fp64."""
    return (np.asarray(B, dtype=np.float64) * np.asarray(D, dtype=np.float64)) @ np.asarray(C, dtype=np.float64)


def energy(A: np.ndarray, Ahat: np.ndarray) -> float:
    A = np.asarray(A, dtype=np.float64)
    diff = A - np.asarray(Ahat, dtype=np.float64)
    return 1.0 - float(np.sum(diff * diff)) / float(np.sum(A * A))


def bpw_eff(mu: float, m: int, n: int, sparsity: float) -> float:
    """§2.6 Eq. (1): mask+sign packing bits per original weight."""
    return mu * (m + n) / max(m, n) * (2.0 - sparsity)


def gaussian_zero_fraction(tau: float) -> float:
    """P(|z| <= tau * E|z|) for z ~ N(0,1): 2 Phi(tau sqrt(2/pi)) - 1 = erf(tau / sqrt(pi))."""
    return math.erf(tau / math.sqrt(math.pi))


# ----------------------------------------------------------------------------
# §2.6 inference with the factors and mask+sign storage
# ----------------------------------------------------------------------------


def factored_matvec(B: np.ndarray, D: np.ndarray, C: np.ndarray, X: np.ndarray) -> np.ndarray:
    """§2.6: y = B (diag(D) (C x)) for each column x of X, in fp64, in the pages' order.

    B: m x k trits, D: k scales, C: k x n trits, X: n x batch.  Returns m x batch.
    """
    z = np.asarray(C, dtype=np.float64) @ np.asarray(X, dtype=np.float64)     # C x: k ternary sums each
    z = np.asarray(D, dtype=np.float64)[:, None] * z                           # diag(D): k multiplies
    return np.asarray(B, dtype=np.float64) @ z                                 # B (.): m ternary sums each


def ternary_op_count(B: np.ndarray, C: np.ndarray) -> int:
    """Add/subtract operations of y = B(diag(D)(Cx)) counted as the nonzero trits touched."""
    return int(np.count_nonzero(B)) + int(np.count_nonzero(C))


def mask_sign_pack(t: np.ndarray):
    """§2.6 mask+sign packing of one trit row: a 1-bit zero/nonzero mask per element and
    one sign bit per nonzero element (1 = negative), both least-significant bit first.

    Returns (mask bytes, sign bytes, number of nonzeros)."""
    t = np.asarray(t, dtype=np.int8)
    nz = t != 0
    mask = np.packbits(nz.astype(np.uint8), bitorder="little")
    signs = np.packbits((t[nz] < 0).astype(np.uint8), bitorder="little")
    return mask, signs, int(nz.sum())


def mask_sign_unpack(mask: np.ndarray, signs: np.ndarray, length: int) -> np.ndarray:
    nz = np.unpackbits(np.asarray(mask, dtype=np.uint8), bitorder="little")[:length].astype(bool)
    cnt = int(nz.sum())
    neg = np.unpackbits(np.asarray(signs, dtype=np.uint8), bitorder="little")[:cnt].astype(bool)
    t = np.zeros(length, dtype=np.int8)
    vals = np.where(neg, -1, 1).astype(np.int8)
    t[nz] = vals
    return t


def mask_sign_bits(B: np.ndarray, C: np.ndarray) -> int:
    """Storage of the factors in mask+sign form: one mask bit per element, one sign bit per nonzero."""
    return int(B.size + C.size + np.count_nonzero(B) + np.count_nonzero(C))


# ----------------------------------------------------------------------------
# §2.5 importance-weighted ALS (sequential, one component at a time)
# ----------------------------------------------------------------------------


def normalized_weights(h: np.ndarray, lam: float) -> np.ndarray:
    """h~ = h / max(h) + lambda (§2.5), computed in fp64 and held in fp32 like the GPU path
    (reading: the weights are stored once per matrix in single precision)."""
    h = np.asarray(h, dtype=np.float64)
    return (h / np.max(h) + lam).astype(np.float32)


def weighted_energy(A: np.ndarray, Ahat: np.ndarray, hw: np.ndarray) -> float:
    """1 - sum_ij h~_j (A - Ahat)^2_ij / sum_ij h~_j A^2_ij."""
    A = np.asarray(A, dtype=np.float64)
    w = np.asarray(hw, dtype=np.float64)[None, :]
    diff = A - np.asarray(Ahat, dtype=np.float64)
    return 1.0 - float(np.sum(w * diff * diff)) / float(np.sum(w * A * A))


def weighted_ls_scale(R: np.ndarray, u: np.ndarray, v: np.ndarray, hw: np.ndarray) -> float:
    """argmin_d sum_ij h~_j (R - d u v^T)^2_ij = u^T R (h~ v) / (||u||^2 sum_j h~_j v_j^2)."""
    u = np.asarray(u, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    w = np.asarray(hw, dtype=np.float64)
    p = float(u @ (np.asarray(R, dtype=np.float64) @ (w * v)))
    if p == 0.0:
        return 0.0
    return p / (float(u @ u) * float(w @ (v * v)))


def half_step_weighted(R: np.ndarray, trits_in: np.ndarray, tau: float, transpose: bool, hw: np.ndarray):
    """One half of §2.3 step 1 under the §2.5 objective.

    transpose=True : x = R^T u, v = T_tau(x)         (V-step on the plain residual: h~ cancels)
    transpose=False: y = R (h~ v), u = T_tau(y)      (U-step on the weighted target W = R diag(h~))
    Returns (pre-threshold vector, threshold, output trits, fallback_used)."""
    if transpose:
        return half_step(R, trits_in, tau, True)
    R = np.asarray(R, dtype=np.float64)
    w = np.asarray(trits_in, dtype=np.float64) * np.asarray(hw, dtype=np.float64)
    pre = R @ w
    out, thr, fb = ternarize(pre, tau)
    return pre, thr, out, fb


def greedy_als_weighted(A: np.ndarray, h: np.ndarray, lam: float, k: int, tau: float, iters: int = 15,
                        seed: int = 0) -> Factorization:
    """§2.5 with §2.3: V-step on the plain residual (h~ cancels there), U-step on
    W = R diag(h~), scale from the weighted normal equation, plain deflation.  The
    energy is the weighted one; the start vectors are those of greedy_als."""
    hw = normalized_weights(h, lam).astype(np.float64)
    R = np.array(A, dtype=np.float64, copy=True)
    m, n = R.shape
    norm_w = float(np.sum(hw[None, :] * R * R))
    if norm_w == 0.0:
        raise ValueError("weighted ||A|| = 0: energy is undefined")
    B = np.zeros((m, k), dtype=np.int8)
    C = np.zeros((k, n), dtype=np.int8)
    D = np.zeros(k, dtype=np.float64)
    energy = np.zeros(k, dtype=np.float64)
    margins = np.zeros(k, dtype=np.float64)
    r2 = norm_w
    for i in range(k):
        u, _, _ = ternarize(start_normals(seed, i, m), tau)
        margin = math.inf
        y = None
        v = None
        for _ in range(iters):
            x = R.T @ u.astype(np.float64)                    # V-step on R
            v, tv, _ = ternarize(x, tau)
            margin = min(margin, relative_margin(x, tv))
            y = R @ (hw * v.astype(np.float64))               # U-step on W = R diag(h~)
            u, tu, _ = ternarize(y, tau)
            margin = min(margin, relative_margin(y, tu))
        p = float(u.astype(np.float64) @ y)                  # u^T R (h~ v)
        nu = int(np.count_nonzero(u))
        sv = float(np.sum(hw[v != 0]))                        # v^T diag(h~) v for ternary v
        d = 0.0 if p == 0.0 else p / (nu * sv)
        if d != 0.0:
            R -= d * np.outer(u.astype(np.float64), v.astype(np.float64))
        r2 -= (p * p) / (nu * sv)
        B[:, i] = u
        C[i, :] = v
        D[i] = d
        energy[i] = 1.0 - r2 / norm_w
        margins[i] = margin
    e_final = 1.0 - float(np.sum(hw[None, :] * R * R)) / norm_w
    return Factorization(B=B, C=C, D=D, energy=energy, energy_final=e_final, norm_a2=norm_w,
                         margins=margins, safeguard_hits=0, residual_norms=None)


# ----------------------------------------------------------------------------
# §2.4 refinement sweeps (blocks of one component)
# ----------------------------------------------------------------------------


@dataclass
class Refinement:
    B: np.ndarray              # m x k int8
    C: np.ndarray              # k x n int8
    D: np.ndarray              # k float64
    sweep_energy: np.ndarray   # per sweep, incremental (weighted when h is given): 1 - r2 / ||A||^2
    energy_final: float        # explicit energy of the final residual
    kept: int                  # visits that kept the stored pair (rescaled)
    margins: np.ndarray        # sweeps x k: closest approach of the refit's half-steps to a threshold tie
    decision_margins: np.ndarray  # sweeps x k: |dec_refit - dec_stored| / max(dec_refit, dec_stored)
    visit_residuals: np.ndarray = field(default=None)  # sweeps x k explicit residual norms after each visit


@dataclass
class Visit:
    u: np.ndarray
    v: np.ndarray
    d: float
    kept: bool             # the stored pair stayed (with its least-squares scale)
    p_old: float           # u_i^T R (h~ v_i) of the added-back residual
    n_old: float           # nnz(u_i) * sum_{v_i != 0} h~
    decrease: float        # decrease of the (weighted) squared residual by the chosen term
    margin: float          # closest approach of the refit's half-steps to a threshold tie
    decision_margin: float


def refine_visit(R: np.ndarray, ui: np.ndarray, vi: np.ndarray, tau: float, iters: int, hw: np.ndarray) -> Visit:
    """One §2.4 visit on the added-back residual R = R_prev + d_i u_i v_i^T: refit from u_i
    (V-step on R, U-step on R diag(h~)), then take the refit or the stored pair, whichever
    decreases the residual more with its least-squares scale (ties go to the refit)."""
    uf = np.asarray(ui, dtype=np.float64)
    vf = np.asarray(vi, dtype=np.float64)
    p_old = float(uf @ (R @ (hw * vf)))
    n_old = float(np.count_nonzero(ui)) * float(np.sum(hw[vf != 0]))
    d_old = 0.0 if (p_old == 0.0 or n_old == 0.0) else p_old / n_old
    dec_old = p_old * d_old
    u = np.asarray(ui, dtype=np.int8).copy()
    v = None
    y = None
    margin = math.inf
    for _ in range(iters):
        x = R.T @ u.astype(np.float64)
        v, tv, _ = ternarize(x, tau)
        margin = min(margin, relative_margin(x, tv))
        y = R @ (hw * v.astype(np.float64))
        u, tu, _ = ternarize(y, tau)
        margin = min(margin, relative_margin(y, tu))
    p = float(u.astype(np.float64) @ y)
    nn = float(np.count_nonzero(u)) * float(np.sum(hw[v != 0]))
    d = 0.0 if p == 0.0 else p / nn
    dec = p * d
    top = max(dec, dec_old)
    dm = abs(dec - dec_old) / top if top > 0.0 else math.inf
    if dec >= dec_old:
        return Visit(u=u, v=v, d=d, kept=False, p_old=p_old, n_old=n_old, decrease=dec, margin=margin,
                     decision_margin=dm)
    return Visit(u=np.asarray(ui, dtype=np.int8).copy(), v=np.asarray(vi, dtype=np.int8).copy(), d=d_old, kept=True,
                 p_old=p_old, n_old=n_old, decrease=dec_old, margin=margin, decision_margin=dm)


def refine_sweeps(A: np.ndarray, B: np.ndarray, D: np.ndarray, C: np.ndarray, sweeps: int, tau: float,
                  iters: int = 15, h: np.ndarray | None = None, lam: float = 0.0,
                  track_residual: bool = False) -> Refinement:
    """§2.4 refinement sweeps with b = 1 on the factors (B, D, C) of A, for the plain
    objective (h None) or the §2.5 weighted one.  Each visit of component i:
    R <- R + d_i u_i v_i^T, refine_visit, R <- R - d u v^T with the chosen term."""
    A = np.asarray(A, dtype=np.float64)
    m, n = A.shape
    k = int(np.asarray(D).shape[0])
    hw = np.ones(n) if h is None else normalized_weights(h, lam).astype(np.float64)
    B = np.array(B, dtype=np.int8, copy=True)
    C = np.array(C, dtype=np.int8, copy=True)
    D = np.array(D, dtype=np.float64, copy=True)
    R = residual_after(A, B, D, C, k)
    norm = float(np.sum(hw[None, :] * A * A))
    r2 = float(np.sum(hw[None, :] * R * R))
    sweep_energy = np.zeros(sweeps)
    margins = np.zeros((sweeps, k))
    dmargins = np.zeros((sweeps, k))
    res = np.zeros((sweeps, k)) if track_residual else None
    kept = 0
    for s in range(sweeps):
        for i in range(k):
            di = float(D[i])
            R += di * np.outer(B[:, i].astype(np.float64), C[i, :].astype(np.float64))   # add back
            vis = refine_visit(R, B[:, i], C[i, :], tau, iters, hw)
            r2 += 2.0 * di * vis.p_old - di * di * vis.n_old
            r2 -= vis.decrease
            B[:, i] = vis.u
            C[i, :] = vis.v
            D[i] = vis.d
            kept += int(vis.kept)
            margins[s, i] = vis.margin
            dmargins[s, i] = vis.decision_margin
            R -= vis.d * np.outer(vis.u.astype(np.float64), vis.v.astype(np.float64))
            if track_residual:
                res[s, i] = float(np.sum(hw[None, :] * R * R))
        sweep_energy[s] = 1.0 - r2 / norm
    e_final = 1.0 - float(np.sum(hw[None, :] * R * R)) / norm
    return Refinement(B=B, C=C, D=D, sweep_energy=sweep_energy, energy_final=e_final, kept=kept,
                      margins=margins, decision_margins=dmargins, visit_residuals=res)
