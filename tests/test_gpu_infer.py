"""Parity of the inference path (§2.6: y = B diag(D) C x, mask+sign storage) with the oracle.

Tolerance of the products (derived from the arithmetic): every term t x of a row
dot is formed exactly (the trit is decoded into an exact power-of-two multiple and
the staged vector entry carries the inverse power of two), and the terms are summed
in fp32: each lane keeps two running sums (even and odd trits of its words), adds
them, and the 32 lane sums are combined by a butterfly.  The rounding error of
z = D (C x) is therefore at most ~(len/64 + 7) 2^-24 |D| (|C| |x|), and y = B z adds
the same relative error on top of the error carried by z.  For len <= 16384 that is
below 3e-5 * (|B| |D| |C| |x|) elementwise, which the tests use (plus 1e-30
absolute).  With small-integer inputs every partial sum is an exactly representable
integer, so the result is exact.  Transposes and the mask+sign storage are
bit-exact.
"""
import numpy as np
import pytest
import torch

import ternary_rank_weight_b200 as ext
from oracle import externd_oracle as ora
from ternary_rank_weight_b200.workloads import WORKLOADS, llm_matrix

pytestmark = pytest.mark.gpu


def _random_factors(m, n, k, density, seed):
    rng = np.random.default_rng(seed)
    p = [density / 2, 1 - density, density / 2]
    B = rng.choice([-1, 0, 1], size=(m, k), p=p).astype(np.int8)
    C = rng.choice([-1, 0, 1], size=(k, n), p=p).astype(np.int8)
    D = (rng.standard_normal(k) * 0.01).astype(np.float32)
    return B, D, C


def _device_factors(B, D, C):
    Bp = torch.from_numpy(ext.pack_trits(B.T.copy())).cuda()     # k rows of m trits (the factor layout)
    Cp = torch.from_numpy(ext.pack_trits(C)).cuda()
    return Bp, torch.from_numpy(D).cuda(), Cp


def _check_matvec(B, D, C, X, Y):
    want = ora.factored_matvec(B, D.astype(np.float64), C, X.T.astype(np.float64)).T
    bound = ora.factored_matvec(np.abs(B), np.abs(D.astype(np.float64)), np.abs(C), np.abs(X.T.astype(np.float64))).T
    err = np.abs(Y.astype(np.float64) - want)
    assert np.all(err <= 3e-5 * bound + 1e-30), float(np.max(err / (bound + 1e-30)))


@pytest.mark.parametrize("rows,length", [(1, 1), (3, 5), (64, 64), (65, 63), (200, 777), (1000, 130)])
def test_transpose_trits_is_exact(rows, length):
    rng = np.random.default_rng(rows * 7 + length)
    T = rng.integers(-1, 2, size=(rows, length)).astype(np.int8)
    Tt = ext.transpose_trits(torch.from_numpy(ext.pack_trits(T)).cuda(), rows, length)
    assert Tt.shape == (length, ext.trit_bytes(rows))
    got = ext.unpack_trits(Tt.cpu().numpy(), rows)
    assert np.array_equal(got, T.T)
    # padding trits stay zero
    full = ext.unpack_trits(Tt.cpu().numpy(), ext.trit_bytes(rows) * 4)
    assert not full[:, rows:].any()


@pytest.mark.parametrize("m,n,k,batch", [(1, 1, 1, 1), (7, 5, 9, 1), (33, 65, 40, 3), (130, 70, 300, 9),
                                         (512, 384, 1024, 2), (40, 90, 77, 5), (64, 33, 129, 6), (19, 200, 64, 7),
                                         (5000, 700, 300, 1), (3000, 1000, 6000, 1),
                                         (16, 60000, 40, 2), (8, 16, 50000, 1)])
def test_matvec_random_factors_match_oracle(m, n, k, batch):
    """Random factors; the last two shapes have rows too long for the staged-vector kernel (n = 60000,
    k = 50000 trits), so one of their two products runs the L1 kernel."""
    B, D, C = _random_factors(m, n, k, 0.45, seed=m + n + k)
    Bp, Dg, Cp = _device_factors(B, D, C)
    Bt = ext.transpose_trits(Bp, k, m)
    X = np.random.default_rng(batch).standard_normal((batch, n)).astype(np.float32)
    Y = ext.matvec(Bt, Dg, Cp, m, n, torch.from_numpy(X).cuda()).cpu().numpy()
    assert Y.shape == (batch, m)
    _check_matvec(B, D, C, X, Y)


def test_matvec_of_a_factorization_matches_oracle_and_reconstruction():
    A = llm_matrix(96, 200, seed=3)
    f = ext.factor(torch.from_numpy(A).cuda(), 2.0, 1.0, seed=2)
    Bg, Cg = f.trits()
    Dh = f.D.cpu().numpy()
    X = np.random.default_rng(5).standard_normal((4, 200)).astype(np.float32)
    Y = ext.matvec(ext.inference_layout(f), f.D, f.C, f.m, f.n, torch.from_numpy(X).cuda()).cpu().numpy()
    _check_matvec(Bg, Dh, Cg, X, Y)
    # the same as (B diag(D) C) x with the reconstruction
    Ah = ext.reconstruct(f.B, f.D, f.C, f.m, f.n).cpu().numpy().astype(np.float64)
    assert np.allclose(Y.T, Ah @ X.T.astype(np.float64), rtol=1e-4, atol=1e-5 * np.abs(Ah).sum(1).max())


def test_matvec_single_vector_and_zero_input():
    B, D, C = _random_factors(20, 30, 50, 0.5, seed=11)
    Bp, Dg, Cp = _device_factors(B, D, C)
    Bt = ext.transpose_trits(Bp, 50, 20)
    x = np.random.default_rng(1).standard_normal(30).astype(np.float32)
    y = ext.matvec(Bt, Dg, Cp, 20, 30, torch.from_numpy(x).cuda()).cpu().numpy()
    assert y.shape == (20,)
    _check_matvec(B, D, C, x[None], y[None])
    y0 = ext.matvec(Bt, Dg, Cp, 20, 30, torch.zeros(30, device="cuda")).cpu().numpy()
    assert np.all(y0 == 0)


@pytest.mark.parametrize("rows,length", [(1, 1), (5, 31), (17, 33), (64, 1000), (300, 2560)])
def test_mask_sign_storage_is_exact(rows, length):
    rng = np.random.default_rng(rows + length)
    T = rng.choice([-1, 0, 1], size=(rows, length), p=[0.3, 0.4, 0.3]).astype(np.int8)
    mask, signs, offs = ext.pack_mask_sign(torch.from_numpy(ext.pack_trits(T)).cuda(), rows, length)
    mask, offs = mask.cpu().numpy(), offs.cpu().numpy()
    bits = np.unpackbits(signs.cpu().numpy().view(np.uint8), bitorder="little")
    assert offs[0] == 0 and offs[-1] == np.count_nonzero(T)
    for r in range(rows):
        m_, s_, c_ = ora.mask_sign_pack(T[r])
        assert np.array_equal(mask[r], m_)
        assert offs[r + 1] - offs[r] == c_
        want_bits = np.unpackbits(s_, bitorder="little")[:c_]
        assert np.array_equal(bits[offs[r]:offs[r + 1]], want_bits)


def test_mask_sign_storage_of_factors_matches_eq1():
    A = llm_matrix(128, 256, seed=9)
    mu, tau = 2.0, 1.0
    f = ext.factor(torch.from_numpy(A).cuda(), mu, tau, seed=1)
    _, _, offB = ext.pack_mask_sign(f.B, f.k, f.m)
    _, _, offC = ext.pack_mask_sign(f.C, f.k, f.n)
    bits = f.k * (f.m + f.n) + int(offB[-1].item()) + int(offC[-1].item())
    Bg, Cg = f.trits()
    zf = (np.count_nonzero(Bg == 0) + np.count_nonzero(Cg == 0)) / (f.k * (f.m + f.n))
    assert bits / (f.m * f.n) == pytest.approx(ora.bpw_eff(mu, f.m, f.n, zf), rel=1e-12)


def test_matvec_headline_factors_full_size():
    """Factors of the 2560 x 6912 workload (k = 7680), batch 1 and 8, against the oracle."""
    w = WORKLOADS["mlp_2560x6912_bf16_mu3_tau1.0"]
    A = torch.from_numpy(w.matrix(0)).cuda()
    f = ext.factor(A, w.mu[0], w.tau[0], seed=w.seeds[0])
    Bg, Cg = f.trits()
    Dh = f.D.cpu().numpy()
    Bt = ext.inference_layout(f)
    for batch in (1, 8):
        X = np.random.default_rng(batch).standard_normal((batch, f.n)).astype(np.float32)
        Y = ext.matvec(Bt, f.D, f.C, f.m, f.n, torch.from_numpy(X).cuda()).cpu().numpy()
        _check_matvec(Bg, Dh, Cg, X, Y)


def test_matvec_small_integers_are_exact():
    """Integer inputs with every partial sum below 2^24: each term t x is formed exactly and
    each sum of integers is exact, so y equals the exact product bit for bit (a dropped or
    sign-flipped trit anywhere would show)."""
    m, n, k = 300, 500, 260
    B, _, C = _random_factors(m, n, k, 0.6, seed=21)
    D = np.ones(k, dtype=np.float32)
    Bp, Dg, Cp = _device_factors(B, D, C)
    Bt = ext.transpose_trits(Bp, k, m)
    for batch in (1, 2, 3, 8):
        X = np.random.default_rng(batch).integers(-8, 9, size=(batch, n)).astype(np.float32)
        Y = ext.matvec(Bt, Dg, Cp, m, n, torch.from_numpy(X).cuda()).cpu().numpy()
        want = (B.astype(np.int64) @ (C.astype(np.int64) @ X.T.astype(np.int64))).T
        assert np.array_equal(Y.astype(np.int64), want), batch


def test_matvec_huge_and_tiny_input_ranges():
    """Inputs near the top of the fp32 range (|x| ~ 2^110: staged with an extra power-of-two
    scale) and tiny ones (~2^-100), mixed in one batch, against the oracle."""
    m, n, k = 96, 130, 200
    B, D, C = _random_factors(m, n, k, 0.5, seed=33)
    D = np.abs(D) * 1e-3 + 1e-4
    D = D.astype(np.float32)
    Bp, Dg, Cp = _device_factors(B, D, C)
    Bt = ext.transpose_trits(Bp, k, m)
    rng = np.random.default_rng(4)
    X = rng.standard_normal((3, n)).astype(np.float32)
    X[0] *= np.float32(2.0 ** 110)
    X[2] *= np.float32(2.0 ** -100)
    Y = ext.matvec(Bt, Dg, Cp, m, n, torch.from_numpy(X).cuda()).cpu().numpy()
    assert np.all(np.isfinite(Y))
    _check_matvec(B, D, C, X, Y)


def test_matvec_rejects_unaligned_factors():
    """The trit rows are read in 16-byte units: factor pointers off a 16-byte boundary are refused
    before any launch."""
    B, D, C = _random_factors(8, 64, 16, 0.5, seed=2)
    Bp, Dg, Cp = _device_factors(B, D, C)
    Bt = ext.transpose_trits(Bp, 16, 8)
    buf = torch.zeros(Cp.numel() + 16, dtype=torch.uint8, device="cuda")
    buf[4:4 + Cp.numel()] = Cp.reshape(-1)
    X = torch.zeros((1, 64), device="cuda")
    Y = torch.empty((1, 8), device="cuda")
    Z = torch.empty((1, 16), device="cuda")
    rc = ext._lib.load().externd_matvec(ext.api._ptr(Bt), ext.api._ptr(Dg), buf.data_ptr() + 4, 8, 64, 16,
                                        ext.api._ptr(X), 1, ext.api._ptr(Y), ext.api._ptr(Z), None)
    assert rc == ext.STATUS["EINVAL"]
