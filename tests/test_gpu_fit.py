"""Parity of the fitted refinements (sf_fit_refinements) with the oracle's fit
(oracle/fit.py), through the C ABI.

Bar: the base codes, steps and offsets are untouched (bit-exact); the fitted
corrections d agree within 1e-8 of the largest base error (both sides are
fp64; they differ only in summation order and in Cholesky versus LU, so the
difference is a small multiple of cond(G + lam I) * n_cal * 2^-53 of it); the
fitted codes are bit-exact except where the oracle's (d / s + 1/2) 2^r lies
within 1e-5 of an integer, far above that difference once scaled by 2^r / s.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import fit as ofit
from bit_decode_selective_b200 import inputs
from bit_decode_selective_b200.ops import QuantWeights

pytestmark = pytest.mark.gpu

ALPHA = 0.01
D_TOL = 1e-8
EDGE = 1e-5


@pytest.fixture(scope="module", autouse=True)
def dev():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    oracle.set_threads(0)


def f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def fit_both(N, K, b, r, G, n_cal, C, k, seed):
    w = inputs.weight(np.random.default_rng(seed), N, K)
    X16 = inputs.calibration_activations(n_cal, K, seed + 1).view(np.uint16)
    qb, rho, sz = oracle.quant_weights(w, b, r, G)
    rho_o, D_o = ofit.fit_refinements(w, qb, sz, r, G, X16, C, k, ALPHA)
    wd = torch.from_numpy(w).cuda()
    qw = QuantWeights.pack(wd, b, r, G)
    base0, sz0 = qw.base.clone(), qw.sz.clone()
    D_g = qw.fit_refinements(wd, torch.from_numpy(X16.view(np.int16)).cuda(), C, k, ALPHA, want_delta=True)
    torch.cuda.synchronize()
    assert torch.equal(qw.base, base0) and torch.equal(qw.sz, sz0)
    gq, grho = qw.unpack()
    assert np.array_equal(gq.cpu().numpy(), qb)
    return w, qb, rho, sz, qw, rho_o, D_o, D_g.cpu().numpy(), grho.cpu().numpy()


def check_codes(rho_o, rho_g, D_o, sz, r, G):
    S = np.repeat(f16(sz[:, :, 0]), G, axis=1)
    t = (D_o / np.where(S == 0, 1.0, S) + 0.5) * (1 << r)
    near = (np.abs(t - np.round(t)) < EDGE) & (S != 0)
    diff = rho_o != rho_g
    assert not np.any(diff & ~near), int((diff & ~near).sum())


@pytest.mark.parametrize("N,K,b,r,G,n_cal,C,k", [
    (256, 2048, 2, 2, 128, 300, 1024, 32),   # two chunks, ragged selection batches
    (128, 1024, 3, 1, 64, 70, 512, 16),      # 3-bit base, 1 refinement bit, 512-channel chunks
    (128, 2048, 4, 2, 32, 1, 2048, 1),       # one calibration row, one 2048-channel chunk
])
def test_fit_matches_oracle(N, K, b, r, G, n_cal, C, k):
    w, qb, rho, sz, qw, rho_o, D_o, D_g, rho_g = fit_both(N, K, b, r, G, n_cal, C, k, 40 + K // 512 + b)
    E = w.astype(np.float64) - oracle.dequant_weights(qb, np.zeros_like(qb), sz, r, G)
    assert np.abs(D_g - D_o).max() <= D_TOL * np.abs(E).max()
    check_codes(rho_o, rho_g, D_o, sz, r, G)


def test_fit_all_selected_keeps_plain_codes():
    # k = chunk: the fit reduces to plain nested quantisation
    w, qb, rho, sz, qw, rho_o, D_o, D_g, rho_g = fit_both(128, 1024, 2, 2, 128, 40, 1024, 1024, 50)
    check_codes(rho_o, rho_g, D_o, sz, 2, 128)
    S = np.repeat(f16(sz[:, :, 0]), 128, axis=1)
    M = np.repeat(f16(sz[:, :, 1]), 128, axis=1)
    t = ((w.astype(np.float64) - M) / S + 0.5) * 4
    near = np.abs(t - np.round(t)) < EDGE
    assert not np.any((rho_g != rho) & ~near)


def test_refined_gemv_with_fitted_codes():
    # the decode-step GEMV reads the refitted codes: parity with the oracle's
    # refined product on the fitted codes, and less error than plain codes on
    # held-out rows of the calibration distribution
    N, K, b, r, G, C, k = 512, 2048, 2, 2, 128, 1024, 32
    w, qb, rho, sz, qw, rho_o, D_o, D_g, rho_g = fit_both(N, K, b, r, G, 400, C, k, 60)
    Xh = inputs.calibration_activations(8, K, 777)
    xd = torch.from_numpy(Xh.view(np.int16)).cuda()
    y, _ = qw.gemv(xd, C, k)
    torch.cuda.synchronize()
    sel = oracle.select_chunks(Xh, C, k)
    y_o = oracle.gemv_refined(qb, rho_g, sz, r, G, Xh, sel, C, k)
    yg = y.cpu().numpy()
    assert np.linalg.norm(yg - y_o) <= 1e-3 * np.linalg.norm(y_o)
    plain = QuantWeights.pack(torch.from_numpy(w).cuda(), b, r, G)
    yp, _ = plain.gemv(xd, C, k)
    torch.cuda.synchronize()
    y_true = Xh.astype(np.float64) @ w.astype(np.float64).T
    assert np.linalg.norm(yg - y_true) < 0.95 * np.linalg.norm(yp.cpu().numpy() - y_true)


def test_fit_benchmarked_shape():
    # the benchmarked fit: 4096 x 4096, 2+2 bits, group 128, 512 calibration
    # rows, k = 32 per 1,024 -- every correction and every code
    w, qb, rho, sz, qw, rho_o, D_o, D_g, rho_g = fit_both(4096, 4096, 2, 2, 128, 512, 1024, 32, 70)
    E = w.astype(np.float64) - oracle.dequant_weights(qb, np.zeros_like(qb), sz, 2, 128)
    assert np.abs(D_g - D_o).max() <= D_TOL * np.abs(E).max()
    check_codes(rho_o, rho_g, D_o, sz, 2, 128)
