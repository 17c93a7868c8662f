"""Pins of the oracle's fitted weight refinements (oracle/fit.py) against what
the mathematics fixes: the all-selected case reduces to plain nested
quantisation, a one-row calibration set has a closed form, the fitted
correction is a stationary point of the stated objective, every fitted code
names the sub-bin that holds the fitted value, and on held-out rows from the
calibration distribution the fitted codes leave less output error than the
plain ones ("StrataFlux -- Selective precision streaming -- What does it
mean?", nested-quantization paragraph)."""
import numpy as np
import pytest

import oracle
from oracle import fit
from bit_decode_selective_b200 import inputs

ALPHA = 0.01


def f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def case(N, K, n_cal, seed, b=2, r=2, G=128):
    w = inputs.weight(np.random.default_rng(seed), N, K)
    qb, rho, sz = oracle.quant_weights(w, b, r, G)
    X16 = inputs.calibration_activations(n_cal, K, seed + 1).view(np.uint16)
    return w, qb, rho, sz, X16


def base_error(w, qb, sz, r, G):
    return w.astype(np.float64) - oracle.dequant_weights(qb, np.zeros_like(qb), sz, r, G)


def test_all_channels_selected_gives_plain_codes():
    # k = C: A = X, so P = (X^T X + lam I)^-1 (X^T X + lam I) = I and d = e
    w, qb, rho, sz, X16 = case(64, 1024, 48, 3)
    r, G = 2, 128
    rho_f, D = fit.fit_refinements(w, qb, sz, r, G, X16, 1024, 1024, ALPHA)
    E = base_error(w, qb, sz, r, G)
    assert np.abs(D - E).max() <= 1e-9 * np.abs(E).max()
    S = np.repeat(f16(sz[:, :, 0]), G, axis=1)
    M = np.repeat(f16(sz[:, :, 1]), G, axis=1)
    t = ((w.astype(np.float64) - M) / S + 0.5) * (1 << r)  # plain nested code before the floor
    near = np.abs(t - np.round(t)) < 1e-6
    diff = rho_f != rho
    assert not np.any(diff & ~near)
    assert diff.sum() <= near.sum()


def test_one_calibration_row_closed_form():
    # one row x, k = 1: only channel c (largest |x|) is selected, G has the one
    # entry x_c^2, lam = alpha x_c^2 / C, and the minimiser is
    #   d_c = (x_c (x . e) + lam e_c) / (x_c^2 + lam),  d_j = e_j for j != c
    w, qb, rho, sz, X16 = case(16, 1024, 1, 5)
    r, G = 2, 128
    _, D = fit.fit_refinements(w, qb, sz, r, G, X16, 1024, 1, ALPHA)
    x = f16(X16[0])
    c = int(np.argmax(np.abs(x)))
    lam = ALPHA * x[c] ** 2 / 1024
    E = base_error(w, qb, sz, r, G)
    want = E.copy()
    want[:, c] = (x[c] * (E @ x) + lam * E[:, c]) / (x[c] ** 2 + lam)
    assert np.allclose(D, want, rtol=1e-9, atol=1e-12 * np.abs(E).max())


def test_fitted_correction_is_stationary_and_beats_plain():
    # d minimises |X e - A d|^2 + lam |d - e|^2 per chunk: its gradient is zero
    # and the objective is no larger than at d = e (plain refinement)
    K, C, k = 2048, 1024, 32
    w, qb, rho, sz, X16 = case(8, K, 300, 7)
    r, G = 2, 128
    _, D = fit.fit_refinements(w, qb, sz, r, G, X16, C, k, ALPHA)
    E = base_error(w, qb, sz, r, G)
    X = f16(X16)
    A = fit.masked_activations(X16, C, k)
    for j in range(K // C):
        J = slice(j * C, (j + 1) * C)
        lam = ALPHA * np.sum(A[:, J] ** 2) / C
        for i in range(E.shape[0]):
            e, d = E[i, J], D[i, J]
            res = X[:, J] @ e - A[:, J] @ d
            grad = -A[:, J].T @ res + lam * (d - e)
            scale = np.abs(A[:, J].T @ (X[:, J] @ e)).max()
            assert np.abs(grad).max() <= 1e-8 * scale
            obj = lambda dd: np.sum((X[:, J] @ e - A[:, J] @ dd) ** 2) + lam * np.sum((dd - e) ** 2)
            assert obj(d) <= obj(e)
            rng = np.random.default_rng(i)
            assert obj(d) <= obj(d + 1e-3 * np.abs(e).max() * rng.standard_normal(C))


def test_fitted_code_names_the_sub_bin_of_the_fitted_value():
    w, qb, rho, sz, X16 = case(32, 1024, 200, 9, b=3, r=2, G=64)
    r, G = 2, 64
    rho_f, D = fit.fit_refinements(w, qb, sz, r, G, X16, 1024, 32, ALPHA)
    S = np.repeat(f16(sz[:, :, 0]), G, axis=1)
    base = oracle.dequant_weights(qb, np.zeros_like(qb), sz, r, G)
    refined = oracle.dequant_weights(qb, rho_f, sz, r, G, refined_mask=np.ones(qb.shape, bool))
    # the fitted value, kept inside the base bin [base - S/2, base + S/2]
    target = base + np.clip(D, -S / 2, S / 2 * (1 - 2.0 ** -20))
    ok = S > 0
    assert np.all(np.abs(refined - target)[ok] <= (S / (1 << (r + 1)) * (1 + 1e-9))[ok])
    assert np.all(rho_f[~ok] == 0)


@pytest.mark.parametrize("b,r", [(2, 2), (3, 1)])
def test_fitted_codes_reduce_held_out_error(b, r):
    # on rows drawn from the calibration distribution but not used in the fit,
    # the refined product with fitted codes is closer to the full-precision one
    N, K, C, k, G = 128, 2048, 1024, 32, 128
    w, qb, rho, sz, X16 = case(N, K, 512, 11, b=b, r=r, G=G)
    rho_f, _ = fit.fit_refinements(w, qb, sz, r, G, X16, C, k, ALPHA)
    Xh = inputs.calibration_activations(128, K, 99)
    sel = oracle.select_chunks(Xh, C, k)
    y_true = Xh.astype(np.float64) @ w.astype(np.float64).T
    y_base = oracle.gemv_refined(qb, rho, sz, r, G, Xh, sel, C, 0)
    err = lambda rh: np.linalg.norm(y_true - oracle.gemv_refined(qb, rh, sz, r, G, Xh, sel, C, k))
    base_err = np.linalg.norm(y_true - y_base)
    assert err(rho) < base_err
    assert err(rho_f) < 0.95 * err(rho)
