"""Fitted weight refinements (TEST INFRASTRUCTURE, like the rest of ``oracle``).

"StrataFlux -- Selective precision streaming -- What does it mean?",
nested-quantization paragraph: for weights the refinement values are not only
copied from the full-precision weights but fitted on a small calibration set,
so that the channels a step refines partly make up for the error of the
channels it leaves at base precision.  The pages give no formula; the reading
written out here (plain numpy in fp64, ``@`` and ``numpy.linalg.solve`` as the
only library steps) is:

* the base codes and the group step/offset stay those of plain nested
  quantisation; only the r refinement bits of each weight are refitted, so the
  refined value still lies in the base bin (the format is unchanged);
* calibration activations X[n][K] pass through the same chunked top-k channel
  selection as decoding; A[n][c] = X[n][c] where channel c is selected for row
  n, else 0;
* per chunk J of C channels and per output row i, the correction d_i[J] (the
  refined minus the base value of the row's weights on J) minimises

      sum_n ( sum_{c in J} X[n][c] e_i[c] - sum_{c in J} A[n][c] d_i[c] )^2
        + lam * sum_{c in J} (d_i[c] - e_i[c])^2

  where e_i = w_i - (base values of row i) is the base error: on every
  calibration row, the chunk's selected channels reproduce the base error of
  the whole chunk, and the ridge term pulls d towards the plain refinement
  (it decides the channels calibration never selects);
* lam = alpha * trace(G) / C with G = A[:, J]^T A[:, J] (lam = 1 where that
  trace is 0), so d_i[J] = P e_i[J] with P = (G + lam I)^-1 (A[:, J]^T X[:, J]
  + lam I);
* the refinement code is the sub-bin of the base bin that holds the fitted
  value: rho = clamp(floor((d / s + 1/2) 2^r), 0, 2^r - 1), 0 where s = 0.

With every channel selected (k = C) A = X, P = I and d = e: the fit returns
plain nested quantisation.
"""
from __future__ import annotations

import numpy as np

from . import dequant_weights, select_chunks


def _f16(bits) -> np.ndarray:
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def fit_projector(A: np.ndarray, X: np.ndarray, alpha: float) -> np.ndarray:
    """P = (A^T A + lam I)^-1 (A^T X + lam I) for one chunk (A, X: [n][C] fp64)."""
    C = A.shape[1]
    G = A.T @ A
    lam = alpha * np.trace(G) / C
    if lam == 0.0:
        lam = 1.0
    eye = np.eye(C)
    return np.linalg.solve(G + lam * eye, A.T @ X + lam * eye)


def masked_activations(X16: np.ndarray, C: int, k: int) -> np.ndarray:
    """A[n][c] = X[n][c] where chunk selection picks channel c for row n, else 0."""
    X = _f16(X16)
    sel = select_chunks(X16, C, k)  # [n][K/C][k]
    mask = np.zeros(X.shape, bool)
    for n in range(X.shape[0]):
        mask[n, sel[n].ravel()] = True
    return np.where(mask, X, 0.0)


def fit_refinements(w: np.ndarray, qb: np.ndarray, sz: np.ndarray, r: int, G: int, X16: np.ndarray,
                    C: int, k: int, alpha: float):
    """Fitted refinement codes rho[N][K] (uint8) and the fitted corrections
    d[N][K] (fp64) of w[N][K] quantised to (qb, sz); X16[n][K] fp16 bits."""
    N, K = w.shape
    X16 = np.ascontiguousarray(X16, np.uint16)
    X = _f16(X16)
    A = masked_activations(X16, C, k)
    E = w.astype(np.float64) - dequant_weights(qb, np.zeros_like(qb), sz, r, G)
    D = np.empty((N, K), np.float64)
    for j in range(K // C):
        J = slice(j * C, (j + 1) * C)
        P = fit_projector(A[:, J], X[:, J], alpha)
        D[:, J] = E[:, J] @ P.T
    S = np.repeat(_f16(sz[:, :, 0]), G, axis=1)
    safe = np.where(S == 0.0, 1.0, S)
    rho = np.floor((D / safe + 0.5) * float(1 << r))
    rho = np.clip(rho, 0.0, float((1 << r) - 1))
    rho[S == 0.0] = 0.0
    return rho.astype(np.uint8), D
