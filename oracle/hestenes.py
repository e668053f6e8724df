"""Hand-written fp64 one-sided Jacobi (Hestenes) SVD, used to cross-check LAPACK.

TEST INFRASTRUCTURE ONLY.  Textbook method (M. R. Hestenes, "Inversion of
matrices by biorthogonalization", 1958; J. Demmel and K. Veselić, "Jacobi's
method is more accurate than QR", 1992): rotate pairs of columns of W = X·J
until every pair is orthogonal; then the column norms of W are the singular
values and J holds the right singular vectors.  Deliberately independent of
numpy.linalg.svd so that the two can pin each other.
"""
from __future__ import annotations

import numpy as np


def hestenes_svd(x: np.ndarray, tol: float = 1e-15, max_sweeps: int = 60):
    """Return (sigma descending, right singular vectors as columns, sweeps used)."""
    w = np.array(x, dtype=np.float64, copy=True)
    n, d = w.shape
    j = np.eye(d)
    for sweep in range(1, max_sweeps + 1):
        rotated = False
        for p in range(d - 1):
            for q in range(p + 1, d):
                a = w[:, p] @ w[:, p]
                b = w[:, q] @ w[:, q]
                c = w[:, p] @ w[:, q]
                if abs(c) <= tol * np.sqrt(a * b) or c == 0.0:
                    continue
                rotated = True
                zeta = (b - a) / (2.0 * c)
                t = np.sign(zeta) / (abs(zeta) + np.sqrt(1.0 + zeta * zeta)) if zeta != 0 else 1.0
                cs = 1.0 / np.sqrt(1.0 + t * t)
                sn = cs * t
                wp, wq = w[:, p].copy(), w[:, q].copy()
                w[:, p] = cs * wp - sn * wq
                w[:, q] = sn * wp + cs * wq
                jp, jq = j[:, p].copy(), j[:, q].copy()
                j[:, p] = cs * jp - sn * jq
                j[:, q] = sn * jp + cs * jq
        if not rotated:
            break
    sigma = np.sqrt((w * w).sum(axis=0))
    order = np.argsort(-sigma, kind="stable")
    return sigma[order], j[:, order], sweep
