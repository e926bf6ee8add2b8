"""Brute-force one-sided Jacobi SVD in fp64.  TEST INFRASTRUCTURE ONLY.

Used by the tests to pin the Newton-Schulz oracle to its closed form
U p^k(S/||M||_F) V^T (the polar-factor target of eq. (2), section 4 of the page
"Muon: An optimizer for hidden layers in neural networks"), by a route that
shares nothing with the iteration itself.

Method: Hestenes' one-sided Jacobi.  Columns of a working copy of M are
orthogonalised pairwise by plane rotations until every pair is orthogonal to
working precision; the column norms are then the singular values, the
normalised columns the left singular vectors, and the accumulated rotations
the right singular vectors.  Meant for small matrices (up to ~128 columns).
"""
from __future__ import annotations

from typing import Tuple

import numpy as np


def jacobi_svd(M: np.ndarray, tol: float = 1e-15, max_sweeps: int = 60) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Thin SVD M = U diag(S) V^T of an r x c matrix, returned as (U, S, Vt).

    U is r x k, S has k entries (descending), Vt is k x c, with k = min(r, c).
    Zero singular values come back with a zero column in U."""
    M = np.asarray(M, dtype=np.float64)
    transposed = M.shape[0] < M.shape[1]
    A = (M.T if transposed else M).copy()   # tall: rows >= cols
    n = A.shape[1]
    V = np.eye(n)
    for _ in range(max_sweeps):
        rotated = False
        for p in range(n - 1):
            for q in range(p + 1, n):
                ap, aq = A[:, p], A[:, q]
                alpha = float(ap @ ap)
                beta = float(aq @ aq)
                gamma = float(ap @ aq)
                if abs(gamma) <= tol * np.sqrt(alpha * beta) or gamma == 0.0:
                    continue
                rotated = True
                zeta = (beta - alpha) / (2.0 * gamma)
                t = np.sign(zeta) / (abs(zeta) + np.sqrt(1.0 + zeta * zeta)) if zeta != 0 else 1.0
                cs = 1.0 / np.sqrt(1.0 + t * t)
                sn = cs * t
                new_p = cs * ap - sn * aq
                new_q = sn * ap + cs * aq
                A[:, p], A[:, q] = new_p, new_q
                vp, vq = V[:, p].copy(), V[:, q].copy()
                V[:, p] = cs * vp - sn * vq
                V[:, q] = sn * vp + cs * vq
        if not rotated:
            break
    S = np.sqrt(np.sum(A * A, axis=0))
    order = np.argsort(-S)
    S = S[order]
    A = A[:, order]
    V = V[:, order]
    U = np.zeros_like(A)
    nz = S > 0
    U[:, nz] = A[:, nz] / S[nz]
    if transposed:
        # M^T = U S V^T  =>  M = V S U^T
        return V, S, U.T
    return U, S, V.T
