"""Truncated-SVD bases and the Eckart-Young error (oracle side).

TraceKV abstract and digest ("sensitivity-aware SVD"): latents come from an
SVD of the KV states.  The sensitivity weights need a model and are out of
scope; their unweighted special case is the plain truncated SVD, whose error
has the closed form of the Eckart-Young theorem:
  ||X - X_r||_F^2 = sum_{i>r} s_i^2,   ||X - X_r||_2 = s_{r+1}.
"""
from __future__ import annotations

import numpy as np


def truncated_basis(X: np.ndarray, r: int):
    """Rank-r right singular basis of X ([T][D]): A = V_r ([D][r]), B = V_r^T ([r][D]),
    and all singular values.  X A B is the best rank-r approximation of X."""
    X = np.asarray(X, np.float64)
    _, s, vt = np.linalg.svd(X, full_matrices=False)
    B = vt[:r, :].copy()
    return B.T.copy(), B, s


def lowrank_residual(X: np.ndarray, A: np.ndarray, B: np.ndarray):
    """(Frobenius, spectral) norms of X - (X A) B."""
    X = np.asarray(X, np.float64)
    R = X - (X @ np.asarray(A, np.float64)) @ np.asarray(B, np.float64)
    return np.linalg.norm(R, "fro"), np.linalg.norm(R, 2)


def eckart_young(s: np.ndarray, r: int):
    """Closed-form optimal rank-r errors from singular values s (descending)."""
    s = np.asarray(s, np.float64)
    fro = np.sqrt(np.sum(s[r:] ** 2))
    spec = s[r] if r < s.size else 0.0
    return fro, spec
