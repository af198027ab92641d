"""Soft-Riesz density over post-RoPE keys (fp64, direct differences).

DensityKV, §3 Method "Soft-Riesz Density" and App. B.1 "From Riesz Energy to a
Smooth Crowding Score": a regularised inverse-power interaction between keys, with
a width (distance scale), a decay exponent and an anti-singularity term; the
density of a key is the sum of its interactions with the keys it is compared to,
and is only compared within one (layer, head).

Reading taken (the pages give the parameters, not the formula):

    x(a, b)   = ||a - b||^2 / h            (h = distance scale, default h = d)
    phi(x)    = (x + eps) ** (-s / 2)      (eps = 1e-3, s = 2 by default)
    rho(a; S) = sum_{b in S, id(b) != id(a)} phi(x(a, b))

The self term is excluded by token identity, so an exact duplicate with another
id still counts (it contributes eps ** (-s/2)).
"""
from __future__ import annotations

import numpy as np


def soft_riesz(x, eps: float, s: float):
    """phi(x) = (x + eps)^(-s/2) in fp64."""
    return (np.asarray(x, dtype=np.float64) + eps) ** (-s / 2.0)


def sq_dists(A: np.ndarray, B: np.ndarray, block: int = 32) -> np.ndarray:
    """||A_i - B_j||^2 by direct differences (no norm expansion), fp64."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    out = np.empty((A.shape[0], B.shape[0]), dtype=np.float64)
    for i0 in range(0, A.shape[0], block):
        diff = A[i0:i0 + block, None, :] - B[None, :, :]
        out[i0:i0 + block] = np.einsum("ijk,ijk->ij", diff, diff)
    return out


def density(rows: np.ndarray, cols: np.ndarray, *, h: float, eps: float, s: float,
            row_ids=None, col_ids=None, weights=None) -> np.ndarray:
    """rho(r) = sum_j w_j * phi(||r - c_j||^2 / h) over columns with id != id(r).

    ``weights`` (default all ones) lets a test express signed sums; the method
    itself only uses unit weights."""
    rows = np.asarray(rows, dtype=np.float64).reshape(-1, np.shape(rows)[-1])
    cols = np.asarray(cols, dtype=np.float64).reshape(-1, np.shape(cols)[-1])
    if rows.shape[0] == 0:
        return np.zeros(0)
    if cols.shape[0] == 0:
        return np.zeros(rows.shape[0])
    phi = soft_riesz(sq_dists(rows, cols) / h, eps, s)
    if weights is not None:
        phi = phi * np.asarray(weights, dtype=np.float64)[None, :]
    if row_ids is not None and col_ids is not None:
        same = np.asarray(row_ids)[:, None] == np.asarray(col_ids)[None, :]
        phi = np.where(same, 0.0, phi)
    return phi.sum(axis=1)
