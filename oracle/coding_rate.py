"""Marginal lossy coding rate, written out from its definition (float64).

Sources (ByteFlow, arXiv 2603.03583):
* paper.rainbus.top summary, "Prerequisites: lossy coding rate": for features
  H in R^{T x d}, R_eps(H) = 1/2 logdet(I + (d/eps^2) H H^T).
* same page, "Method steps", stage 2, and papernotes.org notes, "Key design 2":
  the marginal coding rate dR_t = R_eps(h_{1:t}) - R_eps(h_{1:t-1}).

Positions here are 0-based (the pages' t = 1 is index 0).  R of the empty
prefix is 0, so dR_0 = 1/2 log(1 + c |h_0|^2).  c = d / eps^2 with d the
feature width of H (the summary writes it d_local in stage 2).

Three independent evaluations:

* :func:`coding_rate` / :func:`dR_prefix_logdet` (O1): the definition itself.
  The T x T determinant is evaluated through Sylvester's identity
  det(I_T + c H H^T) = det(I_d + c H^T H); each logdet is twice the sum of the
  logs of a float64 Cholesky diagonal (LAPACK via NumPy).
* :func:`dR_chol_diag` (O2): with G = I_T + c H H^T and G = L L^T, the ratio of
  consecutive leading principal minors of G is L_tt^2 (Schur complement), so
  dR_t = log L_tt.  No Sylvester step; works on the T x T matrix directly.
* ``oracle.rank1`` (O3, plain C): a recursion over t keeping the Cholesky
  factor of M_t = I + c sum_{i<=t} h_i h_i^T, with the matrix determinant
  lemma det(M + c h h^T) = det(M)(1 + c h^T M^-1 h).

Streaming continuation (:func:`dR_continue`): a stream delivered in blocks
keeps, between blocks, the Gram sum S = sum of h h^T over everything seen so
far; the next block's dR follow from the same definition with that prefix
(R of the whole stream so far), so block-wise streaming reproduces the
whole-sequence values exactly.

This file is test infrastructure.  Only the test-suite, the smoke check and
the benchmark's CPU-baseline leg may import it.
"""
from __future__ import annotations

import numpy as np

__all__ = ["coding_rate", "coding_rate_T", "dR_prefix_logdet", "dR_chol_diag", "dR_continue"]


def _logdet_spd(A: np.ndarray) -> float:
    L = np.linalg.cholesky(A)
    return 2.0 * float(np.sum(np.log(np.diag(L))))


def coding_rate(H: np.ndarray, eps2: float) -> float:
    """R_eps(H) = 1/2 logdet(I_d + c H^T H), c = d/eps^2 (Sylvester form)."""
    H = np.asarray(H, dtype=np.float64)
    T, d = H.shape
    c = d / eps2
    return 0.5 * _logdet_spd(np.eye(d) + c * (H.T @ H))


def coding_rate_T(H: np.ndarray, eps2: float) -> float:
    """R_eps(H) = 1/2 logdet(I_T + c H H^T) in the pages' own T x T form."""
    H = np.asarray(H, dtype=np.float64)
    T, d = H.shape
    c = d / eps2
    return 0.5 * _logdet_spd(np.eye(T) + c * (H @ H.T))


def dR_prefix_logdet(H: np.ndarray, eps2: float, ts=None) -> np.ndarray:
    """O1: dR_t = R(h_{0..t}) - R(h_{0..t-1}) for one row, by prefix logdets.

    ``ts`` (sorted or not) selects positions; default all.  The running Gram
    S_t = sum_{i<=t} h_i h_i^T is accumulated in float64 and each R is a fresh
    Cholesky of I + c S.
    """
    H = np.asarray(H, dtype=np.float64)
    T, d = H.shape
    c = d / eps2
    ts = np.arange(T) if ts is None else np.asarray(ts, dtype=np.int64)
    order = np.argsort(ts, kind="stable")
    out = np.empty(len(ts), dtype=np.float64)
    S = np.zeros((d, d))
    upto = 0                      # S holds rows [0, upto)
    I = np.eye(d)
    for j in order:
        t = int(ts[j])
        if upto < t:
            X = H[upto:t]
            S += X.T @ X
            upto = t
        R_prev = 0.5 * _logdet_spd(I + c * S)
        h = H[t]
        R_t = 0.5 * _logdet_spd(I + c * (S + np.outer(h, h)))
        out[j] = R_t - R_prev
    return out


def dR_chol_diag(H: np.ndarray, eps2: float) -> np.ndarray:
    """O2: dR_t = log L_tt with L L^T = I_T + c H H^T (one row)."""
    H = np.asarray(H, dtype=np.float64)
    T, d = H.shape
    c = d / eps2
    G = c * (H @ H.T)
    G[np.diag_indices(T)] += 1.0
    L = np.linalg.cholesky(G)
    return np.log(np.diag(L))


def dR_continue(S0: np.ndarray, H: np.ndarray, eps2: float, ts=None):
    """dR of a new block H given the earlier positions' Gram sum S0 (float64).

    dR_t = R(earlier + h_{0..t}) - R(earlier + h_{0..t-1}) with
    R = 1/2 logdet(I + c S) and S the Gram sum of the positions included.
    Returns (dR at ``ts`` (default all rows of H), S0 + H^T H).
    """
    H = np.asarray(H, dtype=np.float64)
    T, d = H.shape
    c = d / eps2
    S0 = np.asarray(S0, dtype=np.float64)
    ts = np.arange(T) if ts is None else np.asarray(ts, dtype=np.int64)
    order = np.argsort(ts, kind="stable")
    out = np.empty(len(ts), dtype=np.float64)
    S = S0.copy()
    upto = 0
    I = np.eye(d)
    for j in order:
        t = int(ts[j])
        if upto < t:
            X = H[upto:t]
            S += X.T @ X
            upto = t
        h = H[t]
        out[j] = 0.5 * _logdet_spd(I + c * (S + np.outer(h, h))) - 0.5 * _logdet_spd(I + c * S)
    return out, S0 + H.T @ H
