"""H-Net style cosine router and EMA smoothing (float64).

Sources: the ByteGen analysis report (fudan.bigquant.com), "H-Net architecture
and its core components" and "Methodology": the dynamic chunking module
predicts a boundary from the cosine similarity of adjacent byte
representations and uses exponentially weighted smoothing so the discrete
boundaries can be trained end to end.  The pages give no formula; the reading
taken is

  q_t = h_t W_q,  k_t = h_t W_k                (row vectors, W [d, d])
  p_t = 1/2 (1 - cos(q_t, k_{t-1})),  p_0 = 1  (the first byte opens a chunk)
  b_t = [p_t >= 1/2]                            (inclusive threshold)

with cos = 0 when either norm is zero.  The smoothing runs over the router's
chunks k = 0..n-1 (boundary positions t_k, chunk vector z^_k = h_{t_k},
P_k = p_{t_k}):

  zbar_0 = z^_0 (P_0 = 1),  zbar_k = P_k z^_k + (1 - P_k) zbar_{k-1}.

Test infrastructure only.
"""
from __future__ import annotations

import numpy as np

__all__ = ["route_row", "ema", "route"]


def route_row(H: np.ndarray, Wq: np.ndarray, Wk: np.ndarray,
              threshold: float = 0.5):
    """(p [T] float64, boundary [T] bool, chunk positions [n] int64) of one row."""
    H = np.asarray(H, dtype=np.float64)
    q = H @ np.asarray(Wq, dtype=np.float64)
    k = H @ np.asarray(Wk, dtype=np.float64)
    T = H.shape[0]
    p = np.empty(T, dtype=np.float64)
    p[0] = 1.0
    for t in range(1, T):
        nq = np.sqrt(q[t] @ q[t])
        nk = np.sqrt(k[t - 1] @ k[t - 1])
        cos = 0.0 if (nq == 0.0 or nk == 0.0) else (q[t] @ k[t - 1]) / (nq * nk)
        p[t] = 0.5 * (1.0 - cos)
    b = p >= threshold
    return p, b, np.nonzero(b)[0].astype(np.int64)


def ema(zhat: np.ndarray, P: np.ndarray) -> np.ndarray:
    """zbar_k = P_k zhat_k + (1 - P_k) zbar_{k-1}, zbar_{-1} = 0, float64."""
    zhat = np.asarray(zhat, dtype=np.float64)
    out = np.empty_like(zhat)
    prev = np.zeros(zhat.shape[1:], dtype=np.float64)
    for j in range(zhat.shape[0]):
        prev = P[j] * zhat[j] + (1.0 - P[j]) * prev
        out[j] = prev
    return out


def route(H, offsets, Wq, Wk, threshold=0.5, rows=None):
    """Per-row router + smoothing: list of (p, b, chunk_pos, zbar)."""
    rows = range(len(offsets) - 1) if rows is None else rows
    res = []
    for r in rows:
        h = H[offsets[r]:offsets[r + 1]]
        p, b, pos = route_row(h, Wq, Wk, threshold)
        zbar = ema(np.asarray(h, dtype=np.float64)[pos], p[pos])
        res.append((p, b, pos, zbar))
    return res
