"""Boundary selection, gather and multi-linear upsampling (float64 / exact).

Sources (ByteFlow, arXiv 2603.03583):
* Selection: papernotes.org notes, "Key design 2", and paper.rainbus.top
  summary, "Method steps", stage 2: position 1 (BOS) is always kept; the K-1
  positions of largest dR among t = 2..T are added; the K boundaries are sorted
  in time.  The pages give no tie rule; the reading here is larger dR first,
  then the earlier position (a stable sort).  K >= T keeps every position.
* Gather: summary, stage 2: z_k = h_{s_k} (then times W_proj).
* Upsampling: summary, stage 4, and notes, "Key design 4": chunk of t is the
  last boundary at or before t; s~_t = g_c W_{b(t)}; s_t = h_t + s~_t with
  B = 16 bins, one W per bin.  The bin rule is read three ways (the pages
  disagree): OFFSET b = min(t - s_c, B-1) ("relative position within its
  chunk", the default), FRACTION b = floor(B (t - s_c) / L_c) with L_c the
  chunk length, ABSOLUTE b = floor(t B / T) (the summary's b = floor(t/(T/B)),
  0-based).

Backward (gradients of the upsampling for training with the chunker; the
selection itself passes no gradient, notes "Key design 2"): with dS = dL/dS,
  dL/dg_k  = sum over t in chunk k of W_{b(t)} dS_t,
  dL/dW_b  = sum over t in bin b of g_{c(t)} (outer) dS_t,
  dL/dh_t  = dS_t (the residual), and through the gather z_k = h_{s_k} the
  chunk gradient returns to the boundary rows, dL/dh_{s_k} += dL/dz_k.

All positions are 0-based.  Test infrastructure only.
"""
from __future__ import annotations

import numpy as np

__all__ = ["topk_select", "topk_select_rows", "gather", "chunk_of", "bin_of",
           "upsample_row", "upsample", "upsample_backward_row", "upsample_backward", "gather_backward",
           "BIN_OFFSET", "BIN_FRACTION", "BIN_ABSOLUTE"]

BIN_OFFSET, BIN_FRACTION, BIN_ABSOLUTE = 0, 1, 2


def topk_select(dR: np.ndarray, K: int) -> np.ndarray:
    """Boundary positions of one row: {0} plus the K-1 largest dR over t >= 1.

    Equal dR values are ordered by position (earlier first).  Returns int64
    positions in increasing order, exactly min(K, T) of them.
    """
    dR = np.asarray(dR)
    T = dR.shape[0]
    if K < 1:
        raise ValueError("K must be >= 1")
    if K >= T:
        return np.arange(T, dtype=np.int64)
    t = np.arange(1, T)
    # lexsort: last key is primary -> sort by -dR, then by t
    order = np.lexsort((t, -dR[1:].astype(np.float64)))
    chosen = t[order[:K - 1]]
    return np.concatenate([[0], np.sort(chosen)]).astype(np.int64)


def topk_select_rows(dR: np.ndarray, offsets: np.ndarray, K) -> tuple:
    """Per-row selection over a packed batch; returns (idx, idx_offsets)."""
    rows = len(offsets) - 1
    Ks = np.broadcast_to(np.asarray(K, dtype=np.int64), (rows,))
    parts, io = [], np.zeros(rows + 1, dtype=np.int64)
    for r in range(rows):
        a, b = offsets[r], offsets[r + 1]
        sel = topk_select(dR[a:b], int(Ks[r]))
        parts.append(sel)
        io[r + 1] = io[r] + len(sel)
    idx = np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)
    return idx, io


def gather(H: np.ndarray, offsets: np.ndarray, idx: np.ndarray,
           idx_offsets: np.ndarray) -> np.ndarray:
    """z_k = h_{s_k} per row (row-relative positions), rows stacked."""
    out = np.empty((len(idx), H.shape[1]), dtype=H.dtype)
    for r in range(len(offsets) - 1):
        a, b = idx_offsets[r], idx_offsets[r + 1]
        out[a:b] = H[offsets[r] + idx[a:b]]
    return out


def chunk_of(idx_row: np.ndarray, T: int) -> np.ndarray:
    """c(t) = max{k : s_k <= t} for t = 0..T-1 (s_0 = 0 so always defined)."""
    return np.searchsorted(idx_row, np.arange(T), side="right") - 1


def bin_of(idx_row: np.ndarray, T: int, nbins: int, mode: int) -> np.ndarray:
    """Bin index of every position of one row under the given bin rule."""
    t = np.arange(T, dtype=np.int64)
    c = chunk_of(idx_row, T)
    start = idx_row[c]
    if mode == BIN_OFFSET:
        return np.minimum(t - start, nbins - 1)
    if mode == BIN_FRACTION:
        nxt = np.append(idx_row[1:], T)
        length = nxt[c] - start
        return (nbins * (t - start)) // length
    if mode == BIN_ABSOLUTE:
        return (t * nbins) // T
    raise ValueError("unknown bin mode")


def upsample_row(G: np.ndarray, H: np.ndarray, idx_row: np.ndarray,
                 W_bin: np.ndarray, mode: int) -> np.ndarray:
    """s_t = h_t + g_{c(t)} W_{b(t)} for one row, float64.

    G [K, d_g] chunk vectors, H [T, d_l], W_bin [B, d_g, d_l].
    """
    T = H.shape[0]
    B = W_bin.shape[0]
    c = chunk_of(idx_row, T)
    b = bin_of(idx_row, T, B, mode)
    G = np.asarray(G, dtype=np.float64)
    W = np.asarray(W_bin, dtype=np.float64)
    out = np.asarray(H, dtype=np.float64).copy()
    for t in range(T):
        out[t] += G[c[t]] @ W[b[t]]
    return out


def upsample(G, H, offsets, idx, idx_offsets, W_bin, mode=BIN_OFFSET, rows=None):
    """Row-by-row upsampling of a packed batch (``rows`` limits to a subset)."""
    rows = range(len(offsets) - 1) if rows is None else rows
    outs = []
    for r in rows:
        a, b = offsets[r], offsets[r + 1]
        ia, ib = idx_offsets[r], idx_offsets[r + 1]
        outs.append(upsample_row(G[ia:ib], H[a:b], idx[ia:ib], W_bin, mode))
    return outs


def upsample_backward_row(G: np.ndarray, idx_row: np.ndarray, W_bin: np.ndarray,
                          dS: np.ndarray, mode: int):
    """Gradients of one row's s_t = h_t + g_{c(t)} W_{b(t)} given dS_t, float64.

    Returns (dG [K, d_g], dW [B, d_g, d_l] of this row, dH [T, d_l]).  One
    position at a time, straight from the chain rule.
    """
    T = dS.shape[0]
    B = W_bin.shape[0]
    c = chunk_of(idx_row, T)
    b = bin_of(idx_row, T, B, mode)
    G = np.asarray(G, dtype=np.float64)
    W = np.asarray(W_bin, dtype=np.float64)
    dS = np.asarray(dS, dtype=np.float64)
    dG = np.zeros_like(G)
    dW = np.zeros_like(W)
    for t in range(T):
        dG[c[t]] += W[b[t]] @ dS[t]
        dW[b[t]] += np.outer(G[c[t]], dS[t])
    return dG, dW, dS.copy()


def upsample_backward(G, offsets, idx, idx_offsets, W_bin, dS, mode=BIN_OFFSET):
    """Packed batch: (dG [sum K, d_g], dW summed over rows, dH = dS)."""
    dG = np.zeros(np.shape(G), dtype=np.float64)
    dW = np.zeros(np.shape(W_bin), dtype=np.float64)
    for r in range(len(offsets) - 1):
        a, b = offsets[r], offsets[r + 1]
        ia, ib = idx_offsets[r], idx_offsets[r + 1]
        if ib == ia:
            continue
        g, w, _ = upsample_backward_row(G[ia:ib], idx[ia:ib], W_bin, dS[a:b], mode)
        dG[ia:ib] = g
        dW += w
    return dG, dW, np.asarray(dS, dtype=np.float64).copy()


def gather_backward(dZ, offsets, idx, idx_offsets, N):
    """Adjoint of the gather: dH [N, d] with dH[offsets_r + s_k] = dZ_k, zero elsewhere."""
    dZ = np.asarray(dZ, dtype=np.float64)
    dH = np.zeros((N, dZ.shape[1]), dtype=np.float64)
    for r in range(len(offsets) - 1):
        a, b = idx_offsets[r], idx_offsets[r + 1]
        dH[offsets[r] + idx[a:b]] += dZ[a:b]
    return dH
