"""Canon layer of the local encoder: causal depthwise convolution, kernel 4 (float64).

Sources: the ByteFlow notes (papernotes.org), "Key design 1": every local-encoder
layer inserts a Canon layer, in essence a causal one-dimensional convolution
with kernel size 4, which mixes neighbouring bytes at almost no cost; the
ByteFlow summary (paper.rainbus.top), "Method steps", stage 1: each block of
the local encoder is SWA(w_local) + Canon(causal_conv1d, k = 4) + SwiGLU and
its output h_{1:T} feeds the coding-rate chunker.

The pages give no formula beyond "causal 1-D convolution, kernel 4".  The
reading taken is the per-channel (depthwise) causal convolution, each row of a
packed batch on its own (positions before a row's first position count as 0):

    u_t[f] = bias[f] + sum_{j=0..3} w[f, j] h_{t-j}[f]
    out_t  = u_t                 (residual = False)
    out_t  = h_t + u_t           (residual = True)

evaluated exactly in float64 (the inputs are bfloat16 values, so every product
is exact and so is the short sum) and rounded once to bfloat16, round to
nearest with ties to even.

The rounding to bfloat16 turns the value into the chunker's input bits, a
decision that both sides take in the kernel's precision: ``canon_conv_f32``
accumulates in float32 in the kernel's fixed order (bias, residual, taps 0..3;
each product of two bfloat16 values is exact in float32 and each addition
rounds once) before the same rounding.  Its pins tie it to the exact value.

Test infrastructure only.
"""
from __future__ import annotations

import numpy as np

__all__ = ["canon_conv", "round_bf16", "canon_conv_bf16", "canon_conv_f32"]

KERNEL = 4


def canon_conv(H: np.ndarray, offsets: np.ndarray, w: np.ndarray, bias=None,
               residual: bool = False) -> np.ndarray:
    """Unrounded float64 output [N, d] of the Canon convolution over the packed rows."""
    H = np.asarray(H, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    N, d = H.shape
    assert w.shape == (d, KERNEL)
    out = np.zeros((N, d), dtype=np.float64)
    if bias is not None:
        out += np.asarray(bias, dtype=np.float64)[None, :]
    if residual:
        out += H
    offsets = np.asarray(offsets, dtype=np.int64)
    for r in range(len(offsets) - 1):
        a, b = int(offsets[r]), int(offsets[r + 1])
        for j in range(KERNEL):
            # term j: w[:, j] times the input j positions earlier in the same row
            if b - a > j:
                out[a + j:b] += w[:, j][None, :] * H[a:b - j]
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> bfloat16 bit patterns (uint16), one rounding, nearest with ties to even.

    bfloat16 keeps 7 of float64's 52 fraction bits; the 45 dropped bits decide the
    rounding.  Finite, normal-range values only (the workloads' magnitudes)."""
    u = np.ascontiguousarray(x, dtype=np.float64).view(np.uint64)
    drop = np.uint64(45)
    keep_lsb = (u >> drop) & np.uint64(1)
    u = u + (np.uint64((1 << 44) - 1) + keep_lsb)
    u = u & ~np.uint64((1 << 45) - 1)
    # the rounded value has at most 8 significant bits: exact in float32, whose top half is bfloat16
    f = u.view(np.float64).astype(np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def canon_conv_bf16(H, offsets, w, bias=None, residual=False) -> np.ndarray:
    """The Canon output as bfloat16 bit patterns [N, d] (what the chunker consumes)."""
    return round_bf16(canon_conv(H, offsets, w, bias, residual))


def canon_conv_f32(H, offsets, w, bias=None, residual: bool = False) -> np.ndarray:
    """bfloat16 bit patterns [N, d] of the convolution accumulated in float32 in the fixed order
    bias, residual, tap 0, 1, 2, 3, then rounded to nearest-even bfloat16."""
    H = np.asarray(H, dtype=np.float32)
    w = np.asarray(w, dtype=np.float32)
    N, d = H.shape
    acc = np.zeros((N, d), dtype=np.float32)
    if bias is not None:
        acc += np.asarray(bias, dtype=np.float32)[None, :]
    if residual:
        acc = (acc + H).astype(np.float32)
    offsets = np.asarray(offsets, dtype=np.int64)
    for j in range(KERNEL):
        shifted = np.zeros((N, d), dtype=np.float32)          # h_{t-j} within the row, else 0
        for r in range(len(offsets) - 1):
            a, b = int(offsets[r]), int(offsets[r + 1])
            if b - a > j:
                shifted[a + j:b] = H[a:b - j]
        prod = (w[:, j][None, :] * shifted).astype(np.float32)   # exact: 8-bit x 8-bit significands
        acc = (acc + prod).astype(np.float32)                     # one rounding, as the kernel's fma
    u = acc.view(np.uint32)
    bias_bits = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias_bits) >> np.uint32(16)).astype(np.uint16)
