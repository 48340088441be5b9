"""Pins of the backward oracle of the upsampling and the gather.

ByteFlow (paper.rainbus.top summary, "Method steps", stage 4; papernotes.org
notes, "Key design 4"): s_t = h_t + g_{c(t)} W_{b(t)}.  The output is linear in
G for fixed W and linear in W for fixed G, so a central difference of
L = sum_t <dS_t, s_t> along any direction equals the directional derivative
exactly (up to float64 rounding).  The pins below compare the hand-written
backward against such differences of the (separately pinned) forward oracle,
element by element on tiny cases, and against closed forms.
"""
import numpy as np
import pytest

from oracle.chunking import (BIN_ABSOLUTE, BIN_FRACTION, BIN_OFFSET, chunk_of, gather, gather_backward,
                             upsample, upsample_backward, upsample_backward_row, upsample_row)

MODES = [BIN_OFFSET, BIN_FRACTION, BIN_ABSOLUTE]


def _loss(G, H, s, W, dS, mode):
    return float(np.sum(dS * upsample_row(G, H, s, W, mode)))


@pytest.mark.parametrize("mode", MODES)
def test_every_partial_derivative_by_central_difference(mode):
    rng = np.random.default_rng(10 + mode)
    T, B, dg, dl = 41, 16, 3, 2
    s = np.array([0, 1, 5, 6, 24], dtype=np.int64)          # lengths 1, 4, 1, 18, 17 (bin 15 tails)
    G = rng.standard_normal((len(s), dg))
    W = rng.standard_normal((B, dg, dl))
    H = rng.standard_normal((T, dl))
    dS = rng.standard_normal((T, dl))
    dG, dW, dH = upsample_backward_row(G, s, W, dS, mode)
    for i in np.ndindex(G.shape):
        E = np.zeros_like(G)
        E[i] = 1.0
        fd = (_loss(G + E, H, s, W, dS, mode) - _loss(G - E, H, s, W, dS, mode)) / 2
        assert abs(fd - dG[i]) <= 1e-12 * max(1.0, abs(fd)), (i, fd, dG[i])
    for i in np.ndindex(W.shape):
        E = np.zeros_like(W)
        E[i] = 1.0
        fd = (_loss(G, H, s, W + E, dS, mode) - _loss(G, H, s, W - E, dS, mode)) / 2
        assert abs(fd - dW[i]) <= 1e-12 * max(1.0, abs(fd)), (i, fd, dW[i])
    for i in [(0, 0), (17, 1), (40, 0)]:
        E = np.zeros_like(H)
        E[i] = 1.0
        fd = (_loss(G, H + E, s, W, dS, mode) - _loss(G, H - E, s, W, dS, mode)) / 2
        assert abs(fd - dH[i]) <= 1e-12 * max(1.0, abs(fd))


def test_shared_weight_closed_form():
    # every bin with the same W: dG_k = W (sum of dS over chunk k), dW_b = sum over bin b of g (outer) dS
    rng = np.random.default_rng(3)
    T, B, d = 50, 16, 4
    s = np.array([0, 3, 4, 30], dtype=np.int64)
    G = rng.standard_normal((len(s), d))
    Wone = rng.standard_normal((d, d))
    W = np.broadcast_to(Wone, (B, d, d)).copy()
    dS = rng.standard_normal((T, d))
    dG, dW, _ = upsample_backward_row(G, s, W, dS, BIN_OFFSET)
    c = chunk_of(s, T)
    for k in range(len(s)):
        want = Wone @ dS[c == k].sum(axis=0)
        assert np.allclose(dG[k], want, rtol=1e-13, atol=1e-13)
    # sum over bins of dW = G^T-weighted sum over all positions
    assert np.allclose(dW.sum(axis=0), G[c].T @ dS, rtol=1e-12, atol=1e-12)


def test_offset_bins_single_positions():
    # offset mode: bin b < 15 of chunk k is the single position s_k + b
    rng = np.random.default_rng(4)
    T, B, d = 30, 16, 3
    s = np.array([0, 20], dtype=np.int64)                    # chunk 0 of length 20, chunk 1 of 10
    G = rng.standard_normal((2, d))
    W = rng.standard_normal((B, d, d))
    dS = rng.standard_normal((T, d))
    _, dW, _ = upsample_backward_row(G, s, W, dS, BIN_OFFSET)
    assert np.allclose(dW[3], np.outer(G[0], dS[3]) + np.outer(G[1], dS[23]), rtol=1e-13, atol=1e-13)
    assert np.allclose(dW[12], np.outer(G[0], dS[12]), rtol=1e-13, atol=1e-13)
    assert np.allclose(dW[15], np.outer(G[0], dS[15:20].sum(axis=0)), rtol=1e-13, atol=1e-13)


def test_packed_rows_sum_weight_gradients():
    rng = np.random.default_rng(5)
    B, d = 16, 4
    offs = np.array([0, 25, 25, 61], dtype=np.int64)           # an empty row in the middle
    idx = np.array([0, 7, 8, 0, 1, 33], dtype=np.int64)
    io = np.array([0, 3, 3, 6], dtype=np.int64)
    G = rng.standard_normal((6, d))
    W = rng.standard_normal((B, d, d))
    dS = rng.standard_normal((61, d))
    for mode in MODES:
        dG, dW, dH = upsample_backward(G, offs, idx, io, W, dS, mode)
        g0, w0, _ = upsample_backward_row(G[:3], idx[:3], W, dS[:25], mode)
        g2, w2, _ = upsample_backward_row(G[3:], idx[3:], W, dS[25:], mode)
        assert np.allclose(dG, np.concatenate([g0, g2]), rtol=0, atol=0)
        assert np.allclose(dW, w0 + w2, rtol=1e-15, atol=1e-15)
        assert np.array_equal(dH, dS)
        # adjoint identity of the whole packed map: <dS, S(G) - H> = <dG, G> (S - H is linear in G)
        S = upsample(G, np.zeros((61, d)), offs, idx, io, W, mode)
        lhs = sum(float(np.sum(dS[offs[r]:offs[r + 1]] * S[j])) for j, r in enumerate(range(3)))
        assert abs(lhs - float(np.sum(dG * G))) <= 1e-12 * max(1.0, abs(lhs))


def test_gather_backward_is_the_adjoint():
    rng = np.random.default_rng(6)
    offs = np.array([0, 10, 30], dtype=np.int64)
    idx = np.array([0, 4, 9, 0, 2, 3, 19], dtype=np.int64)
    io = np.array([0, 3, 7], dtype=np.int64)
    H = rng.standard_normal((30, 5))
    dZ = rng.standard_normal((7, 5))
    dH = gather_backward(dZ, offs, idx, io, 30)
    assert abs(float(np.sum(gather(H, offs, idx, io) * dZ)) - float(np.sum(H * dH))) <= 1e-12
    # rows that are no boundary get nothing; boundary rows get exactly their chunk's gradient
    assert np.array_equal(dH[10 + 2], dZ[4]) and np.all(dH[1] == 0)
