"""Pins of the selection, gather, upsampling, router and EMA oracles.

Selection: ByteFlow notes "Key design 2" / summary stage 2 (BOS kept, K-1
largest dR over t >= 2, time order).  Upsampling: summary stage 4 and notes
"Key design 4".  Router and EMA: ByteGen report, "H-Net architecture".
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle.chunking import (BIN_ABSOLUTE, BIN_FRACTION, BIN_OFFSET, bin_of, chunk_of,
                             gather, topk_select, topk_select_rows, upsample_row)
from oracle.router import ema, route_row

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- Top-K
def _brute_topk(vals, K):
    """Max-sum subset of size K-1 of {1..T-1}; among equal sums the
    lexicographically smallest position tuple.  Integer values: exact sums."""
    T = len(vals)
    if K >= T:
        return list(range(T))
    best, best_key = None, None
    for sub in itertools.combinations(range(1, T), K - 1):
        s = sum(int(vals[i]) for i in sub)
        key = (-s, sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return [0] + list(best)


@pytest.mark.parametrize("seed", range(40))
def test_topk_brute_force_small(seed):
    rng = np.random.default_rng(seed)
    T = int(rng.integers(1, 13))
    K = int(rng.integers(1, T + 2))
    vals = rng.integers(0, 4, size=T)          # many ties
    got = topk_select(vals.astype(np.float64), K)
    assert list(got) == _brute_topk(vals, K)


def test_topk_contract():
    rng = np.random.default_rng(0)
    dR = rng.random(1000)
    for K in (1, 2, 17, 999, 1000, 1001, 5000):
        s = topk_select(dR, K)
        assert s[0] == 0 and len(s) == min(K, 1000)
        assert np.all(np.diff(s) > 0)
    with pytest.raises(ValueError):
        topk_select(dR, 0)
    # BOS never competes: a huge dR at 0 does not take a slot
    x = np.zeros(10); x[0] = 100.0; x[5] = 1.0
    assert list(topk_select(x, 2)) == [0, 5]


def test_topk_rows_packed():
    rng = np.random.default_rng(1)
    offs = np.array([0, 5, 5, 30], dtype=np.int64)
    dR = rng.random(30)
    idx, io = topk_select_rows(dR, offs, np.array([2, 3, 8]))
    assert list(io) == [0, 2, 2, 10]
    assert list(idx[2:10]) == list(topk_select(dR[5:30], 8))


def test_gather_is_indexing():
    H = np.arange(60, dtype=np.float32).reshape(20, 3)
    offs = np.array([0, 8, 20], dtype=np.int64)
    idx = np.array([0, 5, 0, 3, 11], dtype=np.int64)
    io = np.array([0, 2, 5], dtype=np.int64)
    z = gather(H, offs, idx, io)
    assert np.array_equal(z, H[[0, 5, 8, 11, 19]])


# ---------------------------------------------------------------- upsample
def test_bins_worked_example():
    g = json.load(open(os.path.join(GOLD, "bins_worked_example.json")))
    s = np.array(g["boundaries"], dtype=np.int64)
    T, B = g["T"], g["nbins"]
    assert list(chunk_of(s, T)) == g["chunk"]
    assert list(bin_of(s, T, B, BIN_OFFSET)) == g["bin_offset"]
    assert list(bin_of(s, T, B, BIN_FRACTION)) == g["bin_fraction"]
    assert list(bin_of(s, T, B, BIN_ABSOLUTE)) == g["bin_absolute"]


def test_chunk_of_brute_force():
    rng = np.random.default_rng(4)
    for _ in range(20):
        T = int(rng.integers(1, 60))
        s = np.sort(np.unique(np.concatenate([[0], rng.integers(0, T, size=5)])))
        c = chunk_of(s, T)
        for t in range(T):
            assert c[t] == max(k for k in range(len(s)) if s[k] <= t)


@pytest.mark.parametrize("mode", [BIN_OFFSET, BIN_FRACTION, BIN_ABSOLUTE])
def test_upsample_one_hot_tags_recover_bins(mode):
    # g_c = e_0 for every chunk and W_b[0, :] = b e_0 + e_1: output - h = (b, 1, 0..)
    T, B, d = 57, 16, 4
    s = np.array([0, 2, 3, 30, 50], dtype=np.int64)      # one chunk of length 27 > 16
    G = np.zeros((len(s), d)); G[:, 0] = 1.0
    W = np.zeros((B, d, d))
    for b in range(B):
        W[b, 0, 0] = b
        W[b, 0, 1] = 1.0
    H = np.zeros((T, d))
    out = upsample_row(G, H, s, W, mode)
    assert np.array_equal(out[:, 0], bin_of(s, T, B, mode).astype(np.float64))
    assert np.all(out[:, 1] == 1.0) and np.all(out[:, 2:] == 0.0)


def test_upsample_identity_weights():
    T, B, d = 30, 16, 5
    s = np.array([0, 4, 9, 10], dtype=np.int64)
    rng = np.random.default_rng(1)
    G, H = rng.standard_normal((len(s), d)), rng.standard_normal((T, d))
    W = np.broadcast_to(np.eye(d), (B, d, d))
    out = upsample_row(G, H, s, W, BIN_OFFSET)
    assert np.allclose(out, H + G[chunk_of(s, T)], rtol=0, atol=1e-15)


def test_upsample_bin15_broadcast():
    # positions at offset >= 15 inside one long chunk share one product
    T, B, d = 40, 16, 3
    s = np.array([0], dtype=np.int64)
    rng = np.random.default_rng(2)
    G = rng.standard_normal((1, d))
    W = rng.standard_normal((B, d, d))
    out = upsample_row(G, np.zeros((T, d)), s, W, BIN_OFFSET)
    assert np.allclose(out[15:], out[15]) and not np.allclose(out[14], out[15])


# ---------------------------------------------------------------- router
def test_router_special_angles():
    d = 4
    I = np.eye(d)
    h = np.array([[1.0, 2.0, 0.0, 0.0],
                  [1.0, 2.0, 0.0, 0.0],      # same as before -> p = 0
                  [-1.0, -2.0, 0.0, 0.0],    # opposite -> p = 1
                  [2.0, -1.0, 0.0, 0.0],     # orthogonal -> p = 1/2, a boundary
                  [0.0, 0.0, 0.0, 0.0],      # zero norm -> p = 1/2
                  [0.0, 0.0, 3.0, 0.0]])     # previous zero -> p = 1/2
    p, b, pos = route_row(h, I, I)
    assert np.allclose(p, [1.0, 0.0, 1.0, 0.5, 0.5, 0.5], atol=1e-15)
    assert list(b) == [True, False, True, True, True, True]
    assert list(pos) == [0, 2, 3, 4, 5]


def test_router_uses_both_projections():
    # q_t = h_t W_q against k_{t-1} = h_{t-1} W_k: a swap W_q <-> W_k changes p
    rng = np.random.default_rng(3)
    h = rng.standard_normal((6, 3))
    Wq, Wk = rng.standard_normal((3, 3)), rng.standard_normal((3, 3))
    p1, _, _ = route_row(h, Wq, Wk)
    q, k = h @ Wq, h @ Wk
    t = 4
    want = 0.5 * (1 - q[t] @ k[t - 1] / (np.linalg.norm(q[t]) * np.linalg.norm(k[t - 1])))
    assert abs(p1[t] - want) < 1e-14


def test_ema_closed_forms():
    rng = np.random.default_rng(5)
    z = rng.standard_normal((12, 3))
    assert np.allclose(ema(z, np.ones(12)), z)
    a = 0.3
    out = ema(z, np.full(12, a))
    for k in range(12):
        want = sum(a * (1 - a) ** (k - j) * z[j] for j in range(k + 1))
        assert np.allclose(out[k], want, atol=1e-14)
    P = rng.uniform(0, 1, size=12)
    P[0] = 1.0
    out = ema(z, P)
    for k in range(12):
        want = sum(z[j] * P[j] * np.prod(1 - P[j + 1:k + 1]) for j in range(k + 1))
        assert np.allclose(out[k], want, atol=1e-13)
