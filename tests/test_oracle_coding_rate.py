"""Pins of the float64 coding-rate oracle against closed forms and invariants.

The three oracle evaluations (prefix logdet, Cholesky diagonal of the T x T
Gram, rank-1 recursion in C) are checked against each other, and each against
results fixed by the mathematics of R_eps(H) = 1/2 logdet(I + (d/eps^2) H H^T)
(ByteFlow summary, "Prerequisites: lossy coding rate") and
dR_t = R(h_{1:t}) - R(h_{1:t-1}) (same page, "Method steps", stage 2).
"""
import math

import numpy as np
import pytest

import oracle
from oracle.coding_rate import coding_rate, coding_rate_T, dR_chol_diag, dR_prefix_logdet
from oracle.rank1 import dR_rank1


def _all3(H, eps2):
    H = np.asarray(H, dtype=np.float32)
    offs = np.array([0, H.shape[0]], dtype=np.int64)
    return (dR_prefix_logdet(H, eps2), dR_chol_diag(H, eps2), dR_rank1(H, offs, eps2))


def _rel(a, b):
    return float(np.max(np.abs(a - b) / np.maximum(np.abs(b), 1e-300)))


# ---------------------------------------------------------------- definitions
def test_sylvester_matches_pages_TxT_form():
    rng = np.random.default_rng(11)
    for T, d in [(5, 9), (9, 5), (16, 16), (40, 7)]:
        H = rng.standard_normal((T, d)) / math.sqrt(d)
        for eps2 in (0.5, 0.25, 2.0):
            a, b = coding_rate(H, eps2), coding_rate_T(H, eps2)
            assert abs(a - b) <= 1e-11 * max(1.0, abs(b))


def test_three_oracles_agree_tiny_workload():
    import workloads
    w = workloads.make("tiny")
    a, b, c = _all3(w.row(0), w.eps2)
    assert _rel(a, b) < 1e-9 and _rel(c, b) < 1e-9


@pytest.mark.parametrize("T,d,eps2", [(1, 4, 0.5), (7, 3, 0.5), (30, 8, 0.25),
                                      (64, 16, 1.0), (50, 50, 0.5), (3, 64, 0.5)])
def test_three_oracles_agree_random(T, d, eps2):
    rng = np.random.default_rng(T * 1000 + d)
    H = (rng.standard_normal((T, d)) / math.sqrt(d)).astype(np.float32)
    a, b, c = _all3(H, eps2)
    assert _rel(a, b) < 1e-9 and _rel(c, b) < 1e-9


# ---------------------------------------------------------------- closed forms
def test_orthogonal_rows_closed_form():
    # mutually orthogonal h_t: each is new information, dR_t = 1/2 log(1 + c|h_t|^2)
    rng = np.random.default_rng(1)
    d, T, eps2 = 16, 12, 0.5
    c = d / eps2
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    alpha = rng.uniform(0.1, 2.0, size=T)
    H = (Q[:, :T].T * alpha[:, None])
    want = 0.5 * np.log1p(c * alpha ** 2)
    assert _rel(dR_chol_diag(H, eps2), want) < 1e-10
    assert _rel(dR_prefix_logdet(H, eps2), want) < 1e-10
    # O3 reads float32 inputs: compare on the float32-rounded rows
    H32 = H.astype(np.float32).astype(np.float64)
    _, b, c3 = _all3(H32, eps2)
    assert _rel(c3, b) < 1e-9


def test_repeated_vector_closed_form():
    # h_t = v for all t, a = |v|^2: by Sherman-Morrison
    # dR_t = 1/2 log((1 + c (t+1) a) / (1 + c t a))   (0-based t)
    d, T, eps2 = 8, 25, 0.5
    c = d / eps2
    v = np.array([0.5, -0.25, 0.125, 1.0, -0.75, 0.0, 0.375, 0.25])  # exact in fp32
    a = float(v @ v)
    H = np.tile(v, (T, 1))
    t = np.arange(T)
    want = 0.5 * np.log((1 + c * (t + 1) * a) / (1 + c * t * a))
    for got in _all3(H, eps2):
        assert _rel(got, want) < 1e-9
    # prefix rate R_t = 1/2 log(1 + c t a) (1-based count t)
    for n in (1, 5, T):
        assert abs(coding_rate(H[:n], eps2) - 0.5 * math.log1p(c * n * a)) < 1e-10


def test_axis_aligned_closed_form():
    # h_t = alpha_t e_{k(t)}: independent scalar problems per axis
    rng = np.random.default_rng(3)
    d, T, eps2 = 5, 40, 0.5
    c = d / eps2
    k = rng.integers(0, d, size=T)
    alpha = rng.choice([0.25, 0.5, 1.0, 1.5], size=T)
    H = np.zeros((T, d))
    H[np.arange(T), k] = alpha
    A = np.zeros(d)
    want = np.empty(T)
    for t in range(T):
        before = A[k[t]]
        A[k[t]] += alpha[t] ** 2
        want[t] = 0.5 * math.log((1 + c * A[k[t]]) / (1 + c * before))
    for got in _all3(H, eps2):
        assert _rel(got, want) < 1e-9


def test_two_vector_closed_form():
    # dR_1 = 1/2 log(1 + c(|v|^2 - c (u.v)^2 / (1 + c|u|^2)))
    u = np.array([0.5, 0.25, -0.5, 0.0])
    v = np.array([0.25, 0.75, 0.5, -0.25])
    d, eps2 = 4, 0.5
    c = d / eps2
    H = np.stack([u, v])
    want1 = 0.5 * math.log1p(c * (v @ v - c * (u @ v) ** 2 / (1 + c * (u @ u))))
    want0 = 0.5 * math.log1p(c * (u @ u))
    for got in _all3(H, eps2):
        assert abs(got[0] - want0) < 1e-12 and abs(got[1] - want1) < 1e-12


def test_scalar_d1_closed_form():
    rng = np.random.default_rng(5)
    T, eps2 = 30, 0.5
    c = 1 / eps2
    h = rng.choice([-1.0, -0.5, 0.25, 0.75, 2.0], size=T)
    S = np.cumsum(h ** 2)
    Sprev = np.concatenate([[0.0], S[:-1]])
    want = 0.5 * np.log((1 + c * S) / (1 + c * Sprev))
    for got in _all3(h[:, None], eps2):
        assert _rel(got, want) < 1e-10


# ---------------------------------------------------------------- invariants
def _H(seed, T=48, d=12):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((T, d)) / math.sqrt(d)).astype(np.float32).astype(np.float64)


def test_telescoping_equals_svd_rate():
    H = _H(7)
    eps2 = 0.5
    d = H.shape[1]
    c = d / eps2
    dR = dR_chol_diag(H, eps2)
    for n in (1, 5, 12, 13, 30, 48):
        sig2 = np.linalg.eigvalsh(H[:n].T @ H[:n])
        want = 0.5 * np.sum(np.log1p(c * np.clip(sig2, 0, None)))
        assert abs(np.sum(dR[:n]) - want) < 1e-9 * max(1, want)


def test_bounds():
    H = _H(8)
    eps2 = 0.5
    c = H.shape[1] / eps2
    for got in _all3(H, eps2):
        assert np.all(got >= -1e-12)
        assert np.all(got <= 0.5 * np.log1p(c * np.sum(H ** 2, axis=1)) + 1e-12)


def test_orthogonal_invariance_and_scaling():
    H = _H(9)
    eps2 = 0.5
    d = H.shape[1]
    Q, _ = np.linalg.qr(np.random.default_rng(1).standard_normal((d, d)))
    base = dR_chol_diag(H, eps2)
    assert _rel(dR_chol_diag(H @ Q, eps2), base) < 1e-10
    # dR(H; eps^2) = dR(a H; a^2 eps^2): only c H H^T matters
    assert _rel(dR_chol_diag(3.0 * H, 9.0 * eps2), base) < 1e-10


def test_permuting_the_past_leaves_dR_t():
    H = _H(10)
    eps2 = 0.5
    t = 30
    rng = np.random.default_rng(2)
    P = H.copy()
    P[:t] = H[rng.permutation(t)]
    assert abs(dR_chol_diag(P, eps2)[t] - dR_chol_diag(H, eps2)[t]) < 1e-11


def test_sampled_prefix_logdet_matches_full():
    H = _H(12, T=64, d=10)
    eps2 = 0.25
    full = dR_chol_diag(H, eps2)
    ts = np.array([63, 0, 17, 5, 40])
    assert _rel(dR_prefix_logdet(H, eps2, ts), full[ts]) < 1e-9


def test_ragged_rows_are_independent():
    rng = np.random.default_rng(13)
    H = (rng.standard_normal((70, 6)) / math.sqrt(6)).astype(np.float32)
    offs = np.array([0, 10, 10, 45, 70], dtype=np.int64)   # includes an empty row
    got = dR_rank1(H, offs, 0.5)
    for r in range(4):
        a, b = offs[r], offs[r + 1]
        if b > a:
            assert _rel(got[a:b], dR_chol_diag(H[a:b].astype(np.float64), 0.5)) < 1e-9


# ---------------------------------------------------------------- mutants
# Plausible mistakes; each must fail at least one pin above.
def _mut_no_identity(H, eps2):
    T, d = H.shape
    G = (d / eps2) * (H @ H.T) + 1e-9 * np.eye(T)
    return np.log(np.diag(np.linalg.cholesky(G)))


def _mut_c_without_d(H, eps2):
    T, d = H.shape
    G = np.eye(T) + (1.0 / eps2) * (H @ H.T)
    return np.log(np.diag(np.linalg.cholesky(G)))


def _mut_full_log(H, eps2):       # drops the 1/2 of R
    return 2.0 * dR_chol_diag(H, eps2)


def _mut_shifted(H, eps2):        # dR_t reported at t+1
    x = dR_chol_diag(H, eps2)
    return np.concatenate([[0.5 * math.log1p(H.shape[1] / eps2 * float(H[0] @ H[0]))], x[:-1]])


@pytest.mark.parametrize("mut", [_mut_no_identity, _mut_c_without_d, _mut_full_log, _mut_shifted])
def test_pins_catch_mutants(mut):
    d, T, eps2 = 8, 25, 0.5
    c = d / eps2
    v = np.array([0.5, -0.25, 0.125, 1.0, -0.75, 0.0, 0.375, 0.25])
    a = float(v @ v)
    H = np.tile(v, (T, 1))
    t = np.arange(T)
    want = 0.5 * np.log((1 + c * (t + 1) * a) / (1 + c * t * a))
    with np.errstate(all="ignore"):
        try:
            got = mut(H, eps2)
            bad = not np.all(np.isfinite(got)) or _rel(got, want) > 1e-6
        except np.linalg.LinAlgError:
            bad = True
    assert bad


# ---------------------------------------------------------------- streaming continuation
def test_continuation_matches_whole_sequence_by_other_oracles():
    """Blocks with a carried Gram sum give the whole sequence's dR (checked against the
    Cholesky diagonal of the T x T Gram and the rank-1 recursion, both independent of it)."""
    from oracle.coding_rate import dR_chol_diag, dR_continue
    from oracle.rank1 import dR_rank1
    rng = np.random.default_rng(7)
    d, eps2 = 16, 0.5
    H = (rng.standard_normal((150, d)) / np.sqrt(d)).astype(np.float32).astype(np.float64)   # the C oracle reads fp32
    want = dR_chol_diag(H, eps2)
    want3 = dR_rank1(H, np.array([0, 150]), eps2)
    S = np.zeros((d, d))
    got = []
    for a, b in [(0, 1), (1, 40), (40, 41), (41, 150)]:      # blocks of 1, 39, 1, 109 positions
        dr, S = dR_continue(S, H[a:b], eps2)
        got.append(dr)
    got = np.concatenate(got)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-13)
    assert np.allclose(got, want3, rtol=1e-9, atol=1e-13)
    assert np.allclose(S, H.T @ H, rtol=1e-13, atol=1e-13)


def test_continuation_sampled_positions_and_empty_prefix():
    from oracle.coding_rate import dR_continue, dR_prefix_logdet
    rng = np.random.default_rng(8)
    d, eps2 = 8, 0.25
    H = rng.standard_normal((60, d)) / np.sqrt(d)
    full, _ = dR_continue(np.zeros((d, d)), H, eps2)
    # a zero prefix is the plain definition
    assert np.allclose(full, dR_prefix_logdet(H, eps2), rtol=1e-12, atol=1e-14)
    S20 = H[:20].T @ H[:20]
    part, _ = dR_continue(S20, H[20:], eps2, ts=[0, 13, 39])
    assert np.allclose(part, full[[20, 33, 59]], rtol=1e-12, atol=1e-14)
    # a later byte never gains information: dR of a repeat is smaller than on a fresh state
    again, _ = dR_continue(H.T @ H, H[:1], eps2)
    fresh, _ = dR_continue(np.zeros((d, d)), H[:1], eps2)
    assert again[0] < fresh[0]
