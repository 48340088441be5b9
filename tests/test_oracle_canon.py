"""Pins of the Canon-convolution oracle (ByteFlow notes, "Key design 1"; summary,
"Method steps", stage 1: Canon = causal_conv1d with kernel 4).

The convolution is pinned by its impulse and step responses (closed forms), by
an independent FIR filter from scipy, by row isolation and causality; the
rounding to bfloat16 by hand-worked ties and by brute force over the
neighbouring bfloat16 values.
"""
import numpy as np
import pytest
from scipy.signal import lfilter

from oracle.canon import KERNEL, canon_conv, canon_conv_bf16, canon_conv_f32, round_bf16


def _bf16_vals(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    u = x.view(np.uint32) & np.uint32(0xFFFF0000)        # truncate to bf16-representable values
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- convolution
def test_impulse_response_is_the_kernel():
    d, T = 5, 12
    rng = np.random.default_rng(0)
    w = _bf16_vals(rng, (d, KERNEL))
    for t0 in (0, 3, 9):
        for f in range(d):
            H = np.zeros((T, d))
            H[t0, f] = 2.0
            out = canon_conv(H, np.array([0, T]), w)
            want = np.zeros((T, d))
            for j in range(KERNEL):
                if t0 + j < T:
                    want[t0 + j, f] = 2.0 * w[f, j]
            assert np.array_equal(out, want)


def test_step_response_partial_sums_then_full_sum():
    d, T = 3, 10
    rng = np.random.default_rng(1)
    w = _bf16_vals(rng, (d, KERNEL))
    b = _bf16_vals(rng, (d,))
    a = np.array([0.5, -1.25, 3.0])
    H = np.tile(a, (T, 1))
    out = canon_conv(H, np.array([0, T]), w, bias=b)
    for t in range(T):
        want = b + a * w[:, :min(t + 1, KERNEL)].sum(axis=1)
        assert np.allclose(out[t], want, rtol=0, atol=1e-12)


def test_matches_an_fir_filter_per_channel():
    d, T = 7, 200
    rng = np.random.default_rng(2)
    H = _bf16_vals(rng, (T, d))
    w = _bf16_vals(rng, (d, KERNEL))
    out = canon_conv(H, np.array([0, T]), w)
    for f in range(d):
        ref = lfilter(w[f], [1.0], H[:, f])
        assert np.allclose(out[:, f], ref, rtol=0, atol=1e-12)


def test_rows_are_isolated_and_causal():
    d = 4
    rng = np.random.default_rng(3)
    lens = [5, 1, 0, 9, 2]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    H = _bf16_vals(rng, (int(offs[-1]), d))
    w = _bf16_vals(rng, (d, KERNEL))
    out = canon_conv(H, offs, w, residual=True)
    for r, n in enumerate(lens):
        a = offs[r]
        alone = canon_conv(H[a:a + n], np.array([0, n]), w, residual=True)
        assert np.array_equal(out[a:a + n], alone)
    # causality: changing position t only moves outputs t .. t+3 of the same row
    H2 = H.copy()
    H2[offs[3] + 4] += 1.0
    out2 = canon_conv(H2, offs, w)
    diff = np.nonzero(np.any(out2 != canon_conv(H, offs, w), axis=1))[0]
    assert set(diff.tolist()) <= set(range(offs[3] + 4, offs[3] + 8))


def test_residual_adds_the_input():
    rng = np.random.default_rng(4)
    H = _bf16_vals(rng, (30, 6))
    w = _bf16_vals(rng, (6, KERNEL))
    offs = np.array([0, 11, 30])
    assert np.array_equal(canon_conv(H, offs, w, residual=True), H + canon_conv(H, offs, w))


# ---------------------------------------------------------------- rounding
def test_round_bf16_hand_worked_ties():
    one = 1.0
    cases = [
        (one + 2.0 ** -8, 1.0),                       # halfway, even neighbour 1.0
        (one + 3 * 2.0 ** -8, one + 2.0 ** -6),       # halfway, even neighbour 1 + 2^-6
        (one + 2.0 ** -8 + 2.0 ** -40, one + 2.0 ** -7),   # just above halfway (a float32 detour would tie)
        (-(one + 2.0 ** -8), -1.0),
        (0.0, 0.0),
        (3.0, 3.0),
    ]
    x = np.array([c[0] for c in cases])
    got = round_bf16(x)
    want = (np.array([c[1] for c in cases], dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(got, want)


def test_round_bf16_is_the_nearest_value_by_brute_force():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(4000) * np.exp(rng.uniform(-8, 8, 4000))
    got = round_bf16(x)
    gv = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # candidates: the truncated pattern and its neighbours
    t = (x.astype(np.float32).view(np.uint32) >> 16).astype(np.int64)
    best = np.empty_like(x)
    for i in range(len(x)):
        cands = [((int(t[i]) + k) & 0xFFFF) for k in (-2, -1, 0, 1, 2)]
        vals = np.array([(np.uint32(c) << np.uint32(16)).view(np.float32) for c in cands], dtype=np.float64)
        dist = np.abs(vals - x[i])
        m = dist.min()
        tied = [c for c, dd in zip(cands, dist) if dd == m]
        pick = [c for c in tied if c % 2 == 0] if len(tied) > 1 else tied
        best[i] = np.float64((np.uint32(pick[0]) << np.uint32(16)).view(np.float32))
    assert np.array_equal(gv, best)


def test_bf16_output_is_the_rounded_exact_value():
    rng = np.random.default_rng(6)
    H = _bf16_vals(rng, (64, 8), 0.1)
    w = _bf16_vals(rng, (8, KERNEL), 0.5)
    b = _bf16_vals(rng, (8,), 0.01)
    offs = np.array([0, 20, 64])
    bits = canon_conv_bf16(H, offs, w, b, residual=True)
    exact = canon_conv(H, offs, w, b, residual=True)
    back = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # within half a bfloat16 step of the exact value
    assert np.all(np.abs(back - exact) <= np.abs(exact) * 2.0 ** -8 + 1e-300)


@pytest.mark.parametrize("mutant", ["anticausal", "dropped_tap", "no_row_reset"])
def test_plausible_mistakes_fail_the_pins(mutant):
    d, T = 2, 10
    w = np.array([[1.0, 2.0, 4.0, 8.0], [0.5, 0.25, 0.125, 0.0625]])
    H = np.zeros((T, d))
    H[0, 0] = 1.0                                  # impulse at a row start: taps 0..3 land inside the row
    H[5, 1] = 1.0                                  # impulse at the last position of the first row
    offs = np.array([0, 6, T])                     # rows [0, 6) and [6, 10)
    out = np.zeros((T, d))
    for j in range(KERNEL):
        if mutant == "dropped_tap" and j == 3:
            continue
        if mutant == "anticausal":
            out[:T - j] += w[:, j] * H[j:]
        else:
            out[j:] += w[:, j] * H[:T - j]          # the whole batch as one sequence
    if mutant != "no_row_reset":
        out[6:] = 0.0                              # nothing reaches the second row for the other mutants
    assert not np.array_equal(out, canon_conv(H, offs, w))


def test_float32_order_is_within_a_rounding_of_the_exact_value():
    """The kernel-order float32 accumulation rounds to the same bfloat16 as the exact value
    except next to a rounding boundary, and is never more than one bfloat16 step away."""
    rng = np.random.default_rng(7)
    H = _bf16_vals(rng, (4000, 16), 0.06)
    w = _bf16_vals(rng, (16, KERNEL), 0.5)
    b = _bf16_vals(rng, (16,), 0.02)
    offs = np.array([0, 1500, 1501, 4000])
    for res in (False, True):
        got = canon_conv_f32(H, offs, w, b, residual=res)
        exact = canon_conv(H, offs, w, b, residual=res)
        ref = round_bf16(exact)
        gv = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        assert np.all(np.abs(gv - exact) <= np.abs(exact) * 2.0 ** -7 + 1e-30)
        assert np.mean(got == ref) > 0.999
