"""GPU parity of the Canon layer (causal depthwise conv, kernel 4) and of the
Canon + coding-rate call against the oracle.

ByteFlow notes "Key design 1" / summary "Method steps", stage 1.  The
convolution's output bits are the chunker's input, so they are compared
bit-exactly with the oracle's float32-order evaluation (the rounding decision
taken in the kernel's precision); the coding rate of that output is compared
with the float64 rank-1 oracle at the bf16-input tolerance and its boundaries
outside the tie band.
"""
import numpy as np
import pytest

import workloads
from oracle.canon import canon_conv_f32
from oracle.rank1 import dR_rank1
from parity_util import check_boundaries, check_dR
from oracle.chunking import topk_select

pytestmark = pytest.mark.gpu


def _bits_to_dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _dev_to_bits(t):
    import torch
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _weights(seed, d):
    rng = np.random.default_rng(seed)
    w = workloads.bf16_bits((rng.standard_normal((d, 4)) * 0.5).astype(np.float32))
    b = workloads.bf16_bits((rng.standard_normal(d) * 0.02).astype(np.float32))
    return w, b


def _run_canon(H_bits, offs, T, w_bits, b_bits, residual, ragged):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Hd = _bits_to_dev(H_bits)
    od = torch.from_numpy(offs).cuda() if ragged else None
    out = dbc.canon_conv1d(Hd, _bits_to_dev(w_bits), None if b_bits is None else _bits_to_dev(b_bits),
                           offsets=od, T=T, residual=residual, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return _dev_to_bits(out)


@pytest.mark.parametrize("d", [64, 128, 256, 512])
@pytest.mark.parametrize("residual", [False, True])
def test_canon_bit_exact_ragged_small(d, residual):
    rng = np.random.default_rng(d + residual)
    lens = [1, 2, 3, 4, 5, 0, 37, 70, 300, 33]          # short rows, an empty row, ragged tails
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N = int(offs[-1])
    H = workloads.bf16_bits((rng.standard_normal((N, d)) / np.sqrt(d)).astype(np.float32))
    w, b = _weights(d, d)
    got = _run_canon(H, offs, max(lens), w, b if residual else None, residual, ragged=True)
    ref = canon_conv_f32(workloads.bf16_to_f32(H), offs, workloads.bf16_to_f32(w),
                         workloads.bf16_to_f32(b) if residual else None, residual)
    assert np.array_equal(got, ref)


def test_canon_bit_exact_full_byteflow():
    wl = workloads.make("byteflow")
    w, b = _weights(11, wl.d)
    got = _run_canon(wl.H_bits, wl.offsets, wl.T, w, b, True, ragged=False)
    ref = canon_conv_f32(wl.H, wl.offsets, workloads.bf16_to_f32(w), workloads.bf16_to_f32(b), True)
    assert np.array_equal(got, ref)


def test_canon_then_coding_rate_matches_oracle():
    """chunk_coding_rate_canon on byteflow-shaped rows: Hc bit-exact, dR of Hc within the bf16
    tolerance of the float64 rank-1 oracle, boundaries exact outside the tie band."""
    import torch
    import dynamic_byte_chunking_b200 as dbc
    wl = workloads.make("byteflow", rows=2)
    w, b = _weights(12, wl.d)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Hd = _bits_to_dev(wl.H_bits).view(wl.rows, wl.T, wl.d)
    Hc, dR = dbc.chunk_coding_rate_canon(Hd, _bits_to_dev(w), wl.eps2, _bits_to_dev(b), residual=True,
                                         dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    hc = _dev_to_bits(Hc)
    ref_bits = canon_conv_f32(wl.H, wl.offsets, workloads.bf16_to_f32(w), workloads.bf16_to_f32(b), True)
    assert np.array_equal(hc, ref_bits)
    ref = dR_rank1(workloads.bf16_to_f32(ref_bits), wl.offsets, wl.eps2)
    got = dR.cpu().numpy()
    K = int(wl.K[0])
    for r in range(wl.rows):
        a, e = wl.offsets[r], wl.offsets[r + 1]
        check_dR(got[a:e], ref[a:e], "bf16", f"canon/row{r}")
        sel = topk_select(got[a:e].astype(np.float64), K)
        check_boundaries(sel, ref[a:e], K, f"canon/row{r}")


def test_canon_rejects_bad_arguments():
    import ctypes
    import torch
    import dynamic_byte_chunking_b200 as dbc
    L = dbc.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.canon_conv1d(None, None, 1, 4, 4, 12, None, None, 0, None, None, s) == 2      # d % 8
    assert L.canon_conv1d(None, None, 2, 4, 7, 64, None, None, 0, None, None, s) == 1      # N != rows * T
    assert L.canon_conv1d(None, None, 1, 4, 4, 64, None, None, 0, None, None, s) == 1      # NULL buffers
