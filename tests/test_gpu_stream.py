"""GPU parity of the streaming continuation of the coding rate.

Streams are fed in blocks of uneven sizes (crossing the 64 / 128 / 256 segment
boundaries and starting mid-segment); the concatenated dR must equal the
whole-sequence oracle (the rank-1 recursion, float64) within the dR tolerance,
the carried Gram sum must equal the float64 H^T H of everything fed, and the
windowed selection on the streamed values must equal the oracle's selection on
the same values.
"""
import numpy as np
import pytest

import workloads
from oracle.chunking import topk_select_rows
from oracle.rank1 import dR_rank1
from parity_util import check_dR, record

pytestmark = pytest.mark.gpu


def bf16_dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("blocks", [[1, 63, 64, 200, 256, 700, 764], [2048], [300, 1748]])
def test_stream_blocks_equal_whole_sequence(blocks):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    S, T = 4, sum(blocks)
    w = workloads.make("byteflow", rows=S, T=T, weights=False)
    H = bf16_dev(w.H_bits).view(S, T, w.d)
    state = torch.zeros(S, w.d, w.d, dtype=torch.float64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs, t0 = [], 0
    for n in blocks:
        blk = H[:, t0:t0 + n, :].contiguous()
        outs.append(dbc.chunk_coding_rate_stream(blk, w.eps2, state, t0, dev_status=st).view(S, n))
        t0 += n
    torch.cuda.synchronize()
    assert st.item() == 0
    dR = torch.cat(outs, dim=1).cpu().numpy()
    ref = dR_rank1(w.H, w.offsets, w.eps2).reshape(S, T)
    for r in range(S):
        check_dR(dR[r], ref[r], "bf16", f"stream-{len(blocks)}blocks/row{r}")
    X = np.asarray(w.H, dtype=np.float64).reshape(S, T, w.d)
    want = np.einsum("stk,stl->skl", X, X)
    got = state.cpu().numpy()
    rel = np.abs(got - want).max() / np.abs(want).max()
    record(f"stream-{len(blocks)}blocks:state", max_rel=rel)
    assert rel <= 1e-6


def test_stream_windowed_selection():
    """Causal boundaries: Top-K inside fixed windows of the streamed values."""
    import torch
    import dynamic_byte_chunking_b200 as dbc
    S, T, W, k = 2, 2048, 512, 128
    w = workloads.make("byteflow", rows=S, T=T, weights=False)
    H = bf16_dev(w.H_bits).view(S, T, w.d)
    state = torch.zeros(S, w.d, w.d, dtype=torch.float64, device="cuda")
    outs = []
    for t0 in range(0, T, 256):
        outs.append(dbc.chunk_coding_rate_stream(H[:, t0:t0 + 256, :].contiguous(), w.eps2, state, t0).view(S, 256))
    dR = torch.cat(outs, dim=1).contiguous().view(-1)
    nwin = S * T // W
    idx, io = dbc.chunk_topk_select(dR, k, rows=nwin, T=W)
    torch.cuda.synchronize()
    dRn = dR.cpu().numpy()
    ridx, rio = topk_select_rows(dRn, np.arange(nwin + 1, dtype=np.int64) * W, k)
    assert np.array_equal(io.cpu().numpy(), rio)
    assert np.array_equal(idx.cpu().numpy(), ridx)


# ---------------------------------------------------------------- per-position recursion
@pytest.mark.parametrize("fam,S,blocks", [
    ("byteflow", 3, [1, 1, 3, 64, 250, 381]),       # d = 256, bf16, one-position calls first
    ("byteflow", 2, [256] * 16),                     # 4096 rank-one updates of the carried factor
    ("bytegen", 2, [1, 511, 608]),                   # structured rows (whole 32-byte market events)
    ("tiny", 2, [1, 7, 300]),                        # d = 64, fp32
])
def test_step_equals_whole_sequence(fam, S, blocks):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    T = sum(blocks)
    w = workloads.make(fam, rows=S, T=T, weights=False)
    if w.dtype == "bf16":
        H = bf16_dev(w.H_bits).view(S, T, w.d)
    else:
        H = torch.from_numpy(np.ascontiguousarray(w.H_bits)).cuda().view(S, T, w.d)
    B = dbc.step_state(S, w.d)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs, t0 = [], 0
    for n in blocks:
        outs.append(dbc.chunk_coding_rate_step(H[:, t0:t0 + n, :], w.eps2, B, dev_status=st).view(S, n))
        t0 += n
    torch.cuda.synchronize()
    assert st.item() == 0
    dR = torch.cat(outs, dim=1).cpu().numpy()
    ref = dR_rank1(w.H, w.offsets, w.eps2).reshape(S, T)
    for r in range(S):
        check_dR(dR[r], ref[r], w.dtype, f"step-{fam}-{len(blocks)}calls/row{r}")
    # the carried factor: B^T M B = I for the M of everything fed (M = I + c X^T X)
    X = np.asarray(w.H, dtype=np.float64).reshape(S, T, w.d)
    c = w.d / w.eps2
    Bh = np.triu(B.cpu().numpy().astype(np.float64))
    for r in range(S):
        M = np.eye(w.d) + c * X[r].T @ X[r]
        E = Bh[r].T @ M @ Bh[r] - np.eye(w.d)
        rel = np.abs(E).max()
        record(f"step-{fam}-{len(blocks)}calls/row{r}:BtMB", max_abs=rel)
        assert rel <= 1e-2


def test_step_leaves_lower_triangle_alone():
    import torch
    import dynamic_byte_chunking_b200 as dbc
    w = workloads.make("tiny", rows=1, T=40, weights=False)
    H = torch.from_numpy(np.ascontiguousarray(w.H_bits)).cuda().view(1, 40, w.d)
    B = dbc.step_state(1, w.d)
    low = torch.tril(torch.full((w.d, w.d), 7.0, device="cuda"), diagonal=-1)
    B += low
    dbc.chunk_coding_rate_step(H, w.eps2, B)
    torch.cuda.synchronize()
    assert torch.equal(torch.tril(B[0], diagonal=-1), low)
