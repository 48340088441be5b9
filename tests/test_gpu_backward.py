"""GPU parity of the backward of the upsampling and of the gather.

The oracle is the float64 chain rule (oracle.chunking.upsample_backward*,
gather_backward), pinned on the CPU by exact central differences of the
forward.  Small cases compare every element; the full workloads compare the
oracle on whole rows (byteflow) and, where the oracle cannot cover the batch
(ragged: dW sums over 2.2M positions), the adjoint identities
<dW, W'> = <dS, S(G, W') - H> and <dG, G'> = <dS, S(G', W) - H>, which hold at
any size, with S from the (separately parity-tested) forward call.
"""
import numpy as np
import pytest

import workloads
from oracle.chunking import (BIN_ABSOLUTE, BIN_FRACTION, BIN_OFFSET, gather_backward, upsample_backward,
                             upsample_backward_row)
from parity_util import check_close_rows, record

pytestmark = pytest.mark.gpu


def bf16_dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _random_bounds(rng, lens, K):
    idx, io = [], [0]
    for n, k in zip(lens, K):
        k = min(k, n)
        sel = np.concatenate([[0], np.sort(rng.choice(np.arange(1, n), size=k - 1, replace=False))]) if n else []
        idx.append(np.asarray(sel, dtype=np.int64))
        io.append(io[-1] + len(sel))
    return np.concatenate(idx).astype(np.int64), np.array(io, dtype=np.int64)


@pytest.mark.parametrize("mode", [BIN_OFFSET, BIN_FRACTION, BIN_ABSOLUTE])
def test_upsample_backward_small_ragged_all_modes(mode):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    rng = np.random.default_rng(20 + mode)
    lens = [1, 40, 0, 333, 130, 700]
    K = [1, 3, 1, 20, 130, 30]              # a chunk longer than 16, an empty row, all-singleton rows
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N, d_g, d_l, B = int(offs[-1]), 128, 192, 16
    idx, io = _random_bounds(rng, lens, K)
    Gb = workloads.bf16_bits(rng.standard_normal((len(idx), d_g)).astype(np.float32))
    Wb = workloads.bf16_bits((rng.standard_normal((B, d_g, d_l)) / np.sqrt(d_g)).astype(np.float32))
    dS = rng.standard_normal((N, d_l)).astype(np.float32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dG, dW, dH = dbc.chunk_upsample_backward(torch.from_numpy(dS).cuda(), bf16_dev(Gb), torch.from_numpy(idx).cuda(),
                                             torch.from_numpy(io).cuda(), bf16_dev(Wb), rows=len(lens), T=max(lens),
                                             offsets=torch.from_numpy(offs).cuda(), mode=mode, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    G, W = workloads.bf16_to_f32(Gb), workloads.bf16_to_f32(Wb)
    rG, rW, rH = upsample_backward(G, offs, idx, io, W, dS, mode)
    check_close_rows(dG.cpu().numpy(), rG, f"upsample-bwd-small-m{mode}:dG")
    check_close_rows(dW.cpu().numpy().reshape(B * d_g, d_l), rW.reshape(B * d_g, d_l), f"upsample-bwd-small-m{mode}:dW")
    assert np.array_equal(dH.cpu().numpy(), dS)          # the residual path is a copy


def test_gather_backward_small_exact():
    import torch
    import dynamic_byte_chunking_b200 as dbc
    rng = np.random.default_rng(30)
    lens = [5, 0, 64, 300]
    K = [2, 1, 64, 17]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N, d = int(offs[-1]), 256
    idx, io = _random_bounds(rng, lens, K)
    dZ = rng.standard_normal((len(idx), d)).astype(np.float32)
    base = rng.standard_normal((N, d)).astype(np.float32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dH = torch.from_numpy(base).cuda()
    dbc.chunk_gather_backward(torch.from_numpy(dZ).cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(io).cuda(),
                              rows=len(lens), T=max(lens), dH=dH, offsets=torch.from_numpy(offs).cuda(),
                              accumulate=True, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    # an fp32 add of two fp32 values is their exact float64 sum rounded once
    want = (base.astype(np.float64) + gather_backward(dZ, offs, idx, io, N)).astype(np.float32)
    assert np.array_equal(dH.cpu().numpy(), want)
    # overwrite mode: boundary rows become dZ, the others keep their values
    dH2 = torch.from_numpy(base).cuda()
    dbc.chunk_gather_backward(torch.from_numpy(dZ).cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(io).cuda(),
                              rows=len(lens), T=max(lens), dH=dH2, offsets=torch.from_numpy(offs).cuda(),
                              accumulate=False, dev_status=st)
    got = dH2.cpu().numpy()
    mask = np.zeros(N, dtype=bool)
    for r in range(len(lens)):
        mask[offs[r] + idx[io[r]:io[r + 1]]] = True
    assert np.array_equal(got[~mask], base[~mask])
    assert np.array_equal(got[mask], gather_backward(dZ, offs, idx, io, N)[mask].astype(np.float32))


def _pipeline(w):
    """Forward chunking on the GPU; returns device tensors (H, idx, io, G, offsets or None)."""
    import torch
    import dynamic_byte_chunking_b200 as dbc
    H = bf16_dev(w.H_bits)
    o = torch.from_numpy(w.offsets).cuda()
    oo = None if w.dense else o
    dR = dbc.chunk_coding_rate(H.view(w.rows, w.T, w.d) if w.dense else H, w.eps2, offsets=oo, T=w.T)
    total = int(np.minimum(w.K, w.lengths).sum())
    idx, io = dbc.chunk_topk_select(dR, torch.from_numpy(w.K).cuda(), rows=w.rows, T=w.T, offsets=oo, total=total)
    G = dbc.chunk_gather(H, idx, io, rows=w.rows, T=w.T, offsets=oo, total=total)
    return H, idx, io, G, oo


def test_upsample_backward_full_byteflow():
    import torch
    import dynamic_byte_chunking_b200 as dbc
    w = workloads.make("byteflow")
    H, idx, io, G, oo = _pipeline(w)
    rng = np.random.default_rng(40)
    dS = (rng.standard_normal((w.N, w.d)) / 16).astype(np.float32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dG, dW, dH = dbc.chunk_upsample_backward(torch.from_numpy(dS).cuda(), G, idx, io, bf16_dev(w.W_bin),
                                             rows=w.rows, T=w.T, offsets=oo, dev_status=st)
    # the full chain to H: residual plus the gather's adjoint
    dbc.chunk_gather_backward(dG, idx, io, rows=w.rows, T=w.T, dH=dH, offsets=oo, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    idx_n, io_n = idx.cpu().numpy(), io.cpu().numpy()
    Gn = workloads.bf16_to_f32(G.cpu().view(torch.int16).numpy().view(np.uint16))
    W = w.f32("W_bin")
    rG, rW, _ = upsample_backward(Gn, w.offsets, idx_n, io_n, W, dS, BIN_OFFSET)
    dGn = dG.cpu().numpy()
    check_close_rows(dGn, rG, "full-byteflow-bwd:dG")
    check_close_rows(dW.cpu().numpy().reshape(-1, w.d), rW.reshape(-1, w.d), "full-byteflow-bwd:dW")
    want_H = dS.astype(np.float64) + gather_backward(dGn, w.offsets, idx_n, io_n, w.N)
    assert np.array_equal(dH.cpu().numpy(), want_H.astype(np.float32))


def test_upsample_backward_full_ragged_adjoint():
    import torch
    import dynamic_byte_chunking_b200 as dbc
    w = workloads.make("ragged")
    H, idx, io, G, oo = _pipeline(w)
    rng = np.random.default_rng(41)
    dS = torch.from_numpy((rng.standard_normal((w.N, w.d)) / 16).astype(np.float32)).cuda()
    Wb = bf16_dev(w.W_bin)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dG, dW, _ = dbc.chunk_upsample_backward(dS, G, idx, io, Wb, rows=w.rows, T=w.T, offsets=oo, residual=False,
                                            dev_status=st)
    Z0 = torch.zeros_like(H)
    # <dW, W'> = <dS, S(G, W') - H> for a random W' (bf16)
    Wp = bf16_dev(workloads.bf16_bits((rng.standard_normal(w.W_bin.shape) / 16).astype(np.float32)))
    S1 = dbc.chunk_upsample(G, Z0, idx, io, Wp, rows=w.rows, T=w.T, offsets=oo)
    # <dG, G'> = <dS, S(G', W) - H> for a random G' (bf16)
    Gp = bf16_dev(workloads.bf16_bits((rng.standard_normal(tuple(G.shape)) / 16).astype(np.float32)))
    S2 = dbc.chunk_upsample(Gp, Z0, idx, io, Wb, rows=w.rows, T=w.T, offsets=oo)
    torch.cuda.synchronize()
    assert st.item() == 0
    lhs_w = float(torch.sum(dW.double() * Wp.double()))
    rhs_w = float(torch.sum(dS.double() * S1.double()))
    lhs_g = float(torch.sum(dG.double() * Gp.double()))
    rhs_g = float(torch.sum(dS.double() * S2.double()))
    # scale of the sums: sqrt(#terms) * typical term; relative to the sum of |terms|
    abs_w = float(torch.sum(torch.abs(dS.double() * S1.double())))
    abs_g = float(torch.sum(torch.abs(dS.double() * S2.double())))
    ew, eg = abs(lhs_w - rhs_w) / abs_w, abs(lhs_g - rhs_g) / abs_g
    record("full-ragged-bwd:adjoint", dW_rel=ew, dG_rel=eg)
    assert ew <= 1e-4 and eg <= 1e-4, (ew, eg)
    # whole rows of dG against the oracle (a row's chunk gradients only see that row)
    idx_n, io_n = idx.cpu().numpy(), io.cpu().numpy()
    Gn = workloads.bf16_to_f32(G.cpu().view(torch.int16).numpy().view(np.uint16))
    W = w.f32("W_bin")
    dSn = dS.cpu().numpy()
    dGn = dG.cpu().numpy()
    for r in [0, int(np.argmax(w.lengths))]:
        a, b = w.offsets[r], w.offsets[r + 1]
        ia, ib = io_n[r], io_n[r + 1]
        rg, _, _ = upsample_backward_row(Gn[ia:ib], idx_n[ia:ib], W, dSn[a:b], BIN_OFFSET)
        check_close_rows(dGn[ia:ib], rg, f"full-ragged-bwd:dG-row{r}")
