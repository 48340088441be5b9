"""GPU parity of the upsampler, the chunk projection, the router and the EMA.

Downstream stages are compared with the oracle run on the GPU's own boundary
indices (positions inside the Top-K tie band may legitimately differ).
"""
import numpy as np
import pytest

import workloads
from oracle.chunking import BIN_ABSOLUTE, BIN_FRACTION, BIN_OFFSET, upsample_row
from oracle.router import ema, route_row
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
def test_upsample_small_ragged_all_modes(mode):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    rng = np.random.default_rng(10 + mode)
    lens = [1, 40, 0, 333, 130, 700]
    K = [1, 3, 1, 20, 130, 30]              # includes a chunk longer than 16 and all-singleton rows
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N, d_g, d_l, B = offs[-1], 128, 192, 16
    Hb = workloads.bf16_bits(rng.standard_normal((N, d_l)).astype(np.float32))
    idx, io = _random_bounds(rng, lens, K)
    Gb = workloads.bf16_bits(rng.standard_normal((len(idx), d_g)).astype(np.float32))
    Wb = workloads.bf16_bits((rng.standard_normal((B, d_g, d_l)) / np.sqrt(d_g)).astype(np.float32))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    S = dbc.chunk_upsample(bf16_dev(Gb), bf16_dev(Hb), torch.from_numpy(idx).cuda(),
                           torch.from_numpy(io).cuda(), bf16_dev(Wb), rows=len(lens), T=max(lens),
                           offsets=torch.from_numpy(offs).cuda(), mode=mode, dev_status=st)
    S = S.cpu().numpy()
    assert st.item() == 0
    H, G, W = (workloads.bf16_to_f32(x) for x in (Hb, Gb, Wb))
    for r in range(len(lens)):
        if lens[r] == 0:
            continue
        ref = upsample_row(G[io[r]:io[r + 1]], H[offs[r]:offs[r + 1]], idx[io[r]:io[r + 1]], W, mode)
        check_close_rows(S[offs[r]:offs[r + 1]], ref, f"upsample-small-m{mode}-r{r}")


def _chunk_and_upsample(w, rows_checked, name, project=False):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    H = bf16_dev(w.H_bits)
    o = torch.from_numpy(w.offsets).cuda()
    ragged = not w.dense
    oo = o if ragged else None
    dR = dbc.chunk_coding_rate(H, w.eps2, offsets=oo, T=w.T) if ragged else \
        dbc.chunk_coding_rate(H.view(w.rows, w.T, w.d), w.eps2)
    total = int(np.minimum(w.K, w.lengths).sum())
    idx, io = dbc.chunk_topk_select(dR, torch.from_numpy(w.K).cuda(), rows=w.rows, T=w.T, offsets=oo,
                                    total=total)
    if project:
        Z, Zf, Zb = dbc.chunk_gather(H, idx, io, rows=w.rows, T=w.T, offsets=oo, total=total,
                                     W_proj=bf16_dev(w.W_proj))
        G = Zb
    else:
        G = dbc.chunk_gather(H, idx, io, rows=w.rows, T=w.T, offsets=oo, total=total)
    S = dbc.chunk_upsample(G, H, idx, io, bf16_dev(w.W_bin), rows=w.rows, T=w.T, offsets=oo)
    torch.cuda.synchronize()
    idx_n, io_n = idx.cpu().numpy(), io.cpu().numpy()
    Sn = S.cpu().numpy()
    Gn = workloads.bf16_to_f32(G.cpu().view(torch.int16).numpy().view(np.uint16))
    W = w.f32("W_bin")
    if project:
        Zn = workloads.bf16_to_f32(Z.cpu().view(torch.int16).numpy().view(np.uint16))
        ref = Zn.astype(np.float64) @ w.f32("W_proj").astype(np.float64)
        check_close_rows(Zf.cpu().numpy(), ref, name + ":proj")
        # bf16 output is the RNE of the fp32 output
        assert np.array_equal(workloads.bf16_bits(Zf.cpu().numpy()), G.cpu().view(torch.int16).numpy().view(np.uint16))
    for r in rows_checked:
        a, b = w.offsets[r], w.offsets[r + 1]
        ref = upsample_row(Gn[io_n[r]:io_n[r + 1]], w.H[a:b], idx_n[io_n[r]:io_n[r + 1]], W, BIN_OFFSET)
        check_close_rows(Sn[a:b], ref, f"{name}/row{r}")


def test_upsample_full_byteflow():
    w = workloads.make("byteflow")
    _chunk_and_upsample(w, [0, 5], "full-byteflow-upsample")


def test_projection_and_upsample_full_wide():
    w = workloads.make("wide")
    _chunk_and_upsample(w, [7], "full-wide-upsample", project=True)


def test_upsample_full_ragged():
    w = workloads.make("ragged")
    _chunk_and_upsample(w, [0, int(np.argmax(w.lengths))], "full-ragged-upsample")


# ---------------------------------------------------------------- router
def _route_check(w, rows_checked, name):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    H = bf16_dev(w.H_bits)
    o = torch.from_numpy(w.offsets).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    p, b, ci, co, z = dbc.hnet_route(H, bf16_dev(w.Wq), bf16_dev(w.Wk), offsets=o, T=w.T, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    p, b, ci, co, z = p.cpu().numpy(), b.cpu().numpy(), ci.cpu().numpy(), co.cpu().numpy(), z.cpu().numpy()
    Wq, Wk = w.f32("Wq"), w.f32("Wk")
    worst = 0.0
    for r in rows_checked:
        a, e = w.offsets[r], w.offsets[r + 1]
        pr, br, _ = route_row(w.H[a:e], Wq, Wk)
        dp = np.abs(p[a:e] - pr)
        worst = max(worst, dp.max())
        assert dp.max() <= 1e-3, f"{name}/row{r}: |dp| {dp.max():.2e}"
        clear = np.abs(pr - 0.5) > 1e-3
        assert np.array_equal(b[a:e][clear].astype(bool), br[clear])
        # chunk list = the GPU's own boundaries, in order
        mine = ci[co[r]:co[r + 1]]
        assert np.array_equal(mine, np.nonzero(b[a:e])[0])
        zr = ema(w.H[a:e][mine].astype(np.float64), p[a:e][mine].astype(np.float64))
        check_close_rows(z[co[r]:co[r + 1]], zr, f"{name}/ema-row{r}")
    record(name + ":router", max_abs_dp=worst)


def test_router_full_bytegen():
    w = workloads.make("bytegen")
    _route_check(w, range(0, 64, 8), "full-bytegen")


def test_router_small_ragged_with_empty_rows():
    rng = np.random.default_rng(2)
    lens = [1, 0, 70, 2, 513]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    d = 256
    Hb = workloads.bf16_bits((rng.standard_normal((offs[-1], d)) / 16).astype(np.float32))
    w = workloads.Workload("r", "bf16", d, 0.5, offs, workloads.bf16_to_f32(Hb), Hb, np.ones(5, np.int64))
    w.Wq = workloads.bf16_bits((rng.standard_normal((d, d)) / 16).astype(np.float32))
    w.Wk = workloads.bf16_bits((rng.standard_normal((d, d)) / 16).astype(np.float32))
    _route_check(w, [0, 2, 3, 4], "router-small")
