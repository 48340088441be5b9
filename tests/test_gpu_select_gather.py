"""chunk_topk_select_gather: the boundary selection and the chunk-vector gather in one launch.

The fused call must give exactly the separate calls' results (indices, offsets and a bit-exact
copy of the boundary rows) and the oracle's: ragged rows with per-row K (heavy ties, empty rows,
K = 1, K >= T), dense rows with one K (the kernel writes the offsets itself), fp32 and bf16 H,
rows long enough for the two-call fallback, and the byteflow batch.
"""
import numpy as np
import pytest

import workloads
from oracle.chunking import gather as oracle_gather
from oracle.chunking import topk_select

pytestmark = pytest.mark.gpu


def _np(x):
    import torch
    return x.view(torch.int16).cpu().numpy().view(np.uint16) if x.dtype == torch.bfloat16 else x.cpu().numpy()


def _check(dR_np, H_np, offs, Ks, fused, separate):
    idx_f, io_f, Z_f = (_np(x) for x in fused)
    idx_s, io_s, Z_s = (_np(x) for x in separate)
    assert np.array_equal(io_f, io_s)
    assert np.array_equal(idx_f, idx_s)
    assert np.array_equal(Z_f.view(np.uint8), Z_s.view(np.uint8))
    for r in range(len(offs) - 1):
        a, b = offs[r], offs[r + 1]
        want = topk_select(dR_np[a:b].astype(np.float64), Ks[r]) if b > a else np.zeros(0, np.int64)
        assert np.array_equal(idx_f[io_f[r]:io_f[r + 1]], want), r
    ref = oracle_gather(H_np, offs, idx_f, io_f)
    assert np.array_equal(Z_f.reshape(len(idx_f), -1).view(np.uint8), ref.reshape(len(idx_f), -1).view(np.uint8))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ragged_per_row_K(dtype):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    rng = np.random.default_rng(21)
    lens = [1, 2, 5, 300, 4096, 0, 9000, 777]
    Ks = [1, 5, 1, 300, 1024, 3, 8999, 200]
    d = 128 if dtype == "bf16" else 64
    N = sum(lens)
    vals = rng.random(N).astype(np.float32)
    vals[rng.random(N) < 0.3] = 0.25
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    Hf = (rng.standard_normal((N, d)) / np.sqrt(d)).astype(np.float32)
    if dtype == "bf16":
        Hb = workloads.bf16_bits(Hf)
        Hd = torch.from_numpy(Hb.view(np.int16)).view(torch.bfloat16).cuda()
        H_np = Hb
    else:
        Hd = torch.from_numpy(Hf).cuda()
        H_np = Hf
    dd = torch.from_numpy(vals).cuda()
    o = torch.from_numpy(offs).cuda()
    Kt = torch.tensor(Ks, dtype=torch.int64, device="cuda")
    total = int(np.minimum(Ks, lens).sum())
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fused = dbc.chunk_topk_select_gather(dd, Kt, Hd, rows=len(lens), T=max(lens), offsets=o, total=total,
                                         dev_status=st)
    idx, io = dbc.chunk_topk_select(dd, Kt, rows=len(lens), T=max(lens), offsets=o, total=total)
    Z = dbc.chunk_gather(Hd, idx, io, rows=len(lens), T=max(lens), offsets=o, total=total)
    torch.cuda.synchronize()
    assert st.item() == 0
    _check(vals, H_np, offs, Ks, fused, (idx, io, Z))


@pytest.mark.parametrize("T,K", [(1000, 250), (8192, 2048), (70000, 9000)])
def test_dense_one_K(T, K):
    """Dense rows with one K (offsets written by the kernel); T = 70000 takes the two-call path."""
    import torch
    import dynamic_byte_chunking_b200 as dbc
    rng = np.random.default_rng(T)
    rows, d = 3, 256
    vals = rng.random(rows * T).astype(np.float32)
    vals[::5] = 0.5
    Hb = workloads.bf16_bits((rng.standard_normal((rows * T, d)) / 16).astype(np.float32))
    Hd = torch.from_numpy(Hb.view(np.int16)).view(torch.bfloat16).cuda()
    dd = torch.from_numpy(vals).cuda()
    fused = dbc.chunk_topk_select_gather(dd, K, Hd, rows=rows, T=T)
    idx, io = dbc.chunk_topk_select(dd, K, rows=rows, T=T)
    Z = dbc.chunk_gather(Hd, idx, io, rows=rows, T=T)
    offs = np.arange(rows + 1, dtype=np.int64) * T
    _check(vals, Hb, offs, [K] * rows, fused, (idx, io, Z))


def test_byteflow_batch():
    import torch
    import dynamic_byte_chunking_b200 as dbc
    w = workloads.make("byteflow")
    H = torch.from_numpy(w.H_bits.view(np.int16)).view(torch.bfloat16).cuda()
    dR = dbc.chunk_coding_rate(H.view(w.rows, w.T, w.d), w.eps2)
    K = int(w.K[0])
    fused = dbc.chunk_topk_select_gather(dR, K, H, rows=w.rows, T=w.T)
    idx, io = dbc.chunk_topk_select(dR, K, rows=w.rows, T=w.T)
    Z = dbc.chunk_gather(H, idx, io, rows=w.rows, T=w.T)
    _check(dR.cpu().numpy(), w.H_bits, w.offsets, [K] * w.rows, fused, (idx, io, Z))
