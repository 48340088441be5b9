"""Canary padding around every output buffer: the hot-path calls write exactly
their outputs and nothing before or after them.

Each output is carved from the middle of a larger buffer whose head and tail
hold a canary bit pattern; after the calls the canaries must be unchanged.
Small ragged batches (ragged tails, short and empty rows) through the whole
path: coding rate, Top-K, gather, upsample, Canon convolution.
"""
import numpy as np
import pytest

import workloads

pytestmark = pytest.mark.gpu

PAD_BYTES = 4096
CANARY = 0x5A


def _padded(n_bytes, device):
    import torch
    buf = torch.full((PAD_BYTES + n_bytes + PAD_BYTES,), CANARY, dtype=torch.uint8, device=device)
    return buf, buf[PAD_BYTES:PAD_BYTES + n_bytes]


def _intact(buf):
    b = buf.cpu().numpy()
    return bool(np.all(b[:PAD_BYTES] == CANARY) and np.all(b[-PAD_BYTES:] == CANARY))


@pytest.mark.parametrize("d", [256, 128])
def test_outputs_leave_their_neighbours_untouched(d):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    dev = torch.device("cuda")
    rng = np.random.default_rng(d)
    lens = [300, 1, 0, 77, 1029, 64, 5]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N, rows, T = int(offs[-1]), len(lens), max(lens)
    H = workloads.bf16_bits((rng.standard_normal((N, d)) / np.sqrt(d)).astype(np.float32))
    Hd = torch.from_numpy(H.view(np.int16)).view(torch.bfloat16).to(dev)
    od = torch.from_numpy(offs).to(dev)
    Kv = np.maximum(1, np.array(lens) // 4)
    Kt = torch.from_numpy(Kv.astype(np.int64)).to(dev)
    total = int(np.minimum(Kv, lens).sum())
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    b_dR, dR = _padded(N * 4, dev)
    dR = dR.view(torch.float32)
    dbc.chunk_coding_rate(Hd, 0.5, offsets=od, T=T, dR=dR, dev_status=st)
    b_idx, idx = _padded(total * 8, dev)
    idx = idx.view(torch.int64)
    b_io, io = _padded((rows + 1) * 8, dev)
    io = io.view(torch.int64)
    dbc.chunk_topk_select(dR, Kt, rows=rows, T=T, offsets=od, idx=idx, idx_offsets=io, total=total, dev_status=st)
    b_Z, Z = _padded(total * d * 2, dev)
    Z = Z.view(torch.bfloat16).view(total, d)
    dbc.chunk_gather(Hd, idx, io, rows=rows, T=T, offsets=od, total=total, Z=Z, dev_status=st)
    W = workloads.bf16_bits((rng.standard_normal((16, d, d)) / np.sqrt(d)).astype(np.float32))
    Wd = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).to(dev)
    b_S, S = _padded(N * d * 4, dev)
    S = S.view(torch.float32).view(N, d)
    dbc.chunk_upsample(Z, Hd, idx, io, Wd, rows=rows, T=T, offsets=od, S=S, dev_status=st)
    wc = workloads.bf16_bits((rng.standard_normal((d, 4)) * 0.5).astype(np.float32))
    wcd = torch.from_numpy(wc.view(np.int16)).view(torch.bfloat16).to(dev)
    b_C, C = _padded(N * d * 2, dev)
    C = C.view(torch.bfloat16).view(N, d)
    dbc.canon_conv1d(Hd, wcd, offsets=od, T=T, residual=True, out=C, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, hex(st.item())
    for name, b in [("dR", b_dR), ("idx", b_idx), ("idx_offsets", b_io), ("Z", b_Z), ("S", b_S), ("canon", b_C)]:
        assert _intact(b), f"{name}: canary overwritten"
    # the outputs themselves were written (no canary left inside them)
    assert not np.any(dR.cpu().view(torch.int32).numpy() == 0x5A5A5A5A)
    assert int(io[-1].item()) == total
