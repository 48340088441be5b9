"""The allocation-free upsample entry point matches the workspace one.

chunk_upsample_noalloc serves callers that cannot give the library device
scratch (a server whose device memory is all owned by its own pool, a plugin
that receives only its inputs and outputs).  Its scratch is a static device
array inside libdbc.so.  These checks call it several times in a row with
different inputs, the sizes going large, small, large (the array keeps the
previous call's contents), through the C ABI and once through the Python
binding, and compare with chunk_upsample at the upsampling tolerance of the
parity tests.
This file is collected last on purpose; it passes alone or after the others.
"""
import ctypes

import numpy as np
import pytest

import workloads
from parity_util import check_close_rows

pytestmark = pytest.mark.gpu


def _dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _case(seed, lens, d_g=256, d_l=256, nbins=16):
    rng = np.random.default_rng(seed)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N = int(offs[-1])
    idx, io = [], [0]
    for n in lens:
        k = max(1, n // 4)
        sel = np.concatenate([[0], np.sort(rng.choice(np.arange(1, n), size=k - 1, replace=False))])
        idx.append(sel)
        io.append(io[-1] + len(sel))
    idx = np.concatenate(idx).astype(np.int64)
    io = np.array(io, dtype=np.int64)
    H = workloads.bf16_bits((rng.standard_normal((N, d_l)) / 16).astype(np.float32))
    G = workloads.bf16_bits(rng.standard_normal((len(idx), d_g)).astype(np.float32))
    W = workloads.bf16_bits((rng.standard_normal((nbins, d_g, d_l)) / 16).astype(np.float32))
    return offs, idx, io, H, G, W


def _call_noalloc(L, G, H, offs_d, T, N, d_g, d_l, idx, io, rows, W, nbins, mode, S, st):
    import torch
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.chunk_upsample_noalloc(G.data_ptr(), d_g, H.data_ptr(), 1, offs_d.data_ptr(), T, N, d_l,
                                    idx.data_ptr(), io.data_ptr(), rows, W.data_ptr(), nbins, mode,
                                    S.data_ptr(), st.data_ptr(), s)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_noalloc_matches_workspace_entry_point_twice(mode):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    L = dbc.lib()
    # large, small, large: the small call runs over scratch that a larger call left behind, and the last
    # call over what the small one left; the middle call goes through the Python binding
    cases = [_case(2, [4096, 5, 900]), _case(1, [1, 700, 64, 33]), _case(3, [2000, 3000, 17, 1200])]
    for i, (offs, idx, io, H, G, W) in enumerate(cases):
        rows, N, T = len(offs) - 1, int(offs[-1]), int(np.diff(offs).max())
        nbins, d_g, d_l = W.shape
        Hd, Gd, Wd = _dev_bf16(H), _dev_bf16(G), _dev_bf16(W)
        od, idd, iod = (torch.from_numpy(x).cuda() for x in (offs, idx, io))
        ref = dbc.chunk_upsample(Gd, Hd, idd, iod, Wd, rows=rows, T=T, offsets=od, mode=mode)
        S = torch.full((N, d_l), float("nan"), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        if i == 1:
            dbc.chunk_upsample_noalloc(Gd, Hd, idd, iod, Wd, rows=rows, T=T, offsets=od, mode=mode, S=S,
                                       dev_status=st)
        else:
            rc = _call_noalloc(L, Gd, Hd, od, T, N, d_g, d_l, idd, iod, rows, Wd, nbins, mode, S, st)
            assert rc == 0, dbc.status_string(rc)
        torch.cuda.synchronize()
        assert st.item() == 0
        check_close_rows(S.cpu().numpy(), ref.cpu().numpy(), f"noalloc-m{mode}-{i}")


def test_noalloc_rejects_sizes_above_its_scratch():
    import torch
    import dynamic_byte_chunking_b200 as dbc
    L = dbc.lib()
    N = (1 << 20) + 1
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.chunk_upsample_noalloc(None, 256, None, 1, None, N, N, 256, None, None, 1, None, 16, 0,
                                  None, None, s)
    assert rc == 7   # DBC_ERR_WORKSPACE, returned before any launch
