"""B200 dynamic byte chunking: Python binding of ``libdbc.so``.

Every function here marshals torch tensors into the C ABI declared in
``include/dbc.h`` and calls it on the current CUDA stream; all arithmetic runs
in the library's CUDA kernels.  There is no CPU fallback: importing works
anywhere, but the first call raises if the library is missing or no CUDA
device is present.

The hot path (ByteFlow, arXiv 2603.03583; H-Net router from the ByteGen
report):

* :func:`chunk_coding_rate`  dR_t = R(h_0..t) - R(h_0..t-1) per row;
* :func:`chunk_topk_select`  BOS + the K-1 largest dR (t >= 1), in time order;
* :func:`chunk_gather`       z_k = h_{s_k} (optionally times W_proj);
* :func:`chunk_upsample`     S_t = h_t + g_{c(t)} W_{b(t)};
* :func:`hnet_route`         cosine router p_t, boundaries, chunk list, EMA;
* :func:`canon_conv1d`       the encoder's Canon layer (causal depthwise conv, k = 4),
  :func:`chunk_coding_rate_canon` the Canon layer and the coding rate in one call.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "DbcError", "lib", "lib_path", "version", "status_string", "launch_count",
    "chunk_coding_rate", "chunk_coding_rate_workspace", "chunk_coding_rate_stream",
    "chunk_coding_rate_stream_workspace", "chunk_coding_rate_step", "step_state", "chunk_topk_select",
    "chunk_gather", "chunk_upsample", "chunk_upsample_workspace", "chunk_upsample_noalloc",
    "chunk_upsample_backward", "chunk_upsample_backward_workspace", "chunk_gather_backward",
    "hnet_route", "hnet_route_workspace", "chunk", "canon_conv1d", "chunk_coding_rate_canon",
    "DBC_F32", "DBC_BF16", "BIN_OFFSET", "BIN_FRACTION", "BIN_ABSOLUTE",
    "ERR_NONFINITE", "ERR_TIMEOUT", "ERR_BOUNDS",
]

DBC_F32, DBC_BF16 = 0, 1
BIN_OFFSET, BIN_FRACTION, BIN_ABSOLUTE = 0, 1, 2
ERR_NONFINITE, ERR_TIMEOUT, ERR_BOUNDS = 4, 5, 6

_HERE = os.path.dirname(os.path.abspath(__file__))
# DBC_LIBRARY=debug selects the debug build (device-side invariant checks, see build.py)
lib_path = os.path.join(_HERE, "libdbc_debug.so" if os.environ.get("DBC_LIBRARY") == "debug" else "libdbc.so")
_lib = None

_i64, _sz, _vp, _int, _f32 = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int, ctypes.c_float

_SIGS = {
    "dbc_status_string": (ctypes.c_char_p, [_int]),
    "dbc_version": (_int, []),
    "dbc_launch_count": (ctypes.c_uint64, []),
    "chunk_coding_rate_workspace": (_sz, [_i64, _i64, _i64, _i64]),
    "chunk_coding_rate": (_int, [_vp, _int, _vp, _i64, _i64, _i64, _i64, _f32, _vp, _vp, _sz, _vp, _vp]),
    "chunk_coding_rate_stream_workspace": (_sz, [_i64, _i64, _i64, _i64]),
    "chunk_coding_rate_stream": (_int, [_vp, _int, _i64, _i64, _i64, _i64, _f32, _vp, _vp, _vp, _sz, _vp, _vp]),
    "chunk_coding_rate_step": (_int, [_vp, _int, _i64, _i64, _i64, _f32, _vp, _vp, _vp, _vp]),
    "chunk_topk_select_workspace": (_sz, [_i64]),
    "chunk_topk_select": (_int, [_vp, _vp, _i64, _i64, _i64, _vp, _i64, _vp, _vp, _vp, _sz, _vp, _vp]),
    "chunk_gather": (_int, [_vp, _int, _vp, _i64, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp,
                            _vp, _vp]),
    "chunk_upsample_workspace": (_sz, [_i64, _i64, _int]),
    "chunk_upsample": (_int, [_vp, _i64, _vp, _int, _vp, _i64, _i64, _i64, _vp, _vp, _i64, _vp, _int,
                              _int, _vp, _vp, _sz, _vp, _vp]),
    "chunk_upsample_noalloc": (_int, [_vp, _i64, _vp, _int, _vp, _i64, _i64, _i64, _vp, _vp, _i64, _vp,
                                      _int, _int, _vp, _vp, _vp]),
    "chunk_upsample_backward_workspace": (_sz, [_i64, _i64, _int, _i64]),
    "chunk_upsample_backward": (_int, [_vp, _vp, _i64, _vp, _i64, _i64, _i64, _vp, _vp, _i64, _i64, _vp, _int,
                                       _int, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    "chunk_gather_backward": (_int, [_vp, _i64, _vp, _i64, _vp, _vp, _i64, _i64, _vp, _int, _vp, _vp]),
    "hnet_route_workspace": (_sz, [_i64, _i64, _i64]),
    "canon_conv1d": (_int, [_vp, _vp, _i64, _i64, _i64, _i64, _vp, _vp, _int, _vp, _vp, _vp]),
    "chunk_coding_rate_canon": (_int, [_vp, _vp, _i64, _i64, _i64, _i64, _vp, _vp, _int, _vp, _f32, _vp, _vp, _sz,
                                       _vp, _vp]),
    "hnet_route": (_int, [_vp, _vp, _i64, _i64, _i64, _i64, _vp, _vp, _f32, _int, _vp, _vp, _vp, _vp,
                          _vp, _vp, _sz, _vp, _vp]),
}


class DbcError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")
        self.code = code


def lib():
    """Load libdbc.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise RuntimeError(f"{lib_path} is missing: run `python -m dynamic_byte_chunking_b200.build`")
        L = ctypes.CDLL(lib_path)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def version() -> int:
    return lib().dbc_version()


def launch_count() -> int:
    """Kernels launched by libdbc.so in this process so far."""
    return int(lib().dbc_launch_count())


def status_string(code: int) -> str:
    return lib().dbc_status_string(int(code)).decode()


# ---------------------------------------------------------------- helpers
def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, code: int):
    if code != 0:
        raise DbcError(fn, code)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("dbc kernels take CUDA tensors only (no CPU path)")


def _dtype_code(H) -> int:
    torch = _torch()
    if H.dtype == torch.bfloat16:
        return DBC_BF16
    if H.dtype == torch.float32:
        return DBC_F32
    raise TypeError("H must be bfloat16 or float32")


def _layout(H, offsets, T):
    """(rows, T, N, d, H2d) for a dense [rows, T, d] or packed [N, d] batch."""
    if H.dim() == 3:
        if offsets is not None:
            raise ValueError("a 3-D H is dense; pass offsets only with a packed [N, d] H")
        rows, T_, d = H.shape
        return rows, T_, rows * T_, d, H.reshape(rows * T_, d)
    if H.dim() != 2:
        raise ValueError("H must be [rows, T, d] or [N, d]")
    N, d = H.shape
    if offsets is None:
        if T is None or T <= 0 or N % T:
            raise ValueError("packed dense H needs T dividing N")
        return N // T, T, N, d, H
    rows = offsets.numel() - 1
    if T is None:
        T = int((offsets[1:] - offsets[:-1]).max().item()) if rows > 0 else 0
    return rows, T, N, d, H


def _workspace(nbytes: int, device, workspace=None):
    torch = _torch()
    if workspace is not None and workspace.numel() >= nbytes:
        return workspace
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- API
def chunk_coding_rate_workspace(rows: int, T: int, N: int, d: int) -> int:
    return int(lib().chunk_coding_rate_workspace(rows, T, N, d))


def chunk_coding_rate(H, eps2: float, *, offsets=None, T: Optional[int] = None, dR=None,
                      workspace=None, dev_status=None, stream=None):
    """Marginal coding rate dR (fp32 [N]) of a dense [rows, T, d] or packed [N, d] batch."""
    torch = _torch()
    _require_cuda(H, offsets)
    rows, T, N, d, H2 = _layout(H, offsets, T)
    H2 = H2.contiguous()
    if dR is None:
        dR = torch.empty(N, dtype=torch.float32, device=H.device)
    ws = _workspace(chunk_coding_rate_workspace(rows, T, N, d), H.device, workspace)
    rc = lib().chunk_coding_rate(_ptr(H2), _dtype_code(H2), _ptr(offsets), rows, T, N, d, float(eps2),
                                 _ptr(dR), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream))
    _check("chunk_coding_rate", rc)
    return dR


def chunk_coding_rate_stream_workspace(streams: int, n: int, t0: int, d: int) -> int:
    return int(lib().chunk_coding_rate_stream_workspace(streams, n, t0, d))


def chunk_coding_rate_stream(H, eps2: float, state, t0: int, *, dR=None, workspace=None, dev_status=None,
                             stream=None):
    """dR (fp32 [streams * n]) of n new positions per stream ([streams, n, 256] bf16) that continue
    streams which already consumed t0 positions; ``state`` (float64 [streams, 256, 256], the Gram sum
    of everything seen, zero for new streams) is advanced in place."""
    torch = _torch()
    _require_cuda(H, state)
    if H.dim() != 3:
        raise ValueError("H must be [streams, n, d]")
    streams, n, d = H.shape
    if state.dtype != torch.float64 or tuple(state.shape) != (streams, d, d) or not state.is_contiguous():
        raise TypeError("state must be a contiguous float64 [streams, d, d] tensor")
    H2 = H.contiguous()
    if dR is None:
        dR = torch.empty(streams * n, dtype=torch.float32, device=H.device)
    ws = _workspace(chunk_coding_rate_stream_workspace(streams, n, t0, d), H.device, workspace)
    rc = lib().chunk_coding_rate_stream(_ptr(H2), _dtype_code(H2), streams, n, d, int(t0), float(eps2), _ptr(state),
                                        _ptr(dR), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream))
    _check("chunk_coding_rate_stream", rc)
    return dR


def step_state(streams: int, d: int, device="cuda"):
    """Per-byte stream state of new streams: the identity in fp32 [streams, d, d]."""
    torch = _torch()
    return torch.eye(d, dtype=torch.float32, device=device).repeat(streams, 1, 1).contiguous()


def chunk_coding_rate_step(H, eps2: float, B_state, *, dR=None, dev_status=None, stream=None):
    """dR (fp32 [streams * n]) of n new positions per stream ([streams, n, d], fp32 or bf16, d <= 256),
    one position at a time from the carried factor ``B_state`` (fp32 [streams, d, d], the identity for
    new streams, see ``step_state``), which is advanced in place."""
    torch = _torch()
    _require_cuda(H, B_state)
    if H.dim() != 3:
        raise ValueError("H must be [streams, n, d]")
    streams, n, d = H.shape
    if B_state.dtype != torch.float32 or tuple(B_state.shape) != (streams, d, d) or not B_state.is_contiguous():
        raise TypeError("B_state must be a contiguous float32 [streams, d, d] tensor")
    H2 = H.contiguous()
    if dR is None:
        dR = torch.empty(streams * n, dtype=torch.float32, device=H.device)
    rc = lib().chunk_coding_rate_step(_ptr(H2), _dtype_code(H2), streams, n, d, float(eps2), _ptr(B_state),
                                      _ptr(dR), _ptr(dev_status), _stream(stream))
    _check("chunk_coding_rate_step", rc)
    return dR


def chunk_topk_select(dR, K, *, rows: int, T: int, offsets=None, total: Optional[int] = None,
                      idx=None, idx_offsets=None, dev_status=None, stream=None):
    """(idx int64 [total], idx_offsets int64 [rows+1]): BOS + K-1 largest dR per row, in time order.

    ``K`` is an int or a CUDA int64 tensor [rows]; ``total`` (sum of min(K_r, T_r))
    sizes ``idx`` and is required with per-row K unless ``idx`` is given.
    """
    torch = _torch()
    _require_cuda(dR, offsets)
    N = dR.numel()
    Kp, Ks = (K, 0) if torch.is_tensor(K) else (None, int(K))
    if Kp is not None:
        _require_cuda(Kp)
    if idx is None:
        if total is None:
            if Kp is not None or offsets is not None:
                raise ValueError("pass `total` (or a preallocated idx) with ragged rows or per-row K")
            total = rows * min(Ks, T)
        idx = torch.empty(max(total, 1), dtype=torch.int64, device=dR.device)
    if idx_offsets is None:
        idx_offsets = torch.empty(rows + 1, dtype=torch.int64, device=dR.device)
    rc = lib().chunk_topk_select(_ptr(dR), _ptr(offsets), rows, T, N, _ptr(Kp), Ks, _ptr(idx),
                                 _ptr(idx_offsets), None, 0, _ptr(dev_status), _stream(stream))
    _check("chunk_topk_select", rc)
    if total is not None:
        idx = idx[:total]
    return idx, idx_offsets


def chunk_gather(H, idx, idx_offsets, *, rows: int, T: int, offsets=None, total: Optional[int] = None,
                 Z=None, W_proj=None, Zp_f32=None, Zp_bf16=None, want_f32=True, want_bf16=True,
                 dev_status=None, stream=None):
    """Z = H[s_k] per row (bit-exact); with W_proj also (Z W_proj fp32, bf16)."""
    torch = _torch()
    _require_cuda(H, idx, idx_offsets, offsets, W_proj)
    H2 = H.reshape(-1, H.shape[-1]).contiguous()
    d = H2.shape[1]
    total = idx.numel() if total is None else total
    if Z is None:
        Z = torch.empty(total, d, dtype=H.dtype, device=H.device)
    d_g = 0
    if W_proj is not None:
        d_g = W_proj.shape[1]
        if want_f32 and Zp_f32 is None:
            Zp_f32 = torch.empty(total, d_g, dtype=torch.float32, device=H.device)
        if want_bf16 and Zp_bf16 is None:
            Zp_bf16 = torch.empty(total, d_g, dtype=torch.bfloat16, device=H.device)
    rc = lib().chunk_gather(_ptr(H2), _dtype_code(H2), _ptr(offsets), T, d, _ptr(idx), _ptr(idx_offsets),
                            rows, total, _ptr(Z), _ptr(W_proj), d_g, _ptr(Zp_f32), _ptr(Zp_bf16),
                            _ptr(dev_status), _stream(stream))
    _check("chunk_gather", rc)
    if W_proj is None:
        return Z
    return Z, Zp_f32, Zp_bf16


def chunk_upsample_workspace(rows: int, N: int, nbins: int) -> int:
    return int(lib().chunk_upsample_workspace(rows, N, nbins))


def chunk_upsample(G, H, idx, idx_offsets, W_bin, *, rows: int, T: int, offsets=None, mode: int = BIN_OFFSET,
                   S=None, workspace=None, dev_status=None, stream=None):
    """S = h_t + g_{c(t)} W_{b(t)} (fp32 [N, d_l])."""
    torch = _torch()
    _require_cuda(G, H, idx, idx_offsets, W_bin, offsets)
    H2 = H.reshape(-1, H.shape[-1]).contiguous()
    N, d_l = H2.shape
    nbins, d_g, _ = W_bin.shape
    if S is None:
        S = torch.empty(N, d_l, dtype=torch.float32, device=H.device)
    ws = _workspace(chunk_upsample_workspace(rows, N, nbins), H.device, workspace)
    rc = lib().chunk_upsample(_ptr(G.contiguous()), d_g, _ptr(H2), _dtype_code(H2), _ptr(offsets), T, N, d_l,
                              _ptr(idx), _ptr(idx_offsets), rows, _ptr(W_bin.contiguous()), nbins, int(mode),
                              _ptr(S), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream))
    _check("chunk_upsample", rc)
    return S


def chunk_upsample_noalloc(G, H, idx, idx_offsets, W_bin, *, rows: int, T: int, offsets=None,
                           mode: int = BIN_OFFSET, S=None, dev_status=None, stream=None):
    """chunk_upsample without a workspace: scratch comes from the library's static
    device array (N <= 1048576; calls that overlap on one device race on it)."""
    torch = _torch()
    _require_cuda(G, H, idx, idx_offsets, W_bin, offsets)
    H2 = H.reshape(-1, H.shape[-1]).contiguous()
    N, d_l = H2.shape
    nbins, d_g, _ = W_bin.shape
    if S is None:
        S = torch.empty(N, d_l, dtype=torch.float32, device=H.device)
    rc = lib().chunk_upsample_noalloc(_ptr(G.contiguous()), d_g, _ptr(H2), _dtype_code(H2), _ptr(offsets), T,
                                      N, d_l, _ptr(idx), _ptr(idx_offsets), rows, _ptr(W_bin.contiguous()),
                                      nbins, int(mode), _ptr(S), _ptr(dev_status), _stream(stream))
    _check("chunk_upsample_noalloc", rc)
    return S


def chunk_upsample_backward_workspace(rows: int, N: int, nbins: int, d_l: int) -> int:
    return int(lib().chunk_upsample_backward_workspace(rows, N, nbins, d_l))


def chunk_upsample_backward(dS, G, idx, idx_offsets, W_bin, *, rows: int, T: int, offsets=None,
                            mode: int = BIN_OFFSET, dG=None, dW=None, dH=None, residual: bool = True,
                            workspace=None, dev_status=None, stream=None):
    """Gradients of S = h + g_c W_b: (dG fp32 [K, d_g], dW fp32 [nbins, d_g, d_l], dH fp32 [N, d_l] = dS or
    None when residual is False)."""
    torch = _torch()
    _require_cuda(dS, G, idx, idx_offsets, W_bin, offsets)
    dS2 = dS.reshape(-1, dS.shape[-1]).contiguous()
    if dS2.dtype != torch.float32:
        raise TypeError("dS must be float32")
    N, d_l = dS2.shape
    nbins, d_g, _ = W_bin.shape
    K = G.shape[0]
    dev = dS.device
    if dG is None:
        dG = torch.empty(K, d_g, dtype=torch.float32, device=dev)
    if dW is None:
        dW = torch.empty(nbins, d_g, d_l, dtype=torch.float32, device=dev)
    if residual and dH is None:
        dH = torch.empty(N, d_l, dtype=torch.float32, device=dev)
    ws = _workspace(chunk_upsample_backward_workspace(rows, N, nbins, d_l), dev, workspace)
    rc = lib().chunk_upsample_backward(_ptr(dS2), _ptr(G.contiguous()), d_g, _ptr(offsets), T, N, d_l, _ptr(idx),
                                       _ptr(idx_offsets), rows, K, _ptr(W_bin.contiguous()), nbins, int(mode),
                                       _ptr(dG), _ptr(dW), _ptr(dH if residual else None), _ptr(ws), ws.numel(),
                                       _ptr(dev_status), _stream(stream))
    _check("chunk_upsample_backward", rc)
    return dG, dW, (dH if residual else None)


def chunk_gather_backward(dZ, idx, idx_offsets, *, rows: int, T: int, dH, offsets=None, accumulate: bool = True,
                          dev_status=None, stream=None):
    """dH[row start + s_k] (+)= dZ_k in place; returns dH."""
    _require_cuda(dZ, idx, idx_offsets, dH, offsets)
    dZ = dZ.contiguous()
    K, d = dZ.shape
    rc = lib().chunk_gather_backward(_ptr(dZ), d, _ptr(offsets), T, _ptr(idx), _ptr(idx_offsets), rows, K,
                                     _ptr(dH), int(bool(accumulate)), _ptr(dev_status), _stream(stream))
    _check("chunk_gather_backward", rc)
    return dH


def hnet_route_workspace(rows: int, N: int, d: int) -> int:
    return int(lib().hnet_route_workspace(rows, N, d))


def hnet_route(H, Wq, Wk, *, offsets=None, T: Optional[int] = None, threshold: float = 0.5,
               do_ema: bool = True, workspace=None, dev_status=None, stream=None):
    """(p fp32 [N], boundary u8 [N], chunk_idx int64 [N] (capacity), chunk_offsets int64 [rows+1],
    z_smooth fp32 [N, d] (capacity) or None)."""
    torch = _torch()
    _require_cuda(H, Wq, Wk, offsets)
    rows, T, N, d, H2 = _layout(H, offsets, T)
    H2 = H2.contiguous()
    dev = H.device
    p = torch.empty(N, dtype=torch.float32, device=dev)
    b = torch.empty(N, dtype=torch.uint8, device=dev)
    ci = torch.empty(max(N, 1), dtype=torch.int64, device=dev)
    co = torch.empty(rows + 1, dtype=torch.int64, device=dev)
    z = torch.empty(max(N, 1), d, dtype=torch.float32, device=dev) if do_ema else None
    ws = _workspace(hnet_route_workspace(rows, N, d), dev, workspace)
    rc = lib().hnet_route(_ptr(H2), _ptr(offsets), rows, T, N, d, _ptr(Wq.contiguous()), _ptr(Wk.contiguous()),
                          float(threshold), int(bool(do_ema)), _ptr(p), _ptr(b), _ptr(ci), _ptr(co), _ptr(z),
                          _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream))
    _check("hnet_route", rc)
    return p, b, ci, co, z


def chunk(H, K: int, eps2: float, *, stream=None):
    """Dense convenience pipeline: (dR, idx [rows, K'], Z [rows, K', d]) for H [rows, T, d]."""
    rows, T, d = H.shape
    dR = chunk_coding_rate(H, eps2, stream=stream)
    idx, io = chunk_topk_select(dR, K, rows=rows, T=T, stream=stream)
    Z = chunk_gather(H, idx, io, rows=rows, T=T, stream=stream)
    k = min(K, T)
    return dR.view(rows, T), idx.view(rows, k), Z.view(rows, k, d)


def canon_conv1d(H, w, bias=None, *, offsets=None, T: Optional[int] = None, residual: bool = False, out=None,
                 dev_status=None, stream=None):
    """Canon layer: out_t = bf16(bias (+ h_t) + sum_j w[:, j] h_{t-j}), per row, causal (bf16 in/out)."""
    torch = _torch()
    _require_cuda(H, w, bias, offsets)
    rows, T, N, d, H2 = _layout(H, offsets, T)
    H2 = H2.contiguous()
    if out is None:
        out = torch.empty(N, d, dtype=torch.bfloat16, device=H.device)
    rc = lib().canon_conv1d(_ptr(H2), _ptr(offsets), rows, T, N, d, _ptr(w.contiguous()),
                            _ptr(bias.contiguous() if bias is not None else None), int(bool(residual)), _ptr(out),
                            _ptr(dev_status), _stream(stream))
    _check("canon_conv1d", rc)
    return out


def chunk_coding_rate_canon(H, w, eps2: float, bias=None, *, offsets=None, T: Optional[int] = None,
                            residual: bool = False, Hc=None, dR=None, workspace=None, dev_status=None, stream=None):
    """(Hc, dR): the Canon layer's output and its marginal coding rate, in one call."""
    torch = _torch()
    _require_cuda(H, w, bias, offsets)
    rows, T, N, d, H2 = _layout(H, offsets, T)
    H2 = H2.contiguous()
    if Hc is None:
        Hc = torch.empty(N, d, dtype=torch.bfloat16, device=H.device)
    if dR is None:
        dR = torch.empty(N, dtype=torch.float32, device=H.device)
    ws = _workspace(chunk_coding_rate_workspace(rows, T, N, d), H.device, workspace)
    rc = lib().chunk_coding_rate_canon(_ptr(H2), _ptr(offsets), rows, T, N, d, _ptr(w.contiguous()),
                                       _ptr(bias.contiguous() if bias is not None else None), int(bool(residual)),
                                       _ptr(Hc), float(eps2), _ptr(dR), _ptr(ws), ws.numel(), _ptr(dev_status),
                                       _stream(stream))
    _check("chunk_coding_rate_canon", rc)
    return Hc, dR
