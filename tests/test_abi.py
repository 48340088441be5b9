"""The C-ABI library loads on a CPU-only host and exports every declared entry point.

No kernel is launched here: only symbol lookup, status names, the version and
the host-side workspace queries, which need no device.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dbc.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"DBC_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    import dynamic_byte_chunking_b200 as dbc
    from dynamic_byte_chunking_b200 import build
    build.build()
    return dbc.lib()


def test_header_declares_the_five_entry_points():
    names = _declared()
    for n in ("chunk_coding_rate", "chunk_topk_select", "chunk_gather", "chunk_upsample", "hnet_route"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in _declared():
        assert hasattr(L, n), n


def test_debug_library_exports_every_symbol():
    """The debug build (device-side invariant checks, -DDBC_DEBUG) links and exports the same ABI."""
    from dynamic_byte_chunking_b200 import build
    path = build.build(debug=True)
    D = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(D, n), n
    D.dbc_status_string.restype = ctypes.c_char_p
    assert D.dbc_status_string(6) == b"DBC_ERR_BOUNDS"


def test_status_strings_and_version(L):
    import dynamic_byte_chunking_b200 as dbc
    assert dbc.status_string(0) == "DBC_OK"
    assert dbc.status_string(7) == "DBC_ERR_WORKSPACE"
    assert dbc.version() >= 100


def test_workspace_queries_scale(L):
    import dynamic_byte_chunking_b200 as dbc
    a = dbc.chunk_coding_rate_workspace(8, 8192, 8 * 8192, 256)
    b = dbc.chunk_coding_rate_workspace(16, 8192, 16 * 8192, 256)
    assert 0 < a < b
    assert dbc.chunk_upsample_workspace(8, 65536, 16) > 65536
    # d = 256: the projections are fused on tensor cores; scratch = EMA block maps (3 x nblk x d fp32)
    N = 4096 * 64
    assert dbc.hnet_route_workspace(64, N, 256) >= 3 * (N // 64) * 256 * 4
    # d = 512 keeps an fp32 q|k buffer
    assert dbc.hnet_route_workspace(64, N, 512) >= N * 1024 * 4


def test_argument_errors_return_before_launch(L):
    # Host-side validation runs before any CUDA call, so it works without a GPU.
    f = L.chunk_coding_rate
    # eps2 <= 0
    assert f(None, 1, None, 1, 64, 64, 64, ctypes.c_float(0.0), None, None, 0, None, None) == 1
    # unsupported width
    assert f(None, 1, None, 1, 64, 64, 96, ctypes.c_float(0.5), None, None, 0, None, None) == 2
    # dense N mismatch
    assert f(None, 1, None, 2, 64, 64, 64, ctypes.c_float(0.5), None, None, 0, None, None) == 1
    # empty batch is a no-op success
    assert f(None, 1, None, 0, 64, 0, 64, ctypes.c_float(0.5), None, None, 0, None, None) == 0
    # K < 1
    assert L.chunk_topk_select(None, None, 1, 8, 8, None, 0, None, None, None, 0, None, None) == 1
    # bad bin count / mode
    u = L.chunk_upsample
    assert u(None, 64, None, 1, None, 8, 8, 64, None, None, 1, None, 0, 0, None, None, 0, None, None) == 1
    assert u(None, 64, None, 1, None, 8, 8, 64, None, None, 1, None, 16, 7, None, None, 0, None, None) == 1


def test_backward_argument_errors_return_before_launch(L):
    ub = L.chunk_upsample_backward
    # d_g not a multiple of 128
    assert ub(None, None, 64, None, 8, 8, 64, None, None, 1, 2, None, 16, 0, None, None, None, None, 0, None,
              None) == 2
    # nbins out of range
    assert ub(None, None, 128, None, 8, 8, 64, None, None, 1, 2, None, 0, 0, None, None, None, None, 0, None,
              None) == 1
    # missing outputs
    assert ub(None, None, 128, None, 8, 8, 64, None, None, 1, 2, None, 16, 0, None, None, None, None, 0, None,
              None) == 1
    gb = L.chunk_gather_backward
    # d not a multiple of 4
    assert gb(None, 6, None, 8, None, None, 1, 2, None, 1, None, None) == 2
    # nothing to do
    assert gb(None, 8, None, 8, None, None, 1, 0, None, 1, None, None) == 0
    import dynamic_byte_chunking_b200 as dbc
    assert dbc.chunk_upsample_backward_workspace(8, 65536, 16, 256) >= 2 * 65536 * 256 * 2


def test_stream_argument_errors_and_workspace(L):
    import dynamic_byte_chunking_b200 as dbc
    f = L.chunk_coding_rate_stream
    # fp32 input and d != 256 are not supported on this path
    assert f(None, 0, 1, 8, 256, 0, ctypes.c_float(0.5), None, None, None, 0, None, None) == 2
    assert f(None, 1, 1, 8, 128, 0, ctypes.c_float(0.5), None, None, None, 0, None, None) == 2
    # negative t0, bad eps2
    assert f(None, 1, 1, 8, 256, -1, ctypes.c_float(0.5), None, None, None, 0, None, None) == 1
    assert f(None, 1, 1, 8, 256, 0, ctypes.c_float(0.0), None, None, None, 0, None, None) == 1
    # an empty block is a no-op
    assert f(None, 1, 1, 0, 256, 7, ctypes.c_float(0.5), None, None, None, 0, None, None) == 0
    # the cut depends on t0: a block across 64 / 128 / 256 needs more segments than one inside [256, 512)
    a = dbc.chunk_coding_rate_stream_workspace(4, 256, 1, 256)
    b = dbc.chunk_coding_rate_stream_workspace(4, 256, 256, 256)
    assert a > b > 0


def test_step_argument_errors_return_before_launch(L):
    f = L.chunk_coding_rate_step
    dummy = ctypes.c_void_p(16)          # never dereferenced: every case returns before a launch
    odd = ctypes.c_void_p(20)            # not 16-byte aligned
    # dtype, d above 256 or not a multiple of 4
    assert f(dummy, 7, 1, 1, 256, ctypes.c_float(0.5), dummy, dummy, None, None) == 2
    assert f(dummy, 1, 1, 1, 260, ctypes.c_float(0.5), dummy, dummy, None, None) == 2
    assert f(dummy, 1, 1, 1, 30, ctypes.c_float(0.5), dummy, dummy, None, None) == 2
    # negative sizes, eps2 <= 0, missing buffers, a misaligned state
    assert f(dummy, 1, -1, 1, 256, ctypes.c_float(0.5), dummy, dummy, None, None) == 1
    assert f(dummy, 1, 1, 1, 256, ctypes.c_float(0.0), dummy, dummy, None, None) == 1
    assert f(None, 1, 1, 1, 256, ctypes.c_float(0.5), dummy, dummy, None, None) == 1
    assert f(dummy, 1, 1, 1, 256, ctypes.c_float(0.5), None, dummy, None, None) == 1
    assert f(dummy, 1, 1, 1, 256, ctypes.c_float(0.5), odd, dummy, None, None) == 1
    # no streams or no positions: nothing to do
    assert f(None, 1, 0, 1, 256, ctypes.c_float(0.5), None, None, None, None) == 0
    assert f(None, 1, 3, 0, 256, ctypes.c_float(0.5), None, None, None, None) == 0
