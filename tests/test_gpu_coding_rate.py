"""GPU parity of the coding-rate chunker (dR -> Top-K -> gather) against the oracle.

Small cases span several segments and tiles with ragged tails and run every
position through the float64 rank-1 oracle; full-size cases (the five
workload families at their stated sizes, in the benchmark's launch
configuration) compare every row the oracle can afford, sampled otherwise.
"""
import numpy as np
import pytest

import workloads
from oracle.chunking import gather as oracle_gather
from oracle.chunking import topk_select
from oracle.coding_rate import dR_chol_diag, dR_prefix_logdet
from oracle.rank1 import dR_rank1
from parity_util import check_boundaries, check_dR, record

pytestmark = pytest.mark.gpu


def to_dev(w):
    import torch
    if w.dtype == "bf16":
        H = torch.from_numpy(w.H_bits.view(np.int16)).view(torch.bfloat16)
    else:
        H = torch.from_numpy(np.ascontiguousarray(w.H_bits))
    offs = torch.from_numpy(w.offsets).cuda()
    return H.cuda(), offs


def run_chunker(w, ragged):
    import torch
    import dynamic_byte_chunking_b200 as dbc
    H, offs = to_dev(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = offs if ragged else None
    dR = dbc.chunk_coding_rate(H, w.eps2, offsets=o, T=w.T, dev_status=st)
    Kt = torch.from_numpy(w.K).cuda()
    total = int(np.minimum(w.K, w.lengths).sum())
    idx, io = dbc.chunk_topk_select(dR, Kt, rows=w.rows, T=w.T, offsets=o, total=total, dev_status=st)
    Z = dbc.chunk_gather(H, idx, io, rows=w.rows, T=w.T, offsets=o, total=total, dev_status=st)
    torch.cuda.synchronize()
    return (dR.cpu().numpy(), idx.cpu().numpy(), io.cpu().numpy(), Z, int(st.item()))


def assert_gather_exact(w, Z, idx, io):
    import torch
    ref = oracle_gather(w.H_bits, w.offsets, idx, io)
    got = Z.cpu()
    if w.dtype == "bf16":
        got = got.view(torch.int16).numpy().view(np.uint16)
    else:
        got = got.numpy()
    assert np.array_equal(got, ref)


def check_rows(w, dR_gpu, idx, io, rows, ref, name):
    rtol_band = 0
    for r in rows:
        a, b = w.offsets[r], w.offsets[r + 1]
        check_dR(dR_gpu[a:b], ref[a:b], w.dtype, f"{name}/row{r}")
        rtol_band += check_boundaries(idx[io[r]:io[r + 1]], ref[a:b], int(w.K[r]), f"{name}/row{r}")
    return rtol_band


def _full_rows(w, ragged, rows=None, name=""):
    dR, idx, io, Z, st = run_chunker(w, ragged)
    assert st == 0
    rows = range(w.rows) if rows is None else rows
    sub = np.array(sorted(rows))
    # oracle on the chosen rows only
    offs = np.concatenate([[0], np.cumsum(w.lengths[sub])]).astype(np.int64)
    Hs = np.concatenate([w.row(r) for r in sub]) if len(sub) else np.zeros((0, w.d), np.float32)
    ref_sub = dR_rank1(Hs, offs, w.eps2)
    ref = np.zeros(w.N)
    for j, r in enumerate(sub):
        ref[w.offsets[r]:w.offsets[r + 1]] = ref_sub[offs[j]:offs[j + 1]]
    check_rows(w, dR, idx, io, sub, ref, name)
    # every row: count, order, BOS, and the bit-exact gather
    for r in range(w.rows):
        s = idx[io[r]:io[r + 1]]
        assert len(s) == min(int(w.K[r]), int(w.lengths[r]))
        if len(s):
            assert s[0] == 0 and np.all(np.diff(s) > 0) and s[-1] < w.lengths[r]
    assert_gather_exact(w, Z, idx, io)
    return dR, ref


# ---------------------------------------------------------------- small cases
def test_tiny_full_against_three_oracles():
    w = workloads.make("tiny")
    dR, idx, io, Z, st = run_chunker(w, False)
    assert st == 0
    h = w.row(0)
    o2 = dR_chol_diag(h, w.eps2)
    o1 = dR_prefix_logdet(h, w.eps2)
    assert np.max(np.abs(o1 - o2) / o2) < 1e-9
    check_dR(dR, o2, "f32", "tiny")
    check_boundaries(idx, o2, int(w.K[0]), "tiny")
    assert_gather_exact(w, Z, idx, io)


@pytest.mark.parametrize("fam,kw", [
    ("byteflow", dict(rows=3, T=1500)),
    ("wide", dict(rows=2, T=1200)),
    ("bytegen", dict(rows=3, T=1056)),
    ("tiny", dict(rows=2, T=777)),
])
def test_small_dense(fam, kw):
    w = workloads.make(fam, weights=False, **kw)
    _full_rows(w, False, name=f"small-{fam}")


def test_small_ragged_edge_lengths():
    # row lengths hit every segment edge: 1, 63/64/65, 127/128/129, 255..257,
    # 511..513, 1023..1025, and an empty row
    lens = [1, 63, 64, 65, 127, 128, 129, 255, 256, 257, 511, 512, 513, 0, 1023, 1024, 1025, 1600]
    rng = np.random.default_rng(7)
    H = (rng.standard_normal((sum(lens), 256)) / 16).astype(np.float32)
    Hb = workloads.bf16_bits(H)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    w = workloads.Workload("edges", "bf16", 256, 0.5, offs, workloads.bf16_to_f32(Hb), Hb,
                           np.maximum(1, (np.array(lens) + 3) // 4).astype(np.int64))
    _full_rows(w, True, name="edges")


def test_new_directions_late_in_row():
    # the first 1024 positions of each row span a 16-dimensional subspace, the rest every direction:
    # the whitened rows of the segment at 1024 are large again (|y|^2 in the hundreds), so the
    # in-segment Gram must take all six piece products there, not only in a row's first segments
    d, T, r = 256, 2048, 16
    rng = np.random.default_rng(11)
    rows = []
    for _ in range(2):
        U = np.linalg.qr(rng.standard_normal((d, r)))[0]
        low = rng.standard_normal((1024, r)) @ U.T / 4
        full = rng.standard_normal((T - 1024, d)) / 16
        rows.append(np.concatenate([low, full]))
    Hb = workloads.bf16_bits(np.concatenate(rows).astype(np.float32))
    offs = np.array([0, T, 2 * T], dtype=np.int64)
    w = workloads.Workload("late-directions", "bf16", d, 0.5, offs, workloads.bf16_to_f32(Hb), Hb,
                           np.full(2, T // 4, dtype=np.int64))
    _full_rows(w, False, name="late-directions")


def test_small_ragged_family():
    w = workloads.make("ragged", rows=7, T_range=(300, 2500), weights=False)
    _full_rows(w, True, name="small-ragged")


# ---------------------------------------------------------------- full sizes
def test_full_tiny():
    w = workloads.make("tiny")
    _full_rows(w, False, name="full-tiny")


def test_full_byteflow():
    w = workloads.make("byteflow", weights=False)
    _full_rows(w, False, name="full-byteflow")


def test_full_wide_sampled_rows():
    w = workloads.make("wide", weights=False)
    _full_rows(w, False, rows=[0, 13, 31], name="full-wide")


def test_full_bytegen():
    w = workloads.make("bytegen", weights=False)
    _full_rows(w, False, rows=range(0, 64, 4), name="full-bytegen")


def test_full_ragged_sampled_rows():
    w = workloads.make("ragged", weights=False)
    longest = int(np.argmax(w.lengths))
    shortest = int(np.argmin(w.lengths))
    _full_rows(w, True, rows=sorted({0, 17, 100, 255, longest, shortest}), name="full-ragged")


# ---------------------------------------------------------------- Top-K exactness
def test_topk_bit_exact_on_gpu_dR():
    """Same float32 inputs on both sides: the selection must be identical."""
    import torch
    import dynamic_byte_chunking_b200 as dbc
    rng = np.random.default_rng(3)
    lens = [1, 2, 5, 300, 4096, 16384, 0, 9000]
    Ks = [1, 5, 1, 300, 1024, 4096, 3, 8999]
    N = sum(lens)
    vals = rng.random(N).astype(np.float32)
    vals[rng.random(N) < 0.3] = 0.25          # heavy ties
    vals[100:140] = 0.0
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    d = torch.from_numpy(vals).cuda()
    o = torch.from_numpy(offs).cuda()
    Kt = torch.tensor(Ks, dtype=torch.int64, device="cuda")
    total = int(np.minimum(Ks, lens).sum())
    idx, io = dbc.chunk_topk_select(d, Kt, rows=len(lens), T=max(lens), offsets=o, total=total)
    idx, io = idx.cpu().numpy(), io.cpu().numpy()
    for r in range(len(lens)):
        want = topk_select(vals[offs[r]:offs[r + 1]].astype(np.float64), Ks[r]) if lens[r] else np.zeros(0)
        assert np.array_equal(idx[io[r]:io[r + 1]], want), r


@pytest.mark.parametrize("T,K", [(70000, 9000), (65537, 20000), (60000, 7), (49153, 30000)])
def test_topk_large_rows_from_global_memory(T, K):
    """Long rows: up to 65536 candidates the per-row CTA cluster (slices of up to 8192 keys in each
    CTA's shared memory), beyond that one CTA per row reading the keys from global memory."""
    import torch
    import dynamic_byte_chunking_b200 as dbc
    rng = np.random.default_rng(4)
    vals = rng.random(2 * T).astype(np.float32)
    vals[::7] = 0.5
    d = torch.from_numpy(vals).cuda()
    idx, io = dbc.chunk_topk_select(d, K, rows=2, T=T)
    idx = idx.cpu().numpy()
    for r in range(2):
        assert np.array_equal(idx[r * K:(r + 1) * K], topk_select(vals[r * T:(r + 1) * T].astype(np.float64), K))


def test_nonfinite_input_sets_status_flag():
    import torch
    import dynamic_byte_chunking_b200 as dbc
    w = workloads.make("byteflow", rows=1, T=600, weights=False)
    H, _ = to_dev(w)
    H.view(1, 600, 256)[0, 300, 5] = float("nan")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dbc.chunk_coding_rate(H.view(1, 600, 256), w.eps2, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() & (1 << dbc.ERR_NONFINITE)


def test_chunk_pipeline_dense_api():
    import torch
    import dynamic_byte_chunking_b200 as dbc
    w = workloads.make("byteflow", rows=2, T=2048, weights=False)
    H, _ = to_dev(w)
    dR, idx, Z = dbc.chunk(H.view(2, 2048, 256), 512, w.eps2)
    ref = dR_rank1(w.H, w.offsets, w.eps2)
    check_dR(dR.cpu().numpy().ravel(), ref, "bf16", "pipeline")
    assert idx.shape == (2, 512) and Z.shape == (2, 512, 256)
