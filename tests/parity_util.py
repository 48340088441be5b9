"""Shared helpers of the GPU parity tests (comparisons and tolerances).

Tolerances (spec contract of this library):
* dR: |gpu - oracle| <= rtol * max(|oracle|, 1e-6), rtol 2e-3 for fp32 input,
  1e-2 for bf16 input (fp32 accumulation);
* boundaries: v = the (K-1)-th largest oracle dR over t >= 1; every position
  whose oracle dR lies more than 1e-3 v from v is selected by the GPU exactly
  when the oracle selects it; plus exact count, strict order and idx[0] = 0;
* gather: bit-exact;
* upsample / projection: per element |d| <= 1e-3 (|o| + rms(o_row)) and per
  row |d| / |o| <= 1e-3;
* router: |p_gpu - p_oracle| <= 1e-3, boundary exact where |p_oracle - 1/2| > 1e-3;
  EMA relative 1e-3 per row (norm) on the GPU's own chunk list.
"""
import json
import os

import numpy as np

RTOL_F32 = 2e-3
RTOL_BF16 = 1e-2
BAND = 1e-3


def record(name, **kv):
    path = os.environ.get("DBC_METRICS_OUT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **{k: (float(v) if isinstance(v, (np.floating, float)) else v)
                                                 for k, v in kv.items()}}) + "\n")


def dR_rel_err(gpu, ref):
    return np.abs(gpu.astype(np.float64) - ref) / np.maximum(np.abs(ref), 1e-6)


def check_dR(gpu, ref, dtype, name=""):
    rel = dR_rel_err(gpu, ref)
    rtol = RTOL_F32 if dtype == "f32" else RTOL_BF16
    record(name + ":dR", max_rel=rel.max() if rel.size else 0.0, p99_rel=np.percentile(rel, 99) if rel.size else 0.0)
    assert rel.size == 0 or rel.max() <= rtol, f"{name}: dR max rel {rel.max():.3e} > {rtol}"
    return rel


def check_boundaries(sel_gpu, dR_oracle, K, name=""):
    """sel_gpu: increasing positions of one row chosen by the GPU."""
    from oracle.chunking import topk_select
    T = len(dR_oracle)
    want_n = min(K, T)
    sel_gpu = np.asarray(sel_gpu)
    assert len(sel_gpu) == want_n
    if want_n == 0:
        return 0
    assert sel_gpu[0] == 0
    assert np.all(np.diff(sel_gpu) > 0)
    assert sel_gpu[-1] < T
    if K >= T or K <= 1:
        assert np.array_equal(sel_gpu, topk_select(dR_oracle, K))
        return 0
    ref = topk_select(dR_oracle, K)
    v = np.sort(dR_oracle[1:])[::-1][K - 2]
    g = np.zeros(T, bool); g[sel_gpu] = True
    o = np.zeros(T, bool); o[ref] = True
    outside = np.abs(dR_oracle - v) > BAND * abs(v)
    outside[0] = True
    mism = np.nonzero(outside & (g != o))[0]
    record(name + ":boundaries", band_positions=int((~outside).sum()), mismatches=int(len(mism)))
    assert len(mism) == 0, f"{name}: {len(mism)} boundary mismatches outside the band, e.g. {mism[:5]}"
    return int((~outside).sum())


def check_close_rows(gpu, ref, name="", tol=1e-3):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.abs(gpu - ref)
    rms = np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True))
    elem = d / (np.abs(ref) + rms)
    row = np.linalg.norm(gpu - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)
    record(name, max_elem=elem.max() if elem.size else 0.0, max_row=row.max() if row.size else 0.0)
    assert elem.size == 0 or elem.max() <= tol, f"{name}: elementwise {elem.max():.3e}"
    assert row.size == 0 or row.max() <= tol, f"{name}: row {row.max():.3e}"
