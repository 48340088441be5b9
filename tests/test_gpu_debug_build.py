"""The debug build (libdbc_debug.so, -DDBC_DEBUG: device-side checks of the
library's internal index invariants, which flag DBC_ERR_BOUNDS and skip the
access instead of trapping) runs the whole path on a small ragged batch with
no flag raised and the same results as the release build.

Runs in a child process because the binding loads one library per process
(DBC_LIBRARY=debug selects the debug one).
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
import workloads
import dynamic_byte_chunking_b200 as dbc
w = workloads.make("ragged", rows=5)
H = torch.from_numpy(w.H_bits.view(np.int16)).view(torch.bfloat16).cuda()
offs = torch.from_numpy(w.offsets).cuda()
st = torch.zeros(1, dtype=torch.int32, device="cuda")
dR = dbc.chunk_coding_rate(H, w.eps2, offsets=offs, T=w.T, dev_status=st)
Kt = torch.from_numpy(w.K).cuda()
total = int(np.minimum(w.K, w.lengths).sum())
idx, io = dbc.chunk_topk_select(dR, Kt, rows=w.rows, T=w.T, offsets=offs, total=total, dev_status=st)
Z = dbc.chunk_gather(H, idx, io, rows=w.rows, T=w.T, offsets=offs, total=total, dev_status=st)
Wb = torch.from_numpy(w.W_bin.view(np.int16)).view(torch.bfloat16).cuda()
S = dbc.chunk_upsample(Z, H, idx, io, Wb, rows=w.rows, T=w.T, offsets=offs, dev_status=st)
torch.cuda.synchronize()
print(json.dumps({"lib": dbc.lib_path, "st": int(st.item()), "dR": dR.cpu().numpy().tolist()[:4096:7],
                  "idx": idx.cpu().numpy().tolist(), "S": float(S.double().abs().sum().item())}))
""".replace("ROOT", repr(ROOT))


def _run(lib):
    env = dict(os.environ)
    if lib == "debug":
        env["DBC_LIBRARY"] = "debug"
    else:
        env.pop("DBC_LIBRARY", None)
    out = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_debug_build_runs_clean_and_matches_release():
    from dynamic_byte_chunking_b200 import build
    build.build(debug=True)
    dbg, rel = _run("debug"), _run("release")
    assert dbg["lib"].endswith("libdbc_debug.so") and rel["lib"].endswith("libdbc.so")
    assert dbg["st"] == 0 and rel["st"] == 0
    assert np.array_equal(np.array(dbg["dR"]), np.array(rel["dR"]))
    assert dbg["idx"] == rel["idx"]
    assert dbg["S"] == pytest.approx(rel["S"], rel=1e-9)
