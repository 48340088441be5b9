#!/usr/bin/env python
"""Throughput of the dynamic byte-chunking hot path on B200.

One step = one pass of the whole path over one synthetic ByteFlow-shaped batch
(8 rows x 8192 bytes x d = 256, bf16 AR(1) features, eps^2 = 0.5, K = 2048,
16 upsampling bins): chunk_coding_rate -> chunk_topk_select -> chunk_gather ->
chunk_upsample, all through the C ABI (libdbc.so) on one stream.

Metric: sequence bytes per second (byte positions of the batch / step time).
Timing: W untimed warm-up steps, then exactly K steps, each preceded (outside
its timed interval) by a 256 MB write that flushes the 126 MB L2; CUDA events
on the launching stream; barrier + synchronize around the timed loop; max over
ranks.  The timed steps replay each of the four calls as a CUDA graph captured
after the warm-up (``--no-graph``: eager launches).  Under torchrun one global batch of 8 rows per rank is drawn and its
rows are split over the ranks by the library's row partition (weak scaling, no
collective on the data path).

``--impl reference`` times the float64 CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "coding-rate chunker bytes/sec at B=8,T=8192,d=256,K=2048; % of roofline"
UNIT = "bytes/s"
WORKLOAD = ("byteflow-shaped: rows=8, T=8192, d=256, bf16 AR(1) rho=0.9 features, eps^2=0.5, "
            "K=2048 (BOS + 2047 Top-K), gather, 16-bin upsample d_g=d_l=256, W_bin ~ N(0,1/d)")
FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dbc", choices=["dbc", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--e2e-lanes", type=int, default=2,
                    help="streams (each with its own buffers) that the end-to-end steps rotate over")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the device steps with eager launches instead of CUDA-graph replays")
    ap.add_argument("--rows", action="store_true",
                    help="time every hot-path row on its own workload family (one JSON line per row)")
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--families", default="tiny,byteflow,bytegen,wide,ragged",
                    help="workload families measured by --rows (comma-separated)")
    ap.add_argument("--probe", default=None, metavar="FAMILY",
                    help="run the path twice on one workload family (coding rate, Top-K, gather, upsample, the "
                         "router with EMA where the family has router weights, the Canon layer for bf16 "
                         "families), check the device status and exit: a short, fixed launch sequence for profilers")
    ap.add_argument("--traffic-from", default=None, metavar="CSV",
                    help="convert an ncu --csv launch list with dram__bytes_read.sum and dram__bytes_write.sum "
                         "(taken on this workload) into profiles/dram_traffic_byteflow.json, then exit")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", self.gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- oracle timing
def oracle_pipeline(w, rows):
    """The float64 oracle over the given rows: dR (C, all host threads), Top-K, gather, upsample."""
    from oracle.chunking import BIN_OFFSET, gather, topk_select_rows, upsample
    from oracle.rank1 import dR_rank1
    sub = np.asarray(rows)
    offs = np.concatenate([[0], np.cumsum(w.lengths[sub])]).astype(np.int64)
    H = np.concatenate([w.row(r) for r in sub])
    dR = dR_rank1(H, offs, w.eps2)
    idx, io = topk_select_rows(dR, offs, w.K[sub])
    Z = gather(H, offs, idx, io)
    W = w.f32("W_bin")
    upsample(Z, H, offs, idx, io, W, BIN_OFFSET)
    return int(offs[-1])


def cpu_baseline(w, min_seconds=10.0):
    """The oracle over the whole batch, repeated until about min_seconds of CPU work."""
    t0 = time.perf_counter()
    n = oracle_pipeline(w, range(w.rows))
    first = time.perf_counter() - t0
    reps = max(1, int(np.ceil(min_seconds / max(first, 1e-3))))
    for _ in range(reps - 1):
        n += oracle_pipeline(w, range(w.rows))
    dt = time.perf_counter() - t0
    # the C recursion runs one thread per row; the rest of the oracle is single-threaded
    return {"value": n / dt, "unit": UNIT, "cores": min(w.rows, os.cpu_count() or 1), "kind": "oracle",
            "sample": f"whole batch ({w.rows} x {w.T} positions) x {reps} through the float64 oracle: "
                      f"rank-1 C recursion for dR on all host threads, Top-K, gather, upsample; {dt:.2f} s"}


def strip_comments(text):
    """Kernel source without its comments: whole-line // comments, trailing // comments on lines
    without string literals, and /* */ blocks; blank lines dropped, runs of blanks collapsed."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = []
    for line in text.splitlines():
        if line.lstrip().startswith("//"):
            continue
        if '"' not in line:
            line = re.sub(r"\s*//.*$", "", line)
        line = " ".join(line.split())
        if line:
            out.append(line)
    return "\n".join(out)


def csrc_sha256():
    """Hash of the kernel sources with comments removed, to tell whether a stored ncu capture
    still describes the kernels (a comment edit does not change what was measured)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "dynamic_byte_chunking_b200", "csrc", "*"))):
        with open(f, encoding="utf-8") as fh:
            h.update(os.path.basename(f).encode())
            h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()


def stored_traffic(kernel):
    """DRAM bytes per call of `kernel` from profiles/dram_traffic_byteflow.json, or None when the
    capture is missing or was taken on other kernel sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic_byteflow.json")) as f:
            t = json.load(f)
        if t.get("csrc_sha256") != csrc_sha256():
            return None
        return t["bytes_per_call"].get(kernel)
    except Exception:
        return None


# kernel-name prefixes of each C-ABI call's kernels
STAGE_PREFIX = {"chunk_coding_rate": "cr::", "chunk_topk_select": "tk::", "chunk_gather": "ga::",
                "chunk_upsample": "up::"}


def write_traffic(csv_path):
    """Sum DRAM bytes per C-ABI call from an ncu CSV launch list and store them with the source hash.

    Each call's bytes are the sum over its kernels' launches divided by the number of times the
    call's first kernel launched (one per step)."""
    import csv
    with open(csv_path) as f:
        rows = [r for r in csv.reader(f)]
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    h = rows[hi]
    ki, mi, vi, ui, ii = (h.index("Kernel Name"), h.index("Metric Name"), h.index("Metric Value"),
                          h.index("Metric Unit"), h.index("ID"))
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}
    per_launch = {}
    for r in rows[hi + 1:]:
        if len(r) <= vi or r[mi] not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        name = r[ki]
        b = float(r[vi].replace(",", "")) * scale.get(r[ui], 1)
        per_launch.setdefault(r[ii], [name, 0.0])[1] += b
    out = {}
    for stage, pre in STAGE_PREFIX.items():
        launches = [(n, b) for n, b in per_launch.values() if pre in n]
        if not launches:
            continue
        first = launches[0][0].split("(")[0]
        calls = sum(1 for n, _ in launches if n.split("(")[0] == first)
        out[stage] = sum(b for _, b in launches) / calls
    path = os.path.join(ROOT, "profiles", "dram_traffic_byteflow.json")
    with open(path, "w") as f:
        json.dump({"csrc_sha256": csrc_sha256(), "source": os.path.basename(csv_path),
                   "bytes_per_call": out}, f, indent=1)
    print(json.dumps(out))


def stage_rooflines(avg_ms, N, d, rows, K, nb, pk, src):
    """Achieved / peak of every stage of the step from its event-timed average duration (avg_ms: stage
    name -> ms per call).

    Algorithmic work per call: coding rate 4 d^2 N flop (the rank-1 recursion: 2 d^2 for the solve and
    2 d^2 for the update per position) against the bf16 tensor peak; Top-K, gather and upsample their
    compulsory HBM bytes (read inputs once, write outputs once) against the HBM
    copy bandwidth."""
    flops_cr = 4.0 * d * d * N
    tf = pk.get("bf16_tflops", 1590.0)
    hbm = pk.get("hbm_gbs", 6650.0)
    out = {}
    by = {"chunk_topk_select": N * 4 + rows * K * 8 + (rows + 1) * 8,          # read dR, write idx
          "chunk_gather": 2 * rows * K * d * 2,                                 # read + write chunk rows
          "chunk_upsample": N * d * 2 + rows * K * d * 2 + nb * d * d * 2 + N * d * 4}   # H, G, W in; S out
    for st, ms in avg_ms.items():
        if st == "chunk_coding_rate":
            a = flops_cr / (ms * 1e-3) / 1e12
            out[st] = {"bound": "tensor", "achieved": a, "peak": tf, "unit": "TFLOP/s", "frac": a / tf,
                       "algorithmic": f"4*d^2*N = {flops_cr:.4g} flop per call",
                       "peak_source": src + " bf16 (burst)"}
        else:
            g = by[st] / (ms * 1e-3) / 1e9
            out[st] = {"bound": "hbm", "achieved": g, "peak": hbm, "unit": "GB/s", "frac": g / hbm,
                       "algorithmic": f"{by[st]} bytes per call", "peak_source": src}
    return out


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import workloads
    w = workloads.make("byteflow")
    for i in range(args.warmup):
        oracle_pipeline(w, [i % w.rows])
    t0 = time.perf_counter()
    n = 0
    for i in range(args.steps):
        n += oracle_pipeline(w, [i % w.rows])
    dt = time.perf_counter() - t0
    v = n / dt
    line = {"metric": METRIC, "value": v, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample_per_step": "one row (8192 positions)"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": "one 8192-position row per step through the float64 oracle "
                                       "(one row: one host thread)"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- per-row measurements
def _time(fn, reps, flush, stream):
    import torch
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return float(np.median(ts))


def _time_graph(fn, reps, flush, stream):
    """As _time, with fn captured once in a CUDA graph and replayed (kernel time without the host's
    per-call launch cost)."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    g.replay()
    torch.cuda.synchronize()
    ms = _time(g.replay, reps, flush, stream)
    del g
    return ms


def run_rows(args):
    """Each row of the hot path timed on the workload family it is specified on."""
    import torch
    import workloads
    import dynamic_byte_chunking_b200 as dbc
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    pk, src = peaks()
    hbm, tf = pk.get("hbm_gbs", 6650.0), pk.get("bf16_tflops", 1590.0)

    def bf(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)

    def emit(row, fam, ms, **kv):
        line = {"row": row, "workload": fam, "ms": ms, **kv, "peak_source": src}
        print(json.dumps(line), flush=True)

    for fam in [f for f in args.families.split(",") if f]:
        w = workloads.make(fam)
        H = bf(w.H_bits) if w.dtype == "bf16" else torch.from_numpy(w.H_bits).to(dev)
        offs = torch.from_numpy(w.offsets).to(dev)
        o = offs if not w.dense else None
        N, d, rows, T = w.N, w.d, w.rows, w.T
        ws = torch.empty(dbc.chunk_coding_rate_workspace(rows, T, N, d), dtype=torch.uint8, device=dev)
        dR = torch.empty(N, dtype=torch.float32, device=dev)
        Hx = H if o is not None else H.view(rows, T, d)
        ms = _time(lambda: dbc.chunk_coding_rate(Hx, w.eps2, offsets=o, T=T, dR=dR, workspace=ws), args.reps,
                   flush, stream)
        fl = 4.0 * d * d * N
        emit("A1 coding rate", fam, ms, positions_per_s=N / (ms * 1e-3), tflops=fl / (ms * 1e-3) / 1e12,
             frac_bf16_peak=fl / (ms * 1e-3) / 1e12 / tf)
        if w.dense and d == 256 and w.dtype == "bf16":
            # streaming continuation: the same rows fed as blocks of 256 positions with a carried state
            blk = 256
            Hs = H.view(rows, T, d)
            blocks = [Hs[:, t0:t0 + blk, :].contiguous() for t0 in range(0, T, blk)]
            state = torch.zeros(rows, d, d, dtype=torch.float64, device=dev)
            dRs = torch.empty(rows * blk, dtype=torch.float32, device=dev)
            wss = torch.empty(max(dbc.chunk_coding_rate_stream_workspace(rows, blk, t0, d)
                                  for t0 in range(0, T, blk)), dtype=torch.uint8, device=dev)

            def stream_pass():
                state.zero_()
                for j, b in enumerate(blocks):
                    dbc.chunk_coding_rate_stream(b, w.eps2, state, j * blk, dR=dRs, workspace=wss)

            ms = _time(stream_pass, args.reps, flush, stream)
            emit("NEXT-2 streaming coding rate (blocks of 256)", fam, ms, positions_per_s=N / (ms * 1e-3),
                 blocks=len(blocks), us_per_block=ms * 1e3 / len(blocks), tflops=fl / (ms * 1e-3) / 1e12)
            # latency of the smallest block: one new position per stream, 64 calls in a row mid-sequence
            t_mid = T // 2                       # mid-sequence, with 256 positions after it
            ones = [Hs[:, t:t + 1, :].contiguous() for t in range(t_mid, t_mid + 64)]
            ws1 = torch.empty(max(dbc.chunk_coding_rate_stream_workspace(rows, 1, t, d) for t in range(t_mid, t_mid + 64)),
                              dtype=torch.uint8, device=dev)
            dR1 = torch.empty(rows, dtype=torch.float32, device=dev)

            def byte_steps():
                for j, b in enumerate(ones):
                    dbc.chunk_coding_rate_stream(b, w.eps2, state, t_mid + j, dR=dR1, workspace=ws1)

            ms1 = _time_graph(byte_steps, args.reps, flush, stream)
            ms1e = _time(byte_steps, args.reps, flush, stream)
            emit("NEXT-2 streaming coding rate (one position per call)", fam, ms1, calls=len(ones),
                 us_per_call=ms1 * 1e3 / len(ones), us_per_call_eager=ms1e * 1e3 / len(ones), streams=rows,
                 launch="graph")
            # the per-position recursion (carried inverse factor): the same 64 one-position calls, and
            # 256 positions in one call
            Bst = dbc.step_state(rows, d, device=dev)

            def step_calls():
                for b in ones:
                    dbc.chunk_coding_rate_step(b, w.eps2, Bst, dR=dR1)

            ms2 = _time_graph(step_calls, args.reps, flush, stream)
            ms2e = _time(step_calls, args.reps, flush, stream)
            emit("NEXT-2 per-position recursion (one position per call)", fam, ms2, calls=len(ones),
                 us_per_call=ms2 * 1e3 / len(ones), us_per_call_eager=ms2e * 1e3 / len(ones), streams=rows,
                 launch="graph")
            blk256 = Hs[:, t_mid:t_mid + 256, :].contiguous()
            dR256 = torch.empty(rows * 256, dtype=torch.float32, device=dev)
            ms3 = _time(lambda: dbc.chunk_coding_rate_step(blk256, w.eps2, Bst, dR=dR256), args.reps, flush, stream)
            emit("NEXT-2 per-position recursion (256 positions per call)", fam, ms3, streams=rows,
                 us_per_position=ms3 * 1e3 / 256, positions_per_s=rows * 256 / (ms3 * 1e-3))
            del blocks, state, dRs, wss, ones, ws1, dR1, Bst, blk256, dR256
        if w.dtype == "bf16":
            # NEXT-4: the encoder's Canon layer (causal depthwise conv, k = 4) alone and chained with the chunker
            gen = np.random.default_rng(11)
            wc = bf(workloads.bf16_bits((gen.standard_normal((d, 4)) * 0.5).astype(np.float32)))
            bc = bf(workloads.bf16_bits((gen.standard_normal(d) * 0.02).astype(np.float32)))
            Hc = torch.empty(N, d, dtype=torch.bfloat16, device=dev)
            ms = _time(lambda: dbc.canon_conv1d(Hx, wc, bc, offsets=o, T=T, residual=True, out=Hc), args.reps, flush,
                       stream)
            by = 2 * N * d * 2
            emit("NEXT-4 Canon conv (k=4)", fam, ms, gbs=by / (ms * 1e-3) / 1e9, frac_hbm=by / (ms * 1e-3) / 1e9 / hbm)
            if d in (64, 128, 256, 512):
                ms = _time(lambda: dbc.chunk_coding_rate_canon(Hx, wc, w.eps2, bc, offsets=o, T=T, residual=True,
                                                               Hc=Hc, dR=dR, workspace=ws), args.reps, flush, stream)
                emit("NEXT-4 Canon conv + coding rate", fam, ms, positions_per_s=N / (ms * 1e-3))
            del Hc
        Kt = torch.from_numpy(w.K).to(dev)
        total = int(np.minimum(w.K, w.lengths).sum())
        idx = torch.empty(total, dtype=torch.int64, device=dev)
        io = torch.empty(rows + 1, dtype=torch.int64, device=dev)
        ms = _time(lambda: dbc.chunk_topk_select(dR, Kt, rows=rows, T=T, offsets=o, idx=idx, idx_offsets=io,
                                                 total=total), args.reps, flush, stream)
        by = N * 4 + total * 8
        emit("A2 top-k", fam, ms, gbs=by / (ms * 1e-3) / 1e9, frac_hbm=by / (ms * 1e-3) / 1e9 / hbm)
        Z = torch.empty(total, d, dtype=H.dtype, device=dev)
        ms = _time(lambda: dbc.chunk_gather(H, idx, io, rows=rows, T=T, offsets=o, total=total, Z=Z), args.reps,
                   flush, stream)
        by = 2 * total * d * H.element_size()
        emit("A3 gather", fam, ms, gbs=by / (ms * 1e-3) / 1e9, frac_hbm=by / (ms * 1e-3) / 1e9 / hbm)
        G = Z
        if w.W_proj is not None:
            Wp = bf(w.W_proj)
            dg = Wp.shape[1]
            Zf = torch.empty(total, dg, dtype=torch.float32, device=dev)
            Zb = torch.empty(total, dg, dtype=torch.bfloat16, device=dev)
            ms = _time(lambda: dbc.chunk_gather(H, idx, io, rows=rows, T=T, offsets=o, total=total, Z=Z, W_proj=Wp,
                                                Zp_f32=Zf, Zp_bf16=Zb), args.reps, flush, stream)
            fl = 2.0 * total * d * dg
            emit("A3 gather + W_proj", fam, ms, tflops=fl / (ms * 1e-3) / 1e12, frac_bf16_peak=fl / (ms * 1e-3) / 1e12 / tf)
            G = Zb
        if w.W_bin is not None:
            Wb = bf(w.W_bin)
            nb, dg, dl = Wb.shape
            S = torch.empty(N, dl, dtype=torch.float32, device=dev)
            wsu = torch.empty(dbc.chunk_upsample_workspace(rows, N, nb), dtype=torch.uint8, device=dev)
            ms = _time(lambda: dbc.chunk_upsample(G, H, idx, io, Wb, rows=rows, T=T, offsets=o, S=S, workspace=wsu),
                       args.reps, flush, stream)
            by = N * dl * H.element_size() + total * dg * 2 + nb * dg * dl * 2 + N * dl * 4
            fl = 2.0 * N * dg * dl
            emit("A4 upsample", fam, ms, gbs=by / (ms * 1e-3) / 1e9, frac_hbm=by / (ms * 1e-3) / 1e9 / hbm,
                 tflops=fl / (ms * 1e-3) / 1e12)
            if dg % 128 == 0:
                # backward of the upsampling + the gather's adjoint (dH = dS + scatter of dG)
                gen = torch.Generator(device=dev).manual_seed(7)
                dS = torch.randn(N, dl, dtype=torch.float32, device=dev, generator=gen)
                dG = torch.empty(total, dg, dtype=torch.float32, device=dev)
                dW = torch.empty(nb, dg, dl, dtype=torch.float32, device=dev)
                dH = torch.empty(N, dl, dtype=torch.float32, device=dev)
                wsb = torch.empty(dbc.chunk_upsample_backward_workspace(rows, N, nb, dl), dtype=torch.uint8,
                                  device=dev)

                def bwd():
                    dbc.chunk_upsample_backward(dS, G, idx, io, Wb, rows=rows, T=T, offsets=o, dG=dG, dW=dW, dH=dH,
                                                workspace=wsb)
                    if dg == dl and G is Z:
                        dbc.chunk_gather_backward(dG, idx, io, rows=rows, T=T, dH=dH, offsets=o)

                ms = _time(bwd, args.reps, flush, stream)
                # algorithmic bytes: read dS, G, W; write dG, dW, dH (the scatter into dH re-reads and writes
                # only boundary rows, counted once each way)
                by = (N * dl * 4 + total * dg * 2 + nb * dg * dl * 2 + total * dg * 4 + nb * dg * dl * 4
                      + N * dl * 4 + (2 * total * dl * 4 if dg == dl and G is Z else 0))
                emit("NEXT-1 upsample + gather backward", fam, ms, gbs=by / (ms * 1e-3) / 1e9,
                     frac_hbm=by / (ms * 1e-3) / 1e9 / hbm)
                del dS, dG, dW, dH, wsb
        if w.Wq is not None:
            Wq, Wk = bf(w.Wq), bf(w.Wk)
            wsr = torch.empty(dbc.hnet_route_workspace(rows, N, d), dtype=torch.uint8, device=dev)
            ms = _time(lambda: dbc.hnet_route(H, Wq, Wk, offsets=offs, T=T, do_ema=False, workspace=wsr), args.reps,
                       flush, stream)
            fl = 4.0 * N * d * d
            emit("A5 router", fam, ms, tflops=fl / (ms * 1e-3) / 1e12, frac_bf16_peak=fl / (ms * 1e-3) / 1e12 / tf)
            ms2 = _time(lambda: dbc.hnet_route(H, Wq, Wk, offsets=offs, T=T, do_ema=True, workspace=wsr), args.reps,
                        flush, stream)
            p, b, ci, co, z = dbc.hnet_route(H, Wq, Wk, offsets=offs, T=T, do_ema=True, workspace=wsr)
            nchunks = int(co[-1].item())
            by = nchunks * d * (H.element_size() + 4) + nchunks * 12
            emit("A6 EMA (router + EMA minus router)", fam, ms2 - ms, chunks=nchunks,
                 gbs=by / max((ms2 - ms) * 1e-3, 1e-9) / 1e9)
        del w, H, offs, ws, dR
        torch.cuda.empty_cache()


def run_probe(family, reps=2):
    """The path `reps` times on one family, in a fixed launch order (for ncu -k / -s / -c)."""
    import torch
    import workloads
    import dynamic_byte_chunking_b200 as dbc
    dev = torch.device("cuda", 0)
    w = workloads.make(family)
    H = torch.from_numpy(w.H_bits.view(np.int16)).view(torch.bfloat16).to(dev) if w.dtype == "bf16" else \
        torch.from_numpy(w.H_bits).to(dev)
    rows, T, d, N = w.rows, w.T, w.d, w.N
    o = None if w.dense else torch.from_numpy(w.offsets).to(dev)
    Hx = H.view(rows, T, d) if w.dense else H
    Kt = torch.from_numpy(w.K).to(dev)
    total = int(np.minimum(w.K, w.lengths).sum())
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(dbc.chunk_coding_rate_workspace(rows, T, N, d), dtype=torch.uint8, device=dev)
    dR = torch.empty(N, dtype=torch.float32, device=dev)
    Wb = (torch.from_numpy(w.W_bin.view(np.int16)).view(torch.bfloat16).to(dev)
          if w.W_bin is not None and w.W_proj is None else None)
    Wq = torch.from_numpy(w.Wq.view(np.int16)).view(torch.bfloat16).to(dev) if w.Wq is not None else None
    Wk = torch.from_numpy(w.Wk.view(np.int16)).view(torch.bfloat16).to(dev) if w.Wk is not None else None
    canon = None
    if w.dtype == "bf16":
        gen = np.random.default_rng(11)
        to_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        canon = (to_dev(workloads.bf16_bits((gen.standard_normal((d, 4)) * 0.5).astype(np.float32))),
                 to_dev(workloads.bf16_bits((gen.standard_normal(d) * 0.02).astype(np.float32))),
                 torch.empty(N, d, dtype=torch.bfloat16, device=dev))
    for _ in range(reps):
        dbc.chunk_coding_rate(Hx, w.eps2, offsets=o, T=T, dR=dR, workspace=ws, dev_status=st)
        idx, io = dbc.chunk_topk_select(dR, Kt, rows=rows, T=T, offsets=o, total=total, dev_status=st)
        Z = dbc.chunk_gather(H, idx, io, rows=rows, T=T, offsets=o, total=total, dev_status=st)
        if Wb is not None:
            dbc.chunk_upsample(Z, H, idx, io, Wb, rows=rows, T=T, offsets=o, dev_status=st)
        if Wq is not None:
            dbc.hnet_route(Hx, Wq, Wk, offsets=o, T=T, do_ema=True, dev_status=st)
        if canon is not None:
            dbc.canon_conv1d(Hx, canon[0], canon[1], offsets=o, T=T, residual=True, out=canon[2], dev_status=st)
    torch.cuda.synchronize()
    if st.item() != 0:
        raise RuntimeError(f"device status flags {st.item():#x}")
    print(json.dumps({"probe": family, "reps": reps, "launches": dbc.launch_count()}))


# ---------------------------------------------------------------- device arm
def main():
    args = parse()
    if args.traffic_from:
        write_traffic(args.traffic_from)
        return
    if args.probe:
        run_probe(args.probe)
        return
    if args.impl == "reference":
        run_reference(args)
        return
    if args.rows:
        run_rows(args)
        return
    import torch
    import workloads
    import dynamic_byte_chunking_b200 as dbc

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    stream = torch.cuda.current_stream()

    # one global batch of 8 rows per rank (weak scaling), its rows split over the ranks by the
    # library's row partition (contiguous blocks for a dense batch); no collective on the data path
    from dynamic_byte_chunking_b200 import sharding
    w = workloads.make("byteflow", seed=1, rows=8 * world)
    mine = sharding.partition_rows(w.lengths, world)[rank]
    H_bits, _ = sharding.shard_rows_host(w.H_bits, w.offsets, mine)
    rows, T, d, K = len(mine), w.T, w.d, int(w.K[0])
    N = rows * T
    H_host = torch.from_numpy(np.ascontiguousarray(H_bits).view(np.int16)).view(torch.bfloat16).pin_memory()
    H = H_host.to(dev).view(rows, T, d)
    Wb = torch.from_numpy(w.W_bin.view(np.int16)).view(torch.bfloat16).to(dev)
    nb = Wb.shape[0]
    dR = torch.empty(N, dtype=torch.float32, device=dev)
    idx = torch.empty(rows * K, dtype=torch.int64, device=dev)
    io = torch.empty(rows + 1, dtype=torch.int64, device=dev)
    Z = torch.empty(rows * K, d, dtype=torch.bfloat16, device=dev)
    S = torch.empty(N, d, dtype=torch.float32, device=dev)
    ws_cr = torch.empty(dbc.chunk_coding_rate_workspace(rows, T, N, d), dtype=torch.uint8, device=dev)
    ws_up = torch.empty(dbc.chunk_upsample_workspace(rows, N, nb), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    # the step: the four calls
    calls = {
        "chunk_coding_rate": lambda Hx: dbc.chunk_coding_rate(Hx, w.eps2, dR=dR, workspace=ws_cr, dev_status=st),
        "chunk_topk_select": lambda Hx: dbc.chunk_topk_select(dR, K, rows=rows, T=T, idx=idx, idx_offsets=io,
                                                              dev_status=st),
        "chunk_gather": lambda Hx: dbc.chunk_gather(Hx, idx, io, rows=rows, T=T, total=rows * K, Z=Z,
                                                    dev_status=st),
        "chunk_upsample": lambda Hx: dbc.chunk_upsample(Z, Hx, idx, io, Wb, rows=rows, T=T, S=S, workspace=ws_up,
                                                        dev_status=st)}
    stages = ["chunk_coding_rate", "chunk_topk_select", "chunk_gather", "chunk_upsample"]
    ns_ = len(stages)

    def step(Hx, ev=None):
        for i, name in enumerate(stages):
            if ev is not None:
                ev[i].record(stream)
            calls[name](Hx)
        if ev is not None:
            ev[ns_].record(stream)

    def check_status(when):
        # collective, so that every rank stops together when any rank saw a device flag
        flags = st.to(torch.int64)
        if pg:
            pg.all_reduce(flags, op=pg.ReduceOp.MAX)
        if flags.item() != 0:
            raise RuntimeError(f"device status flags {flags.item():#x} {when}")

    for _ in range(args.warmup):
        flush.zero_()
        step(H)
    torch.cuda.synchronize()
    check_status("during warm-up")

    # The timed steps replay each call as a CUDA graph (captured once, after the warm-up): the same
    # kernels with the same arguments, minus the host launch gaps between them.  `gpu_launches`
    # counts the kernels the graphs hold times the replays.
    graphs, per_step_launches, launch_mode = None, None, "eager"
    if not args.no_graph:
        try:
            l0 = dbc.launch_count()
            graphs = []
            for name in stages:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    calls[name](H)
                graphs.append(g)
            per_step_launches = dbc.launch_count() - l0
            torch.cuda.synchronize()
            for _ in range(2):
                flush.zero_()
                for g in graphs:
                    g.replay()
            torch.cuda.synchronize()
            check_status("during the graph warm-up")
            launch_mode = "cuda_graph"
        except Exception as exc:          # keep the eager steps if a capture is refused
            graphs = None
            launch_mode = "eager (graph capture failed: %s)" % str(exc).splitlines()[0][:120]
            torch.cuda.synchronize()

    def timed_step(ev):
        if graphs is None:
            step(H, ev)
            return
        for s_, g in enumerate(graphs):
            ev[s_].record(stream)
            g.replay()
        ev[ns_].record(stream)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(ns_ + 1)] for _ in range(args.steps)]
    gpu_id = str(local)
    try:
        props = torch.cuda.get_device_properties(dev)
        if getattr(props, "uuid", None) is not None:
            gpu_id = "GPU-" + str(props.uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    launches0 = dbc.launch_count()
    for k in range(args.steps):
        flush.zero_()
        timed_step(evs[k])
    torch.cuda.synchronize()
    launches = dbc.launch_count() - launches0 if graphs is None else per_step_launches * args.steps
    if pg:
        pg.barrier()
    time.sleep(0.2)
    clocks = sampler.stop()

    per_stage = np.zeros(ns_)
    total = 0.0
    for e in evs:
        for s in range(ns_):
            per_stage[s] += e[s].elapsed_time(e[s + 1])
        total += e[0].elapsed_time(e[ns_])
    t_ms = torch.tensor([total], dtype=torch.float64, device=dev)
    if pg:
        pg.all_reduce(t_ms, op=pg.ReduceOp.MAX)
    total_max = float(t_ms.item())
    ms_per_step = total_max / args.steps
    value = N * world / (ms_per_step * 1e-3)

    # ---- roofline of every stage, and of the dominant one (the coding-rate call)
    pk, src = peaks()
    avg = per_stage / args.steps          # ms per call
    stage_roof = stage_rooflines(dict(zip(stages, avg)), N, d, rows, K, nb, pk, src)
    dom = int(np.argmax(avg))
    roof = dict(stage_roof[stages[dom]])
    roof["traffic"] = stored_traffic(stages[dom])
    roof["kernel"] = stages[dom]
    # the metric's own definition: positions / (coding rate + Top-K + gather)
    t_chunk = float(sum(a_ for s_, a_ in zip(stages, avg) if s_ != "chunk_upsample"))
    value_chunk = N * world / (t_chunk * 1e-3)

    # ---- end to end through host buffers: every step copies its H from pinned host memory to the
    # device, runs the path through the API and reads (idx, Z, S) back into pinned host memory.  Steps
    # rotate over --e2e-lanes lanes, each with its own stream and buffers, so one step's device-to-host
    # copies overlap the next steps' host-to-device copies and compute (full-duplex copy engines).
    e2e = None
    if args.e2e_steps > 0:
        class Lane:
            def __init__(self):
                self.s = torch.cuda.Stream(device=dev)
                self.H = torch.empty(rows, T, d, dtype=torch.bfloat16, device=dev)
                self.dR = torch.empty(N, dtype=torch.float32, device=dev)
                self.idx = torch.empty(rows * K, dtype=torch.int64, device=dev)
                self.io = torch.empty(rows + 1, dtype=torch.int64, device=dev)
                self.Z = torch.empty(rows * K, d, dtype=torch.bfloat16, device=dev)
                self.S = torch.empty(N, d, dtype=torch.float32, device=dev)
                self.ws_cr = torch.empty_like(ws_cr)
                self.ws_up = torch.empty_like(ws_up)
                self.o_idx = torch.empty(rows * K, dtype=torch.int64).pin_memory()
                self.o_Z = torch.empty(rows * K, d, dtype=torch.bfloat16).pin_memory()
                self.o_S = torch.empty(N, d, dtype=torch.float32).pin_memory()

            def step(self):
                with torch.cuda.stream(self.s):
                    flush.zero_()
                    self.H.copy_(H_host.view(rows, T, d), non_blocking=True)
                    dbc.chunk_coding_rate(self.H, w.eps2, dR=self.dR, workspace=self.ws_cr, dev_status=st,
                                          stream=self.s)
                    dbc.chunk_topk_select(self.dR, K, rows=rows, T=T, idx=self.idx, idx_offsets=self.io,
                                          dev_status=st, stream=self.s)
                    dbc.chunk_gather(self.H, self.idx, self.io, rows=rows, T=T, total=rows * K, Z=self.Z,
                                     dev_status=st, stream=self.s)
                    dbc.chunk_upsample(self.Z, self.H, self.idx, self.io, Wb, rows=rows, T=T, S=self.S,
                                       workspace=self.ws_up, dev_status=st, stream=self.s)
                    self.o_idx.copy_(self.idx, non_blocking=True)
                    self.o_Z.copy_(self.Z, non_blocking=True)
                    self.o_S.copy_(self.S, non_blocking=True)

        nl = max(1, args.e2e_lanes)
        lanes = [Lane() for _ in range(nl)]
        torch.cuda.synchronize()
        for k in range(2 * nl):               # warm-up of every lane
            lanes[k % nl].step()
        torch.cuda.synchronize()
        main_s = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main_s)
        for ln in lanes:
            ln.s.wait_event(e0)
        for k in range(args.e2e_steps):
            lanes[k % nl].step()
        for ln in lanes:
            ev = torch.cuda.Event()
            ev.record(ln.s)
            main_s.wait_event(ev)
        e1.record(main_s)
        e1.synchronize()
        te = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
        if pg:
            pg.all_reduce(te, op=pg.ReduceOp.MAX)
        ms_e2e = float(te.item()) / args.e2e_steps
        ln = lanes[0]
        e2e = {"value": N * world / (ms_e2e * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": int(H_host.numel() * 2),
               "d2h_bytes_per_step": int(ln.o_idx.numel() * 8 + ln.o_Z.numel() * 2 + ln.o_S.numel() * 4),
               "ms_per_step": ms_e2e,
               "pipelining": f"{nl} lanes (streams) take steps in turn: device-to-host copies of one step overlap "
                             "the next steps' host-to-device copies and compute"}
        del lanes

    torch.cuda.synchronize()
    check_status("after the timed steps")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOAD, "rows_per_gpu": rows, "T": T, "d": d, "K": K, "nbins": nb,
                           "global_batch": 8 * world,
                           "parallelism": f"dp{world}: rows of one global batch split by sharding.partition_rows",
                           "l2": "flushed by a 256 MB write before every timed step",
                           "step": " -> ".join(stages), "launch": launch_mode},
                "stage_ms": {s: float(a) for s, a in zip(stages, avg)},
                "value_chunk": {"value": value_chunk, "unit": UNIT, "ms": t_chunk,
                                "definition": "positions / (coding rate + Top-K + gather)"},
                "stage_roofline": stage_roof,
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
                "clocks": clocks}
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
