"""Seeded synthetic inputs for the byte-chunking hot path.

This module is shared by the oracle tests, the CUDA parity tests and the
benchmark.  It only draws random numbers and rounds them to the storage
precision; it holds none of the chunking arithmetic (no coding rate, no
selection, no upsampling, no routing).

Five workload families are defined, each a synthetic stand-in with the shapes
and statistics of the pages' workloads (real corpora are not used):

* ``tiny``      1 x 512 x 64 fp32, iid N(0, 1/d) features, eps^2 = 0.5, K = 128.
* ``byteflow``  8 x 8192 x 256 bf16, AR(1) rho = 0.9 along t per feature,
                eps^2 = 0.5, K = 2048, 16 upsampling bins W_bin ~ N(0, 1/d).
                (ByteFlow summary: T = 8192 byte sequences, B = 16 bins.)
* ``wide``      32 x 8192 x 512 bf16, AR(1) rho = 0.95 with restarts after
                Geometric(1/24) positions, eps^2 = 0.25, K = 1024, a 512 -> 1536
                chunk projection and 16 bins mapping 1536 -> 512.
* ``bytegen``   64 x 4096 x 256 bf16 built from a 32-byte packed market-event
                byte stream (ByteGen analysis report: PackedEvent format, event
                type mix of its Table 1, inter-event time median 0.271 ms and
                mean 13.311 ms): H = E[byte] + PE(t mod 32)/sqrt(d) + noise of
                variance 0.1; eps^2 = 0.5, K = 1024; router weights W_q, W_k.
* ``ragged``    256 sequences with lengths uniform in [1024, 16384], packed with
                int64 offsets, AR(1) rho = 0.9, d = 256, eps^2 = 0.5,
                K_i = ceil(T_i / 4), 16 bins.

Every family can be drawn at reduced sizes (fewer rows, shorter T) with the
same value distribution, which is what the small parity cases use.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "FAMILIES", "make", "bf16_bits", "bf16_to_f32",
    "NBINS", "DG_WIDE",
]

NBINS = 16          # position-in-chunk bins of the upsampler
DG_WIDE = 1536      # d_global of the wide family's chunk projection


# --------------------------------------------------------------------------
# storage-precision helpers (formatting only)
# --------------------------------------------------------------------------
def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns as uint16.  Inputs are finite by construction.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# workload container
# --------------------------------------------------------------------------
@dataclasses.dataclass
class Workload:
    """One synthetic batch.

    ``H`` is always float32 holding exactly the stored values (for bf16
    workloads the widened bf16 values); ``H_bits`` is what the device gets
    (uint16 bf16 patterns, or the float32 array itself for fp32 workloads).
    Rows are packed back to back: row ``r`` is ``H[offsets[r]:offsets[r+1]]``.
    """
    name: str
    dtype: str                      # "f32" or "bf16"
    d: int
    eps2: float
    offsets: np.ndarray             # int64 [rows + 1]
    H: np.ndarray                   # float32 [N, d]
    H_bits: np.ndarray              # uint16 [N, d] (bf16) or float32 [N, d]
    K: np.ndarray                   # int64 [rows]: chunks kept per row
    W_bin: Optional[np.ndarray] = None     # uint16 bf16 [NBINS, d_g, d_l]
    W_proj: Optional[np.ndarray] = None    # uint16 bf16 [d, d_g]
    Wq: Optional[np.ndarray] = None        # uint16 bf16 [d, d]
    Wk: Optional[np.ndarray] = None        # uint16 bf16 [d, d]
    byte_stream: Optional[np.ndarray] = None  # uint8 [N] (bytegen only)
    seed: int = 0

    @property
    def rows(self) -> int:
        return int(self.offsets.shape[0] - 1)

    @property
    def N(self) -> int:
        return int(self.offsets[-1])

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.offsets)

    @property
    def dense(self) -> bool:
        L = self.lengths
        return bool(np.all(L == L[0]))

    @property
    def T(self) -> int:
        """Common row length for dense batches, max length for ragged ones."""
        return int(self.lengths.max())

    def row(self, r: int) -> np.ndarray:
        return self.H[self.offsets[r]:self.offsets[r + 1]]

    def f32(self, name: str) -> np.ndarray:
        """A bf16 weight widened exactly to float32."""
        return bf16_to_f32(getattr(self, name))


# --------------------------------------------------------------------------
# value distributions
# --------------------------------------------------------------------------
def _ar1(rng: np.random.Generator, rows: int, T: int, d: int, rho: float,
         restart_p: float = 0.0) -> np.ndarray:
    """Per-feature AR(1) along t with unit stationary variance.

    x_0 ~ N(0,1); x_t = rho x_{t-1} + sqrt(1-rho^2) xi_t.  With restart_p > 0 a
    restart happens before position t with probability restart_p (so segment
    lengths are Geometric(restart_p), support >= 1) and x_t is redrawn N(0,1).
    """
    s = math.sqrt(1.0 - rho * rho)
    xi = rng.standard_normal((T, rows, d), dtype=np.float32)
    if restart_p > 0.0:
        restart = rng.random((T, rows)) < restart_p
    x = np.empty((T, rows, d), dtype=np.float32)
    x[0] = xi[0]
    r32, s32 = np.float32(rho), np.float32(s)
    for t in range(1, T):
        nxt = r32 * x[t - 1] + s32 * xi[t]
        if restart_p > 0.0:
            m = restart[t]
            nxt[m] = xi[t][m]
        x[t] = nxt
    return np.ascontiguousarray(x.transpose(1, 0, 2))  # [rows, T, d]


def _gauss_bf16(rng: np.random.Generator, shape, var: float) -> np.ndarray:
    w = rng.standard_normal(shape, dtype=np.float32) * np.float32(math.sqrt(var))
    return bf16_bits(w)


# ByteGen Table 1 event-type mix (ADD, MODIFY, CANCEL, FILL, OTHER) with the
# "OTHER" share split over the two remaining type codes of a 1-byte type field
# holding values 0..5.
_EVENT_TYPE_P = np.array([0.315, 0.368, 0.313, 0.002, 0.001, 0.001])


def _packed_events(rng: np.random.Generator, rows: int, events: int) -> np.ndarray:
    """Byte stream of 32-byte little-endian packed market events.

    Field layout (the pages give the fields, not offsets; this layout is ours):
    [0] type, [1..7] 56-bit order id, [8..15] u64 timestamp ns,
    [16..23] int64 price (random walk in ticks), [24..27] u32 size (Zipf 1.5),
    [28..31] u32 flags.
    """
    n = rows * events
    p = _EVENT_TYPE_P / _EVENT_TYPE_P.sum()
    etype = rng.choice(6, size=n, p=p).astype(np.uint64)
    oid = rng.integers(0, 1 << 56, size=n, dtype=np.uint64)
    mu = math.log(0.271e6)                      # median 0.271 ms in ns
    sigma = math.sqrt(2.0 * math.log(13.311 / 0.271))  # mean 13.311 ms
    gaps = rng.lognormal(mu, sigma, size=(rows, events))
    t0 = rng.integers(1_700_000_000_000_000_000, 1_800_000_000_000_000_000,
                      size=(rows, 1), dtype=np.int64).astype(np.float64)
    ts = (t0 + np.cumsum(gaps, axis=1)).astype(np.uint64).reshape(n)
    steps = rng.choice(np.array([-1, 1], dtype=np.int64), size=(rows, events))
    p0 = rng.integers(5_000_000, 10_000_000, size=(rows, 1), dtype=np.int64)
    price = (p0 + np.cumsum(steps, axis=1)).reshape(n).view(np.uint64)
    size = np.minimum(rng.zipf(1.5, size=n), (1 << 32) - 1).astype(np.uint64)
    flags = rng.integers(0, 1 << 32, size=n, dtype=np.uint64)

    out = np.zeros((n, 32), dtype=np.uint8)
    def put(col, val, nbytes):
        for b in range(nbytes):
            out[:, col + b] = ((val >> np.uint64(8 * b)) & np.uint64(0xFF)).astype(np.uint8)
    put(0, etype, 1)
    put(1, oid, 7)
    put(8, ts, 8)
    put(16, price, 8)
    put(24, size, 4)
    put(28, flags, 4)
    return out.reshape(rows, events * 32)


def _sinusoid(period: int, d: int) -> np.ndarray:
    """Standard sinusoidal position table (base 10000) for positions 0..period-1."""
    pos = np.arange(period, dtype=np.float64)[:, None]
    i = np.arange(d // 2, dtype=np.float64)[None, :]
    ang = pos / np.power(10000.0, 2.0 * i / d)
    pe = np.zeros((period, d), dtype=np.float64)
    pe[:, 0::2] = np.sin(ang)
    pe[:, 1::2] = np.cos(ang)
    return pe


# --------------------------------------------------------------------------
# families
# --------------------------------------------------------------------------
FAMILIES = ("tiny", "byteflow", "wide", "bytegen", "ragged")
_DEFAULT_SEED = {"tiny": 0, "byteflow": 1, "wide": 2, "bytegen": 3, "ragged": 4}


def make(name: str, seed: Optional[int] = None, rows: Optional[int] = None,
         T: Optional[int] = None, K: Optional[int] = None,
         T_range: Optional[tuple] = None, weights: bool = True) -> Workload:
    """Draw one batch of family ``name``.

    ``rows``/``T``/``K`` shrink a dense family for small parity cases (K then
    defaults to the family's T/K ratio).  For ``ragged`` use ``rows`` and
    ``T_range`` = (min_len, max_len).  ``weights=False`` skips the weight draws.
    """
    if name not in FAMILIES:
        raise ValueError(f"unknown workload family {name!r}")
    seed = _DEFAULT_SEED[name] if seed is None else seed
    rng = np.random.default_rng(seed)

    if name == "tiny":
        rows = 1 if rows is None else rows
        T = 512 if T is None else T
        d = 64
        K = max(1, T // 4) if K is None else K
        H = (rng.standard_normal((rows * T, d), dtype=np.float32)
             * np.float32(1.0 / math.sqrt(d)))
        offs = np.arange(rows + 1, dtype=np.int64) * T
        return Workload(name, "f32", d, 0.5, offs, H, H,
                        np.full(rows, K, dtype=np.int64), seed=seed)

    if name in ("byteflow", "wide"):
        if name == "byteflow":
            rows = 8 if rows is None else rows
            T = 8192 if T is None else T
            d, rho, rp, eps2 = 256, 0.9, 0.0, 0.5
            K = max(1, T // 4) if K is None else K
        else:
            rows = 32 if rows is None else rows
            T = 8192 if T is None else T
            d, rho, rp, eps2 = 512, 0.95, 1.0 / 24.0, 0.25
            K = max(1, T // 8) if K is None else K
        x = _ar1(rng, rows, T, d, rho, rp)
        Hb = bf16_bits((x * np.float32(1.0 / math.sqrt(d))).reshape(rows * T, d))
        offs = np.arange(rows + 1, dtype=np.int64) * T
        w = Workload(name, "bf16", d, eps2, offs, bf16_to_f32(Hb), Hb,
                     np.full(rows, K, dtype=np.int64), seed=seed)
        if weights:
            if name == "byteflow":
                w.W_bin = _gauss_bf16(rng, (NBINS, d, d), 1.0 / d)
            else:
                w.W_proj = _gauss_bf16(rng, (d, DG_WIDE), 1.0 / d)
                w.W_bin = _gauss_bf16(rng, (NBINS, DG_WIDE, d), 1.0 / DG_WIDE)
        return w

    if name == "bytegen":
        rows = 64 if rows is None else rows
        T = 4096 if T is None else T
        if T % 32:
            raise ValueError("bytegen rows hold whole 32-byte events")
        d = 256
        K = max(1, T // 4) if K is None else K
        stream = _packed_events(rng, rows, T // 32).reshape(rows * T)
        E = rng.standard_normal((256, d)) * math.sqrt(1.0 / d)
        pe = _sinusoid(32, d) / math.sqrt(d)
        noise = rng.standard_normal((rows * T, d)) * math.sqrt(0.1)
        pos = np.tile(np.arange(T) % 32, rows)
        Hf = (E[stream] + pe[pos] + noise).astype(np.float32)
        Hb = bf16_bits(Hf)
        offs = np.arange(rows + 1, dtype=np.int64) * T
        w = Workload(name, "bf16", d, 0.5, offs, bf16_to_f32(Hb), Hb,
                     np.full(rows, K, dtype=np.int64), byte_stream=stream, seed=seed)
        if weights:
            w.Wq = _gauss_bf16(rng, (d, d), 1.0 / d)
            w.Wk = _gauss_bf16(rng, (d, d), 1.0 / d)
            w.W_bin = _gauss_bf16(rng, (NBINS, d, d), 1.0 / d)
        return w

    # ragged
    rows = 256 if rows is None else rows
    lo, hi = (1024, 16384) if T_range is None else T_range
    d, rho = 256, 0.9
    lens = rng.integers(lo, hi + 1, size=rows, dtype=np.int64)
    offs = np.zeros(rows + 1, dtype=np.int64)
    offs[1:] = np.cumsum(lens)
    N = int(offs[-1])
    s = np.float32(math.sqrt(1.0 - rho * rho))
    Hb = np.empty((N, d), dtype=np.uint16)
    from scipy.signal import lfilter  # AR(1) filter per sequence
    scale = np.float32(1.0 / math.sqrt(d))
    for r in range(rows):
        n = int(lens[r])
        e = rng.standard_normal((n, d), dtype=np.float32)
        e[1:] *= s
        x = lfilter([1.0], [1.0, -rho], e, axis=0).astype(np.float32)
        Hb[offs[r]:offs[r + 1]] = bf16_bits(x * scale)
    Kr = (lens + 3) // 4
    w = Workload(name, "bf16", d, 0.5, offs, bf16_to_f32(Hb), Hb, Kr, seed=seed)
    if weights:
        w.W_bin = _gauss_bf16(rng, (NBINS, d, d), 1.0 / d)
    return w
