"""Oracle for the dynamic byte-chunking hot path: plain, slow, float64 CPU code.

TEST INFRASTRUCTURE.  Only the test-suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import, call, link or execute anything in this
package.  The CUDA product path never reaches it, and the two share no code:
the only common module is ``workloads`` (seeded inputs, no chunking arithmetic).

Contents (each function cites the passage it follows):
* ``coding_rate``  R_eps and dR by prefix logdets (O1) and by the Cholesky
                   diagonal of the T x T Gram (O2);
* ``rank1``        dR by a rank-1 Cholesky recursion in plain C (O3, timed);
* ``chunking``     Top-K boundary selection, gather, multi-linear upsampling;
* ``router``       cosine router and EMA smoothing.

Pins (tests under ``tests/test_oracle*.py``): closed forms for orthogonal,
repeated, axis-aligned and two-vector inputs, d = 1; the telescoping sum vs the
SVD; bounds and invariances; O1 = O2 = O3; brute-force Top-K on T <= 12; one-hot
and identity upsampling tags; router special angles; EMA closed forms.
"""
from . import coding_rate, chunking, router, rank1  # noqa: F401
from .coding_rate import coding_rate as R_eps, dR_prefix_logdet, dR_chol_diag  # noqa: F401
from .rank1 import dR_rank1  # noqa: F401
from .chunking import (topk_select, topk_select_rows, gather, chunk_of, bin_of,  # noqa: F401
                       upsample_row, upsample, BIN_OFFSET, BIN_FRACTION, BIN_ABSOLUTE)
from .router import route_row, ema, route  # noqa: F401
