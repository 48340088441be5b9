"""Row sharding for data-parallel runs (one process per GPU).

Rows (sequences) are independent units of the chunking path: dR, Top-K,
gather, upsampling and the router never read across a row.  A multi-GPU run
therefore partitions the rows over ranks and needs no collective on the data
path; results stay on their rank (or are gathered by the caller if it wants
them in one place).

* dense batches: contiguous, near-equal blocks of rows;
* ragged batches: longest-processing-time greedy on the per-row cost
  (the coding-rate work grows linearly in the row length), then each rank's
  rows are kept in their original order.
"""
from __future__ import annotations

import heapq
from typing import List, Sequence

import numpy as np

__all__ = ["partition_rows", "shard_offsets", "shard_rows_host"]


def partition_rows(lengths: Sequence[int], world: int, dense: bool | None = None) -> List[np.ndarray]:
    """Row indices owned by each rank (every row exactly once, ascending per rank)."""
    lengths = np.asarray(lengths, dtype=np.int64)
    rows = len(lengths)
    if world < 1:
        raise ValueError("world must be >= 1")
    if dense is None:
        dense = rows == 0 or bool(np.all(lengths == lengths[0]))
    if dense:
        bounds = np.linspace(0, rows, world + 1).round().astype(np.int64)
        return [np.arange(bounds[r], bounds[r + 1], dtype=np.int64) for r in range(world)]
    heap = [(0, r) for r in range(world)]            # (load, rank)
    owner = np.empty(rows, dtype=np.int64)
    for i in np.argsort(-lengths, kind="stable"):
        load, r = heapq.heappop(heap)
        owner[i] = r
        heapq.heappush(heap, (load + int(lengths[i]), r))
    return [np.nonzero(owner == r)[0].astype(np.int64) for r in range(world)]


def shard_offsets(lengths: Sequence[int], mine: np.ndarray) -> np.ndarray:
    """int64 offsets [len(mine) + 1] of a rank's rows packed back to back."""
    lengths = np.asarray(lengths, dtype=np.int64)
    out = np.zeros(len(mine) + 1, dtype=np.int64)
    out[1:] = np.cumsum(lengths[mine])
    return out


def shard_rows_host(H: np.ndarray, offsets: np.ndarray, mine: np.ndarray):
    """(H_shard, offsets_shard) gathered on the host for one rank."""
    offsets = np.asarray(offsets, dtype=np.int64)
    parts = [H[offsets[r]:offsets[r + 1]] for r in mine]
    Hs = np.concatenate(parts) if parts else H[:0]
    return Hs, shard_offsets(np.diff(offsets), mine)
