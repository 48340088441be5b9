"""Data-parallel sharding of rows, checked with world_size-2 gloo ranks on CPU.

Each rank takes its rows, runs the chunking computation on them alone, and the
gathered per-rank results must equal the single-process result on the whole
batch (rows are independent, so no collective is needed on the data path).
The per-rank computation here is the float64 oracle (no GPU on this host); the
same partition drives bench.py's one-process-per-GPU runs.
"""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads
from dynamic_byte_chunking_b200.sharding import partition_rows, shard_rows_host


def test_partition_covers_rows_once_and_balances():
    rng = np.random.default_rng(0)
    lens = rng.integers(1024, 16385, size=256)
    for world in (1, 2, 3, 8):
        parts = partition_rows(lens, world)
        allr = np.concatenate(parts)
        assert np.array_equal(np.sort(allr), np.arange(256))
        loads = np.array([lens[p].sum() for p in parts])
        assert loads.max() - loads.min() <= lens.max()          # LPT bound
        for p in parts:
            assert np.all(np.diff(p) > 0)
    dense = partition_rows(np.full(10, 8192), 4)
    assert np.array_equal(np.concatenate(dense), np.arange(10))          # contiguous blocks in order
    assert max(len(p) for p in dense) - min(len(p) for p in dense) <= 1
    assert all(len(p) == 0 for p in partition_rows([], 3))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from oracle.chunking import gather, topk_select_rows
        from oracle.rank1 import dR_rank1
        w = workloads.make("ragged", rows=9, T_range=(100, 700), weights=False)
        mine = partition_rows(w.lengths, world)[rank]
        Hs, offs = shard_rows_host(w.H, w.offsets, mine)
        dR = dR_rank1(Hs, offs, w.eps2, nthreads=1)
        idx, io = topk_select_rows(dR, offs, w.K[mine])
        Z = gather(Hs, offs, idx, io)
        per_row = {int(r): (dR[offs[j]:offs[j + 1]], idx[io[j]:io[j + 1]], Z[io[j]:io[j + 1]])
                   for j, r in enumerate(mine)}
        out = [None] * world
        dist.all_gather_object(out, per_row)
        if rank == 0:
            merged = {}
            for d in out:
                merged.update(d)
            q.put(merged)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_single_process():
    from oracle.chunking import gather, topk_select_rows
    from oracle.rank1 import dR_rank1
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    merged = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = workloads.make("ragged", rows=9, T_range=(100, 700), weights=False)
    dR = dR_rank1(w.H, w.offsets, w.eps2)
    idx, io = topk_select_rows(dR, w.offsets, w.K)
    Z = gather(w.H, w.offsets, idx, io)
    assert sorted(merged) == list(range(w.rows))
    for r in range(w.rows):
        a, b = w.offsets[r], w.offsets[r + 1]
        d_r, i_r, z_r = merged[r]
        assert np.allclose(d_r, dR[a:b], rtol=1e-12, atol=0)
        assert np.array_equal(i_r, idx[io[r]:io[r + 1]])
        assert np.array_equal(z_r, Z[io[r]:io[r + 1]])
