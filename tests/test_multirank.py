"""Data-parallel host logic of bench.py on CPU ranks (gloo, world size 2).

The decode step shards by sequence: rank r owns sequences r*B .. r*B+B-1 and no data crosses ranks;
the only collective is the max over ranks of the timed region. These tests run that logic in two
spawned CPU processes: the max reduction, the weak-scaling throughput, that the shards are disjoint
and generate exactly the rows of one global batch, and that a rank which fails before the
collective ends the other rank's wait with an error instead of a hang.
"""
import multiprocessing as mp
import os
import socket
import sys
import traceback

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, mode, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import datetime

        import torch
        import torch.distributed as dist

        import bench
        import workloads as W

        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=20))
        if mode == "fail" and rank == 1:
            raise RuntimeError("rank 1 fails before the collective")
        B, steps = 4, 10
        ms_local = 100.0 + 37.5 * rank
        ms_max = bench.reduce_max(ms_local, "cpu", world)
        value = bench.weak_value(B, world, steps, ms_max)
        off = bench.shard_offset(rank, B)
        wl = W.WORKLOADS["reindex_b128_n1m"]
        seqs = torch.arange(off, off + B)
        qpos = torch.full((B,), wl.context - 1, dtype=torch.int64)
        rows = W.cache_values(wl.seed, "iq", seqs, qpos.unsqueeze(-1), 256, 1.0)[:, 0]
        gathered = [None] * world
        dist.all_gather_object(gathered, (off, rows.view(torch.int16).numpy().tobytes()))
        dist.destroy_process_group()
        q.put((rank, "ok", ms_max, value, gathered if rank == 0 else None))
    except Exception as e:  # reported to the parent, never raised past the process
        q.put((rank, "error", repr(e), traceback.format_exc(), None))


def _run(world, mode, timeout=120):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(world):
            r = q.get(timeout=timeout)
            out[r[0]] = r[1:]
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    return out


def test_max_over_ranks_and_weak_scaling():
    import torch

    import workloads as W

    out = _run(2, "ok")
    assert out[0][0] == "ok" and out[1][0] == "ok", out
    for r in (0, 1):
        _, ms_max, value, _ = out[r]
        assert ms_max == 137.5
        assert value == pytest.approx(4 * 2 * 10 / 0.1375)
    gathered = out[0][3]
    offs = [g[0] for g in gathered]
    assert offs == [0, 4]
    # the two shards are exactly the rows of one global batch of 8 sequences
    wl = W.WORKLOADS["reindex_b128_n1m"]
    seqs = torch.arange(8)
    qpos = torch.full((8,), wl.context - 1, dtype=torch.int64)
    glob = W.cache_values(wl.seed, "iq", seqs, qpos.unsqueeze(-1), 256, 1.0)[:, 0].view(torch.int16).numpy()
    assert gathered[0][1] == glob[:4].tobytes()
    assert gathered[1][1] == glob[4:].tobytes()
    assert gathered[0][1] != gathered[1][1]


def test_failed_rank_ends_the_wait_with_an_error():
    out = _run(2, "fail")
    assert out[1][0] == "error" and "fails before the collective" in out[1][1]
    assert out[0][0] == "error", out[0]
