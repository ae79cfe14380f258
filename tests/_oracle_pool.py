"""The oracle's results for many sequences (or prefill rows) of a full-size workload, computed in
spawned host processes (never forked from a process that used CUDA), so that a full-size GPU test
can check every sequence of a workload and not only a sample."""
from __future__ import annotations

import multiprocessing as mp
import os


def _seq_job(job):
    name, b, rows = job
    import torch

    torch.set_num_threads(1)  # one process per core: no intra-op threads on top
    from oracle import workload as OW

    wl = OW.workload(name)
    c, inp = OW.build_sequence(wl, b)
    r = OW.run_step(c, wl, inp, rows=rows)
    del c
    return b, r


def oracle_steps(name, seqs, rows=None, procs=None):
    """{sequence: oracle step result} for the listed sequences of workload `name` (for a prefill
    chunk or a multi-token decode, `rows` selects the query rows; a list of lists gives one job per
    row group, all on sequence 0). Workers start with OMP_NUM_THREADS=1 and one torch thread."""
    procs = procs or max(1, min(16, os.cpu_count() or 1))
    if rows is not None and rows and isinstance(rows[0], (list, tuple)):
        jobs = [(name, 0, list(g)) for g in rows]
    else:
        jobs = [(name, b, rows) for b in seqs]
    old = os.environ.get("OMP_NUM_THREADS")
    os.environ["OMP_NUM_THREADS"] = "1"
    try:
        with mp.get_context("spawn").Pool(min(procs, len(jobs))) as pool:
            out = pool.map(_seq_job, jobs, chunksize=1)
    finally:
        if old is None:
            os.environ.pop("OMP_NUM_THREADS", None)
        else:
            os.environ["OMP_NUM_THREADS"] = old
    if rows is not None and rows and isinstance(rows[0], (list, tuple)):
        merged = {"rows": {}}
        for _, r in out:
            merged["rows"].update(r["rows"])
        return {0: merged}
    return dict(out)
