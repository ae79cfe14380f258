"""The oracle's side of the workloads: one sequence's cache and one step, regenerated on the host
from the seeded generator (workloads/__init__.py), positions filled exactly as the GPU builder fills
them. TEST INFRASTRUCTURE (tests, smoke and bench.py's CPU baseline only)."""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import workloads as W

from . import LatentCache, SeqCache


def _v(seed, stream, b, p, width):
    return W.cache_values(seed, stream, torch.tensor([b]), torch.as_tensor(p, dtype=torch.int64), width)[0]


def workload(name, context=None):
    wl = W.WORKLOADS[name]
    return dataclasses.replace(wl, context=context) if context else wl


def build_sequence(wl, b):
    """Returns (cache, inputs) of sequence b before its step."""
    N, seed = wl.context, wl.seed
    inp = {}
    if wl.mode == "latent_index":
        # the pages' own indexer: the MXFP4 key of every visible entry
        c = LatentCache(cap=N, swa_cap=128)
        for a in range(0, N, 16384):
            c.append(a, idx_k=_v(seed, "lik", b, torch.arange(a, min(N, a + 16384)), 128))
        inp["idx_q"] = _v(seed, "liq", b, [N - 1], wl.hi * 128)[0].reshape(wl.hi, 128)
        return c, inp
    if wl.mode == "latent":
        # the pages' own shape: the latent rows of the selected entries and the window rows
        c = LatentCache(cap=N, swa_cap=128)
        idx = W.distinct_sorted(seed, "sel", torch.tensor([b]), N - 1, wl.k)[0].numpy()
        inp["idx"] = idx.astype(np.int32)
        lat = _v(seed, "lat", b, idx.astype(np.int64), 512)
        for j, pp in enumerate(idx):
            c.append(int(pp), latent=lat[j:j + 1])
        pw = torch.arange(N - wl.win, N)
        c.append(N - wl.win, swa=_v(seed, "lsw", b, pw, 512))
        inp["q"] = _v(seed, "lq", b, [N - 1], 64 * 512)[0].reshape(64, 512)
        return c, inp
    if wl.mode == "prefill":
        p0 = N - wl.tq
        c = SeqCache(cap=N, swa_cap=1 << (wl.tq + wl.win - 1).bit_length())
        for a in range(0, p0, 16384):
            p = torch.arange(a, min(p0, a + 16384))
            c.append(a, kv=_v(seed, "kv", b, p, 256), idx_k=_v(seed, "ik", b, p, 256))
        pw = torch.arange(p0 - wl.win, p0)
        c.append(p0 - wl.win, swa_kv=_v(seed, "swa", b, pw, 256))
        p = torch.arange(p0, N)
        for n, s, w in (("kv", "kv", 256), ("idx_k", "ik", 256), ("swa_kv", "swa", 256), ("idx_q", "iq", 256),
                        ("q", "q", 2048)):
            inp[n] = _v(seed, s, b, p, w)
        return c, inp
    if wl.mode == "draft":
        p0 = N - wl.tq
        c = SeqCache(cap=N, swa_cap=1 << (wl.tq + wl.win - 1).bit_length(), hk=4)
        for a in range(0, p0, 16384):
            p = torch.arange(a, min(p0, a + 16384))
            c.append(a, kv=_v(seed, "kv", b, p, 256), idx_k=_v(seed, "ik", b, p, 256))
        pw = torch.arange(p0 - wl.win, p0)
        c.append(p0 - wl.win, swa_kv=_v(seed, "swa", b, pw, 256))
        p = torch.arange(p0, N)
        for n, s, w in (("kv", "kv", 256), ("idx_k", "ik", 256), ("swa_kv", "swa", 256), ("idx_q", "iq", 256),
                        ("q", "q", 2048)):
            inp[n] = _v(seed, s, b, p, w)
        return c, inp
    c = SeqCache(cap=N, swa_cap=128, hk=4)
    if wl.mode == "full":
        for a in range(0, N - 1, 16384):
            p = torch.arange(a, min(N - 1, a + 16384))
            c.append(a, kv=_v(seed, "kv", b, p, 256), idx_k=_v(seed, "ik", b, p, 256))
    elif wl.mode == "reindex":
        pool = W.distinct_sorted(seed, "pool", torch.tensor([b]), N // wl.bs, wl.pool_blocks)[0].numpy()
        inp["pool"] = pool.astype(np.int32)
        p = (torch.from_numpy(pool.astype(np.int64)).unsqueeze(1) * wl.bs + torch.arange(wl.bs)).reshape(-1)
        kv, ik = _v(seed, "kv", b, p, 256), _v(seed, "ik", b, p, 256)
        for j in range(pool.size):
            c.append(int(p[j * wl.bs]), kv=kv[j * wl.bs:(j + 1) * wl.bs], idx_k=ik[j * wl.bs:(j + 1) * wl.bs])
    else:  # minimal
        idx = W.distinct_sorted(seed, "sel", torch.tensor([b]), N - 1, wl.k)[0].numpy()
        inp["idx"] = idx.astype(np.int32)
        kv = _v(seed, "kv", b, idx.astype(np.int64), 256)
        for j, pp in enumerate(idx):
            c.append(int(pp), kv=kv[j:j + 1])
    pw = torch.arange(N - wl.win, N - 1)
    c.append(N - wl.win, swa_kv=_v(seed, "swa", b, pw, 256))
    qp = [N - 1]
    inp["swa_kv"] = _v(seed, "swa", b, qp, 256)
    inp["q"] = _v(seed, "q", b, qp, 2048)[0]
    if wl.mode != "minimal":
        inp["idx_q"] = _v(seed, "iq", b, qp, 256)[0]
    if wl.mode == "full":
        inp["kv"] = _v(seed, "kv", b, qp, 256)
        inp["idx_k"] = _v(seed, "ik", b, qp, 256)
    return c, inp


def run_step(c, wl, inp, rows=None):
    """One decode step (or the listed rows of a prefill chunk or a multi-token decode; all rows when
    rows is None) of the oracle. Returns a dict of results: idx/out/lse for one-row decode, else
    rows = {row: (idx, out, lse)}."""
    N = wl.context
    r = {}
    if wl.mode == "latent_index":
        r["idx"], _ = c.index_topk_full(N - 1, inp["idx_q"], k=wl.k, relu=True)
        return r
    if wl.mode == "latent":
        r["idx"] = inp["idx"]
        r["out"], r["lse"] = c.attend(N - 1, inp["q"], inp["idx"], win=wl.win)
        return r
    if wl.mode in ("prefill", "draft"):
        p0 = N - wl.tq
        c.append(p0, kv=inp["kv"], idx_k=inp["idx_k"], swa_kv=inp["swa_kv"])
        r["rows"] = {}
        for i in (range(wl.tq) if rows is None else rows):
            idx = c.index_topk_full(p0 + i, inp["idx_q"][i], k=wl.k)
            r["rows"][i] = (idx,) + c.sparse_attend(p0 + i, inp["q"][i], idx)
        return r
    if wl.mode == "full":
        c.append(N - 1, kv=inp["kv"], idx_k=inp["idx_k"], swa_kv=inp["swa_kv"])
        if wl.pool_blocks:
            r["idx"], r["pool"], r["pool_n"] = c.index_topk_full(N - 1, inp["idx_q"], k=wl.k, pool_blocks=wl.pool_blocks)
        else:
            r["idx"] = c.index_topk_full(N - 1, inp["idx_q"], k=wl.k)
    elif wl.mode == "reindex":
        c.append(N - 1, swa_kv=inp["swa_kv"])
        r["idx"] = c.index_topk_reindex(N - 1, inp["idx_q"], inp["pool"], len(inp["pool"]), k=wl.k)
    else:
        c.append(N - 1, swa_kv=inp["swa_kv"])
        r["idx"] = inp["idx"]
    r["out"], r["lse"] = c.sparse_attend(N - 1, inp["q"], r["idx"])
    return r
