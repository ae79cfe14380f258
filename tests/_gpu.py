"""Helpers for the GPU parity tests: the same seeded inputs, generated on the device for libcsa2
and regenerated on the host for the oracle (never copied from the device to the oracle)."""
from __future__ import annotations

import numpy as np
import torch

import compressed_sparse_attention_append_b200 as csa
import oracle
import workloads as W

DEV = "cuda"


def values(seed, stream, b, p, width, device, sigma=1.0):
    """bf16 [len(b), P, width] for sequences b ([B]) at positions p ([P] or [B, P])."""
    b = torch.as_tensor(b, dtype=torch.int64, device=device)
    p = torch.as_tensor(p, dtype=torch.int64, device=device)
    if p.dim() == 1:
        p = p.unsqueeze(0).expand(b.numel(), -1)
    return W.cache_values(seed, stream, b, p, width, sigma)


def query_values(seed, stream, b, qpos, width, device, sigma=1.0):
    """bf16 [len(b), width] for the query of sequence b at position qpos[b]."""
    b = torch.as_tensor(b, dtype=torch.int64, device=device)
    q = torch.as_tensor(qpos, dtype=torch.int64, device=device)
    return W.cache_values(seed, stream, b, q.unsqueeze(-1), width, sigma)[:, 0]


def gpu_fill(cache: csa.Cache, shape, seed, batch, n, sigma=1.0, chunk=4096, main=True, indexer=True, swa=True):
    """Append positions 0..n-1 of every sequence (bf16 from the generator, made on the GPU)."""
    b = torch.arange(batch, device=DEV)
    for p0 in range(0, n, chunk):
        t = min(chunk, n - p0)
        p = torch.arange(p0, p0 + t, device=DEV)
        pos = torch.full((batch,), p0, dtype=torch.int64, device=DEV)
        kv = values(seed, "kv", b, p, 256, DEV, sigma).contiguous() if main else None
        ik = values(seed, "ik", b, p, 256, DEV, sigma).contiguous() if indexer else None
        sw = values(seed, "swa", b, p, 256, DEV, sigma).contiguous() if swa else None
        csa.csa2_quantize_append(shape, cache, batch, t, pos, kv, ik, sw)


def oracle_seq(seed, b, n, cap, swa_cap, sigma=1.0, positions=None):
    """The oracle's cache of sequence b with positions 0..n-1 (or `positions`) appended."""
    c = oracle.SeqCache(cap=cap, swa_cap=swa_cap)
    pos = np.arange(n) if positions is None else np.asarray(positions)
    # contiguous runs keep the oracle's append simple
    runs = np.split(pos, np.nonzero(np.diff(pos) != 1)[0] + 1) if pos.size else []
    for r in runs:
        for p0 in range(0, r.size, 8192):
            rr = torch.from_numpy(r[p0:p0 + 8192])
            kv = values(seed, "kv", [b], rr, 256, "cpu", sigma)[0]
            ik = values(seed, "ik", [b], rr, 256, "cpu", sigma)[0]
            sw = values(seed, "swa", [b], rr, 256, "cpu", sigma)[0]
            c.append(int(rr[0]), kv=kv, idx_k=ik, swa_kv=sw)
    return c


def bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def attn_tol(oracle_out: np.ndarray, sigma: float = 1.0):
    """Tolerance of fp32 attention against the fp64 oracle: fp16 products of exact dequantised
    values, fp32 accumulation of <= 2176 terms and exp2 of fp32 logits give an error well below
    2e-3 of the output scale at unit-variance inputs; the scale grows with sigma."""
    return 2e-3 * max(1.0, sigma)
