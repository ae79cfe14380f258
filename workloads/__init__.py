"""Seeded synthetic inputs for the CSA2 layer step, shared by tests, bench.py and smoke().

This module holds none of the method's arithmetic. It only produces:
  * counter-addressed bf16 values with a near-Gaussian distribution (sum of twelve 16-bit
    uniforms, i.e. Irwin-Hall(12), unit variance, support +-6 sigma), scaled by sigma and
    clipped to +-clip (the pages bound post-RoPE magnitudes by about 26);
  * random distinct position / block-id sets, emitted in ascending order;
  * the shapes of the workloads (five layer-step configurations and a multi-token decode).

Every value is a pure function of (seed, stream, counter) built from integer operations,
one exact power-of-two scaling, one fp32 multiply by sigma, a clamp and one fp32 -> bf16
round-to-nearest-even. The same torch code therefore gives bit-identical values on the CPU
and on a GPU, so the oracle regenerates on the host exactly the inputs that a GPU run
generated on the device, without reading anything back from the device.

Definition (splitmix64 as published by Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", 2014):
    base      = splitmix64(seed * 2^32 + stream)
    h_j       = splitmix64(base + 3 * n + j),  j = 0, 1, 2   (64-bit wrapping adds)
    S         = sum over j and i < 4 of ((h_j >> 16 i) & 0xFFFF)
    z         = (S - 393210) / 65536
    value     = bf16_rne(clamp(fp32(z) * sigma, -clip, clip))
Cache counters address (sequence b, position p, channel c) as ((b << 21) + p) * width + c.
"""
from __future__ import annotations

import dataclasses

import torch

M64 = (1 << 64) - 1


def _s64(c: int) -> int:
    """Python int -> the signed int64 with the same 64-bit pattern."""
    c &= M64
    return c - (1 << 64) if c >= (1 << 63) else c


_GOLDEN = _s64(0x9E3779B97F4A7C15)
_C1 = _s64(0xBF58476D1CE4E5B9)
_C2 = _s64(0x94D049BB133111EB)

STREAM = {"kv": 1, "ik": 2, "swa": 3, "q": 4, "iq": 5, "pool": 6, "sel": 7,
          # the pages' own shape: 512-channel latent, 128-channel indexer key, window rows, query,
          # indexer query
          "lat": 8, "lik": 9, "lsw": 10, "lq": 11, "liq": 12}
POS_BITS = 21  # positions per sequence addressed by the counters: < 2^21


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of an int64 bit pattern."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64(x: torch.Tensor) -> torch.Tensor:
    z = x + _GOLDEN
    z = (z ^ _srl(z, 30)) * _C1
    z = (z ^ _srl(z, 27)) * _C2
    return z ^ _srl(z, 31)


def splitmix64_int(x: int) -> int:
    z = (x + 0x9E3779B97F4A7C15) & M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def stream_base(seed: int, stream: str | int) -> int:
    sid = STREAM[stream] if isinstance(stream, str) else int(stream)
    return _s64(splitmix64_int(((seed << 32) + sid) & M64))


def gaussian_bf16(seed: int, stream, counters: torch.Tensor, sigma: float = 1.0, clip: float = 26.0) -> torch.Tensor:
    """bf16 values for int64 `counters` (any shape, any device)."""
    base = stream_base(seed, stream)
    n3 = counters.to(torch.int64) * 3 + base
    s = None
    for j in range(3):
        h = splitmix64(n3 + j)
        for i in range(4):
            u = _srl(h, 16 * i) & 0xFFFF if i else h & 0xFFFF
            s = u if s is None else s + u
        del h
    z = (s - 393210).to(torch.float32) * (1.0 / 65536.0)
    del s
    z = torch.clamp(z * float(sigma), -float(clip), float(clip))
    return z.to(torch.bfloat16)


def cache_counters(b: torch.Tensor, p: torch.Tensor, width: int) -> torch.Tensor:
    """Counters for channels 0..width-1 of positions p (shape [..., P]) of sequences b ([...] or
    broadcastable): result [..., P, width]."""
    row = (b.to(torch.int64).unsqueeze(-1) << POS_BITS) + p.to(torch.int64)
    ch = torch.arange(width, dtype=torch.int64, device=p.device)
    return row.unsqueeze(-1) * width + ch


def cache_values(seed: int, stream, b: torch.Tensor, p: torch.Tensor, width: int, sigma: float = 1.0) -> torch.Tensor:
    return gaussian_bf16(seed, stream, cache_counters(b, p, width), sigma)


def distinct_sorted(seed: int, stream, b: torch.Tensor, n_range: int, count: int) -> torch.Tensor:
    """For each sequence in b (1-D), `count` distinct values of [0, n_range) chosen uniformly,
    ascending. Keys are unique, so the choice does not depend on the device's top-k."""
    base = stream_base(seed, stream)
    j = torch.arange(n_range, dtype=torch.int64, device=b.device)
    ctr = (b.to(torch.int64).unsqueeze(-1) << POS_BITS) + j
    h = splitmix64(ctr + base)
    key = ((_srl(h, 1) >> 22) << 22) | j  # unique: low bits carry the value itself
    sel = torch.topk(key, count, dim=-1, largest=False, sorted=False).indices
    return torch.sort(sel, dim=-1).values


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: str            # "full" | "reindex" | "minimal" | "prefill" | "draft" | "latent" | "latent_index"
    batch: int
    context: int         # N: visible positions for a decode query (query at N-1)
    seed: int
    k: int = 512
    pool_blocks: int = 0  # Full: blocks kept in the pool; Reindex: blocks given
    tq: int = 1           # query rows per sequence (prefill chunk length, draft tokens verified)
    hq: int = 16
    d: int = 128
    hi: int = 4
    di: int = 64
    hk: int = 4
    win: int = 128
    bs: int = 8


# The five layer-step workloads, shapes as stated for this hot path, and a multi-token decode.
WORKLOADS = {
    "full_b1_n4096": Workload("full_b1_n4096", "full", 1, 4096, seed=0),
    "full_b64_n131072": Workload("full_b64_n131072", "full", 64, 131072, seed=1, pool_blocks=2048),
    "reindex_b128_n1m": Workload("reindex_b128_n1m", "reindex", 128, 1 << 20, seed=2, pool_blocks=2000),
    "minimal_b256_n262144": Workload("minimal_b256_n262144", "minimal", 256, 262144, seed=3),
    "prefill_t4096_at_1m": Workload("prefill_t4096_at_1m", "prefill", 1, (1 << 20) + 4096, seed=4, tq=4096),
    # multi-token decode: each sequence appends 5 draft tokens at N-5 .. N-1 and verifies them together
    # (Full index over every visible position, row t sees positions <= N-5+t; no block pool)
    "draft_b64_n131072_tq5": Workload("draft_b64_n131072_tq5", "draft", 64, 131072, seed=5, tq=5),
    # the pages' own attention shape: 64 query heads x 512 over the 512-channel latent (K = V), a
    # decode row per sequence at N - 1 with 512 inherited selected entries and a 128-token window
    "latent_b128_n131072": Workload("latent_b128_n131072", "latent", 128, 131072, seed=6, hq=64, d=512),
    # the pages' own indexer: 32 query heads x 128 over one 128-channel MXFP4 key per entry, ReLU
    # scores, Top-512 of every visible entry, a decode row per sequence at N - 1
    "latent_index_b128_n131072": Workload("latent_index_b128_n131072", "latent_index", 128, 131072, seed=7, hi=32,
                                          di=128),
}
