"""Pins of the oracle's index scores (R2-R4), Top-K (R5, R6), block pool (R10) and Reindex.

Scores are checked against exact rational arithmetic on values decoded through the golden
E2M1 table and torch's E4M3 decoder; Top-K and pool against Python's sorted(); the pool
against the containment property that follows from its definition ("Pushing KV Cache
Compression to 890 Bytes per Token", sec. VI "Shortlist-of-a-shortlist", sec. IX Figure 4).
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import golden_rows

E2M1 = {int(c, 16): Fraction(float(v)) for c, v in golden_rows("e2m1_values.txt")}
E4M3 = [Fraction(float(v)) if not math.isnan(v) else None
        for v in torch.arange(256).to(torch.uint8).view(torch.float8_e4m3fn).double().tolist()]


def frac_dequant(data_row, scale_row, ch):
    out = []
    for c in range(ch):
        b = int(data_row[c // 2])
        code = (b >> 4) if c & 1 else (b & 15)
        out.append(E2M1[code] * E4M3[int(scale_row[c // 16])])
    return out


def make_cache(orc, n, hk=4, seed=0, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    c = orc.SeqCache(cap=n, swa_cap=256, hk=hk)
    kv = (torch.randn(n, 256, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    ik = (torch.randn(n, hk * 64, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    c.append(0, kv=kv, idx_k=ik)
    return c


def exact_scores(orc, c, idx_q, positions, hk, relu=False):
    qd, qs = orc.quantize_rows(idx_q, 64)
    hi = qd.shape[0]
    qv = [frac_dequant(qd[h], qs[h], 64) for h in range(hi)]
    out = []
    for p in positions:
        tot = Fraction(0)
        for h in range(hi):
            g = h * hk // hi
            kv = frac_dequant(c.ik_data[p, g * 32:(g + 1) * 32], c.ik_scale[p, g * 4:(g + 1) * 4], 64)
            dot = sum(a * b for a, b in zip(qv[h], kv))
            tot += max(dot, Fraction(0)) if relu else dot
        out.append(tot)
    return out


@pytest.mark.parametrize("hk,sigma", [(4, 1.0), (4, 8.0), (1, 1.0), (2, 0.01)])
def test_scores_exact(orc, hk, sigma):
    n = 48
    c = make_cache(orc, n, hk=hk, seed=hk, sigma=sigma)
    q = (torch.randn(4, 64, generator=torch.Generator().manual_seed(9)) * sigma).clamp(-26, 26).to(torch.bfloat16)
    pos = np.arange(n)
    got = c.scores(q, pos)
    want = exact_scores(orc, c, q, pos, hk)
    for g, w in zip(got, want):
        assert Fraction(g) == w  # the fp64 value is the exact rational
        assert (w * (1 << 20)).denominator == 1 and abs(w) < 2 ** 31
    got_r = c.scores_relu(q, pos)
    want_r = exact_scores(orc, c, q, pos, hk, relu=True)
    assert all(Fraction(g) == w for g, w in zip(got_r, want_r))


def test_score_one_hot_closed_form(orc):
    """q nonzero only at head 2, channel 37 (value 6*s_q): score = 6 s_q * deq(k[p, 2, 37])."""
    c = make_cache(orc, 16, seed=5)
    q = torch.zeros(4, 64)
    q[2, 37] = 3.0
    qb = q.to(torch.bfloat16)
    qd, qs = orc.quantize_rows(qb, 64)
    sq = orc.e4m3_decode(int(qs[2, 2]))
    assert sq == 0.5  # 3/6
    for p in range(16):
        kd = c.ik_data[p, 2 * 32 + 37 // 2]
        code = (kd >> 4) if 37 & 1 else (kd & 15)
        kval = orc.e2m1_decode(int(code)) * orc.e4m3_decode(int(c.ik_scale[p, 2 * 4 + 37 // 16]))
        assert c.scores(qb, [p])[0] == 6 * sq * kval


def brute_topk(scores, pos, k):
    ranked = sorted(zip(scores, pos), key=lambda t: (-t[0], t[1]))[:k]
    sel = sorted(p for _, p in ranked)
    return sel + [-1] * (k - len(sel))


@pytest.mark.parametrize("n,k,levels", [(0, 8, 3), (5, 8, 3), (100, 16, 4), (1000, 512, 7), (3000, 512, 1000)])
def test_topk_vs_sorted(orc, n, k, levels):
    rng = np.random.default_rng(n + k)
    s = rng.integers(0, levels, n).astype(np.float64) * 0.25  # many exact ties
    p = rng.permutation(10 * n + 1)[:n].astype(np.int64)
    got, m = orc.topk(s, p, k)
    assert got.tolist() == brute_topk(s.tolist(), p.tolist(), k)
    assert m == min(n, k)


def brute_pool(scores, bs, pb):
    n = len(scores)
    nb = (n + bs - 1) // bs
    bsc = [max(scores[b * bs:min(n, (b + 1) * bs)]) for b in range(nb)]
    return brute_topk(bsc, list(range(nb)), pb), min(nb, pb)


@pytest.mark.parametrize("n,pb", [(1, 4), (37, 4), (64, 8), (1001, 16), (5000, 2048)])
def test_pool_vs_brute(orc, n, pb):
    rng = np.random.default_rng(n)
    s = rng.integers(0, 9, n).astype(np.float64)
    got, m = orc.pool(s, 8, pb)
    want, wm = brute_pool(s.tolist(), 8, pb)
    assert got.tolist() == want and m == wm


@pytest.mark.parametrize("n,pb,k", [(4096, 512, 512), (4099, 600, 512), (2000, 64, 64)])
def test_full_topk_inside_pool_and_reindex_equals_full(orc, n, pb, k):
    """With pool_blocks >= k, every Top-k position lies in a pool block, so Reindex over the
    pool with the same query returns the Full Top-k."""
    c = make_cache(orc, n, seed=n)
    q = torch.randn(4, 64, generator=torch.Generator().manual_seed(n)).to(torch.bfloat16)
    qpos = n - 1
    idx, pool, pool_n = c.index_topk_full(qpos, q, k=k, pool_blocks=pb)
    blocks = set(pool[:pool_n].tolist())
    assert all(i // 8 in blocks for i in idx if i >= 0)
    assert pool_n == min(pb, (n + 7) // 8)
    assert list(pool[:pool_n]) == sorted(pool[:pool_n])
    re = c.index_topk_reindex(qpos, q, pool, pool_n, k=k)
    assert np.array_equal(re, idx)
    # independent Top-k over explicitly computed scores
    s = c.scores(q, np.arange(n))
    assert idx.tolist() == brute_topk(s.tolist(), list(range(n)), k)


def test_reindex_respects_causality_and_small_pool(orc):
    n = 200
    c = make_cache(orc, n, seed=3)
    q = torch.randn(4, 64, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    pool = np.array([0, 3, 7, 20, 24], np.int32)
    qpos = 163  # block 20 partially visible (160..163), block 24 not at all
    got = c.index_topk_reindex(qpos, q, pool, 5, k=64)
    cand = [b * 8 + j for b in pool for j in range(8) if b * 8 + j <= qpos]
    s = c.scores(q, np.array(cand))
    assert got.tolist() == brute_topk(s.tolist(), cand, 64)
    assert len([i for i in got if i >= 0]) == len(cand) == 28


def test_full_mode_small_context(orc):
    c = make_cache(orc, 100, seed=8)
    q = torch.randn(4, 64, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    idx = c.index_topk_full(9, q, k=16)
    assert idx.tolist() == list(range(10)) + [-1] * 6


@pytest.mark.parametrize("qpos", [0, 1, 2, 3, 98, 99, 150, 201])
def test_ratio_two_sees_only_complete_entries(orc, qpos):
    """R12 with r = 2: entry e summarises tokens 2e and 2e + 1, so a query at token i may use e only
    when 2e + 1 <= i. Full, pool and Reindex must rank exactly those entries."""
    n = 120
    c = make_cache(orc, n, seed=21)
    q = torch.randn(4, 64, generator=torch.Generator().manual_seed(qpos)).to(torch.bfloat16)
    vis = [e for e in range(n) if 2 * e + 1 <= qpos]  # brute force from the definition
    k = 24
    idx, pool, pool_n = c.index_topk_full(qpos, q, k=k, pool_blocks=5, ratio=2)
    if vis:
        s = c.scores(q, np.array(vis)).tolist()
        assert idx.tolist() == brute_topk(s, vis, k)
        bp, bpn = brute_pool(s, 8, 5)
        assert pool_n == bpn and pool.tolist() == bp
        # the same entries as the uncompressed cache queried at the last visible entry
        assert idx.tolist() == c.index_topk_full(len(vis) - 1, q, k=k).tolist()
    else:
        assert idx.tolist() == [-1] * k and pool_n == 0
    blocks = np.array([0, 4, 9, 14], np.int32)
    got = c.index_topk_reindex(qpos, q, blocks, 4, k=k, ratio=2)
    cand = [b * 8 + j for b in blocks for j in range(8) if b * 8 + j in set(vis)]
    want = brute_topk(c.scores(q, np.array(cand)).tolist(), cand, k) if cand else [-1] * k
    assert got.tolist() == want
