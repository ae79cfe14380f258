"""The latent indexer's arithmetic and selection (latent_index.cu), modelled on the host in numpy and
checked against the oracle and brute force.

* Scoring: twice each E2M1 value as an integer (code nibble c -> +-{0,1,2,3,4,6,8,12}[c & 7], code
  2j of a byte in its low nibble), exact integer dots per (head, 32-channel block), each times the
  product of the two E8M0 block scales in fp64, summed over blocks and then heads (the ReLU variant
  clamps each head's dot at 0). This must equal 4 x the oracle's fp64 score for every position,
  which shows that the blockwise order of the sums loses nothing against the oracle's
  channel-by-channel order on such data.
* Selection: the orderable 64-bit key of each fp64 score (-0 folded onto +0), a radix select over
  eight 8-bit digits from the most significant one, then an ordered compaction of the keys above
  the k-th key T and of the lowest positions among those equal to T. This must give the Top-k of a
  full sort (score descending, position ascending), in ascending order, padded with -1, on random,
  heavily tied, all-equal and signed-zero rows.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W

MAG2 = [0, 1, 2, 3, 4, 6, 8, 12]  # twice the E2M1 magnitudes


def twice_values(codes: np.ndarray) -> np.ndarray:
    """[.., B] packed code bytes -> [.., 2B] integers (twice the E2M1 values)."""
    out = np.zeros(codes.shape[:-1] + (2 * codes.shape[-1],), np.int64)
    for half, off in ((codes & 15, 0), (codes >> 4, 1)):
        v = np.array([MAG2[c & 7] * (-1 if c & 8 else 1) for c in half.reshape(-1)], np.int64)
        out[..., off::2] = v.reshape(half.shape)
    return out


def model_scores(qcodes, qscale, kcodes, kscale, relu):
    qi, ki = twice_values(qcodes), twice_values(kcodes)
    hi, n = qi.shape[0], ki.shape[0]
    out = np.zeros(n)
    for p in range(n):
        total = 0.0
        for h in range(hi):
            dot = 0.0
            for b in range(4):
                I = int((qi[h, 32 * b:32 * b + 32] * ki[p, 32 * b:32 * b + 32]).sum())
                dot += float(I) * (math.ldexp(1.0, int(qscale[h, b]) - 127) * math.ldexp(1.0, int(kscale[p, b]) - 127))
            total += 0.0 if (relu and dot < 0.0) else dot
        out[p] = total
    return out


def score_key(s):
    u = (np.asarray(s, np.float64) + 0.0).view(np.uint64)
    return np.where(u >> np.uint64(63), ~u, u | np.uint64(1 << 63))


def model_select(keys, k):
    n = len(keys)
    if n <= k:
        return np.concatenate([np.arange(n), -np.ones(k - n, np.int64)])
    prefix, mask, rem = np.uint64(0), np.uint64(0), k
    for shift in range(56, -1, -8):
        m = (keys & mask) == prefix
        hist = np.bincount(((keys[m] >> np.uint64(shift)) & np.uint64(255)).astype(np.int64), minlength=256)
        acc, d = 0, 255
        while d > 0 and acc + hist[d] < rem:
            acc += hist[d]
            d -= 1
        rem -= acc
        prefix |= np.uint64(d) << np.uint64(shift)
        mask |= np.uint64(255) << np.uint64(shift)
    eq = keys == prefix
    eq_rank = np.cumsum(eq) - eq
    out = np.nonzero((keys > prefix) | (eq & (eq_rank < rem)))[0]
    assert len(out) == k
    return out


def full_sort_topk(s, k):
    n = len(s)
    top = np.sort(np.lexsort((np.arange(n), -np.asarray(s)))[:min(n, k)])
    return np.concatenate([top, -np.ones(k - len(top), np.int64)]) if n < k else top


@pytest.mark.parametrize("relu", [False, True])
@pytest.mark.parametrize("sigma", [1.0, 8.0, 1e-3])
def test_blockwise_exact_scores_equal_the_oracle(orc, relu, sigma):
    seed, n, hi = 5, 200, 32
    b = torch.tensor([0])
    keys = W.cache_values(seed, "lik", b, torch.arange(n), 128, sigma)[0]
    q = W.cache_values(seed, "liq", b, torch.tensor([n - 1]), hi * 128, sigma)[0, 0].reshape(hi, 128)
    oc = orc.LatentCache(n, 128)
    oc.append(0, idx_k=keys)
    idx, ref = oc.index_topk_full(n - 1, q, k=32, relu=relu)
    qd, qs = orc.mx_quantize_rows(q, 128)
    got = model_scores(qd, qs, oc.kdata[:n], oc.kscale[:n], relu)
    assert np.array_equal(got, 4.0 * ref)
    assert np.array_equal(model_select(score_key(got), 32), idx)


def test_radix_select_equals_full_sort():
    rng = np.random.default_rng(3)
    for trial in range(160):
        n, k = int(rng.integers(1, 4000)), int(rng.integers(1, 600))
        kind = trial % 4
        if kind == 0:
            s = rng.standard_normal(n)
        elif kind == 1:
            s = np.round(rng.standard_normal(n) * 3)  # many ties
        elif kind == 2:
            s = np.zeros(n)  # every score equal: the k lowest positions
        else:
            s = np.where(rng.random(n) < 0.5, -0.0, 0.0)  # signed zeros tie
        assert np.array_equal(model_select(score_key(s), k), full_sort_topk(s, k)), (trial, n, k)


def test_score_key_orders_like_the_scores():
    s = np.array([-np.inf, -1e300, -2.5, -1e-300, -0.0, 0.0, 1e-300, 3.0, 1e300, np.inf])
    key = score_key(s)
    assert (np.diff(key.astype(object)) >= 0).all()
    assert key[4] == key[5]  # -0 and +0 tie
    assert (np.diff(key[5:].astype(object)) > 0).all() and (np.diff(key[:5].astype(object)) > 0).all()
