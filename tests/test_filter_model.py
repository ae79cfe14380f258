"""The tensor-core filter's selection rule (several query rows per sequence), modelled on the host
and checked against brute force.

The device computes approximate scores S^ (fp32 MMA accumulation) with |S^ - S| <= eps for the exact
integer score S, and keeps the selection exact by these steps (index_mma.cu, mma_final_kernel):
  * tau = the R-th largest of the row's maxima over sampled 128-position tiles;
  * candidates = every visible position with S^ >= tau - 2 eps (rounded down), in per-item lists of
    bounded length;
  * the row is handed to the exact scan unless at least k candidates have S^ >= tau, no list
    overflowed and there are at most 4096 candidates;
  * A = the k-th largest S^ among the candidates with the low 8 bits of its orderable fp32 image
    cleared (a lower bound); R = {S^ >= A - 2 eps}; R is ranked by the exact S (score descending,
    position ascending).
These tests run that rule in numpy with scores perturbed anywhere within +-eps (random, and the worst
case: true members pushed down by eps and the others up by eps) and check that every row the rule
keeps gets exactly the Top-k of a full sort, and that the hand-over conditions catch the rows whose
estimate or lists cannot guarantee it.
"""
import numpy as np
import pytest

TILE, CAP, MAXR = 128, 4096, 4096


def order_f32(x):
    """Orderable uint32 image of fp32 values (larger float <-> larger image)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)


def unorder_f32(o):
    o = np.asarray(o, np.uint64)
    u = np.where(o & 0x80000000, o & 0x7FFFFFFF, (~o) & 0xFFFFFFFF).astype(np.uint32)
    return u.view(np.float32)


def exact_topk(S, k):
    """Top-k positions by (S descending, position ascending), returned ascending."""
    idx = np.lexsort((np.arange(len(S)), -S))[:k]
    return np.sort(idx)


def filter_model(S, Shat, eps, k, st, target=1536, item_tiles=64, subcap=64):
    """The device rule on one row (all positions visible). Returns the ascending Top-k, or None when
    the row would be handed to the exact scan."""
    n = len(S)
    assert n > CAP  # rows of at most 4096 positions are rescored whole on the device
    nt = (n + TILE - 1) // TILE
    ns = (nt + st - 1) // st
    samples = [s * st + (s * 7) % st for s in range(ns)]
    samples = [t for t in samples if t < nt]
    maxima = np.array([Shat[t * TILE:(t + 1) * TILE].max() for t in samples], np.float32)
    f = 1.0 - np.exp(128.0 * np.log1p(-target / n))
    R = int(np.clip(np.ceil(f * len(maxima)), 1, len(maxima)))
    tau = np.float32(np.sort(maxima)[::-1][R - 1])
    thr = np.float32(np.float64(tau) - 2.0 * eps)
    if np.float64(thr) > np.float64(tau) - 2.0 * eps:  # rounded down
        thr = np.nextafter(thr, np.float32(-np.inf))
    cand = np.nonzero(Shat >= thr)[0]
    # per-item lists of bounded length
    per_item = np.bincount(cand // (TILE * item_tiles), minlength=(nt + item_tiles - 1) // item_tiles)
    if (per_item > subcap).any() or len(cand) > CAP:
        return None
    if (Shat[cand] >= tau).sum() < k:
        return None
    img = order_f32(Shat[cand])
    kth = np.sort(img)[::-1][k - 1]
    A = unorder_f32(kth & ~np.uint64(0xFF))
    lo = np.float32(np.float64(A) - 2.0 * eps)
    if np.float64(lo) > np.float64(A) - 2.0 * eps:
        lo = np.nextafter(lo, np.float32(-np.inf))
    Rset = cand[Shat[cand] >= lo]
    if len(Rset) > MAXR:
        return None
    # the self-check on every rescored position
    if (np.abs(Shat[Rset].astype(np.float64) - S[Rset]) > eps).any():
        return None
    sel = Rset[np.lexsort((Rset, -S[Rset]))[:k]]
    return np.sort(sel)


def perturb(S, eps, rng, mode, k):
    if mode == "random":
        noise = rng.uniform(-eps, eps, len(S))
    else:  # worst case: the true Top-k pushed down, everything else pushed up
        noise = np.full(len(S), eps)
        noise[exact_topk(S, k)] = -eps
    out = (S + noise).astype(np.float32)
    # keep |S^ - S| <= eps after the fp32 rounding of the sum
    over = np.abs(out.astype(np.float64) - S) > eps
    out[over] = S[over].astype(np.float32)
    return out


@pytest.mark.parametrize("mode", ["random", "adversarial"])
@pytest.mark.parametrize("n,seed", [(20000, 1), (131072, 2), (262144, 3)])
def test_filter_rule_gives_the_exact_topk(n, seed, mode):
    rng = np.random.default_rng(seed)
    k, eps = 512, 0.25
    # integer-valued scores on a Gaussian scale with many near-ties around the k-th score
    S = np.round(rng.standard_normal(n) * 64.0).astype(np.float64)
    Shat = perturb(S, eps, rng, mode, k)
    st = max(1, ((n + TILE - 1) // TILE + 255) // 256)
    got = filter_model(S, Shat, eps, k, st, subcap=4096)
    ref = exact_topk(S, k)
    assert got is not None  # a well-spread row keeps the filter
    assert np.array_equal(got, ref)


def test_filter_rule_hands_over_a_row_whose_estimate_is_too_high():
    """Large scores only in the sampled tiles: tau lands above all but a few positions, fewer than k
    candidates reach it, and the row goes to the exact scan instead of returning a wrong set."""
    rng = np.random.default_rng(5)
    n, k, eps, st = 65536, 512, 0.25, 4
    S = np.round(rng.standard_normal(n) * 16.0).astype(np.float64)
    for s in range(((n + TILE - 1) // TILE + st - 1) // st):
        t = s * st + (s * 7) % st
        S[t * TILE:t * TILE + 2] += 1000.0  # two huge keys in every sampled tile only
    Shat = perturb(S, eps, rng, "random", k)
    assert filter_model(S, Shat, eps, k, st, subcap=4096) is None


def test_filter_rule_hands_over_overflowing_lists_and_equal_scores():
    """All scores equal (a zero query): every position is a candidate, the lists overflow, and the
    row goes to the exact scan (which returns the k lowest positions)."""
    n, k = 20000, 512
    S = np.zeros(n)
    Shat = np.zeros(n, np.float32)
    assert filter_model(S, Shat, 0.0, k, 1, subcap=64) is None
    assert np.array_equal(exact_topk(S, k), np.arange(k))


def test_filter_rule_self_check_catches_a_broken_error_bound():
    """A score off by more than eps near the cut: the rescored set's self-check hands the row over
    rather than trusting a candidate set that may miss a true member."""
    rng = np.random.default_rng(7)
    n, k, eps = 20000, 512, 0.25
    S = np.round(rng.standard_normal(n) * 64.0).astype(np.float64)
    Shat = perturb(S, eps, rng, "random", k)
    ref = exact_topk(S, k)
    kth = S[ref].min()
    near = np.nonzero(np.abs(S - kth) < 1.0)[0][0]
    Shat[near] = np.float32(S[near] + 3.0)  # an error of 3 > eps
    assert filter_model(S, Shat, eps, k, max(1, (n // TILE + 255) // 256), subcap=4096) is None


def test_lower_bound_of_kth_image_keeps_at_least_k():
    """Clearing the low 8 bits of the k-th largest orderable image gives a value with at least k
    candidates at or above it, for positive, negative and mixed-sign scores."""
    rng = np.random.default_rng(11)
    for scale, shift in ((1.0, 0.0), (1.0, -50.0), (1e-3, 0.0), (1e6, 0.0)):
        x = (rng.standard_normal(3000) * scale + shift).astype(np.float32)
        img = order_f32(x)
        for k in (1, 17, 512, 3000):
            kth = np.sort(img)[::-1][k - 1]
            A = unorder_f32(kth & ~np.uint64(0xFF))
            assert (x >= A).sum() >= k
            assert A <= unorder_f32(kth)


def test_filter_rule_margins_are_tight():
    """A constructed row where both 2 eps margins are needed. Every tile holds a key with S^ = tau and
    S = tau - eps (k of them); position 0 has S = tau - eps too, but S^ = tau - 2 eps. Position 0 wins
    the tie on S by its lower position, so it is a true member, and only an admission threshold of
    tau - 2 eps and a rescoring floor of A - 2 eps keep it."""
    n, k, eps, tau = 20480, 512, 1.0, 10.0
    S = np.full(n, -100.0)
    Shat = np.full(n, -100.0, np.float32)
    high = (np.arange(k) * n) // k + 1  # one in every 128-position tile, none at position 0
    S[high], Shat[high] = tau - eps, tau
    S[0], Shat[0] = tau - eps, tau - 2 * eps
    ref = exact_topk(S, k)
    assert ref[0] == 0
    got = filter_model(S, Shat, eps, k, 1, subcap=4096)
    assert got is not None and np.array_equal(got, ref)
