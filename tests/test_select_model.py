"""The decode select's placement rule, modelled on the host and checked against brute force.

The select kernel never orders two keys by their bins: bins only decide which keys reach the exact
comparison. These tests check the two facts that argument rests on, on a host model of the rule:
  * the bin functions (score rounded to fp32 with round-to-nearest-even, then sign, exponent and
    mantissa bits) never put a larger key in a lower bin, including at every rounding boundary;
  * keys above the cut bin, plus the keys above the second-level cut inside it, plus the exact
    ranking of the keys left in the second-level cut bin, give exactly the Top-k of a full sort
    (score descending, position ascending) on random, tied, all-equal and skewed rows.
"""
import numpy as np
import pytest

KEY_BINS, SUB_BINS = 2048, 1024
SEL_CAND, TIE_CAP = 4096, 256  # candidate list and pairwise-ranked tie bin of one row


def f32_bits(scores):
    """int64 scores -> bits of their fp32 rounding (numpy converts with round-to-nearest-even)."""
    return np.asarray(scores, dtype=np.int64).astype(np.float32).view(np.uint32).astype(np.int64)


def key_bin(scores):
    b = f32_bits(scores)
    em = (b >> 19) & 0xFFF
    f = np.where(em != 0, em - (126 << 4), 0)
    return np.where(b >> 31, KEY_BINS // 2 - 1 - f, KEY_BINS // 2 + f)


def sub_bin(scores):
    b = f32_bits(scores)
    sb = (b >> 9) & (SUB_BINS - 1)
    return np.where(b >> 31, SUB_BINS - 1 - sb, sb)


def select_model(scores, k):
    """Top-k positions (ascending) by the histogram placement rule: exact, or None where the kernel
    settles the row by radix select instead (more than 4096 keys at or above the cut bin, or more
    than 256 keys left in the second-level cut bin)."""
    n = len(scores)
    if n <= k:
        return list(range(n))
    kb, sb = key_bin(scores), sub_bin(scores)
    hist = np.bincount(kb, minlength=KEY_BINS)
    cum = np.cumsum(hist[::-1])
    bstar = KEY_BINS - 1 - int(np.searchsorted(cum, k))  # the bin where the count from the top reaches k
    above = int(hist[bstar + 1:].sum())
    if above + int(hist[bstar]) > SEL_CAND:
        return None
    sel = list(np.nonzero(kb > bstar)[0])
    inbin = np.nonzero(kb == bstar)[0]
    need = k - above
    shist = np.bincount(sb[inbin], minlength=SUB_BINS)
    if shist.sum() > need:
        scum = np.cumsum(shist[::-1])
        sstar = SUB_BINS - 1 - int(np.searchsorted(scum, need))
        above2 = int(shist[sstar + 1:].sum())
        sel += [i for i in inbin if sb[i] > sstar]
        ties = [i for i in inbin if sb[i] == sstar]
        if len(ties) > TIE_CAP:
            return None
        ties.sort(key=lambda i: (-int(scores[i]), i))
        sel += ties[:need - above2]
    else:
        sel += list(inbin)
    return sorted(int(i) for i in sel)


def brute(scores, k):
    order = sorted(range(len(scores)), key=lambda i: (-int(scores[i]), i))
    return sorted(order[:k])


def test_bins_are_monotone_at_rounding_boundaries():
    # every power of two and the values around it, both signs, and the fp32 rounding midpoints
    vals = [0]
    for e in range(0, 51):
        for d in (-3, -2, -1, 0, 1, 2, 3):
            vals += [(1 << e) + d, -((1 << e) + d)]
        if e >= 25:  # integers that fp32 cannot hold: just below, at and above a rounding midpoint
            step = 1 << (e - 24)
            for m in (3, 5, 7):
                mid = (1 << e) + m * step // 2
                vals += [mid - 1, mid, mid + 1, -(mid - 1), -mid, -(mid + 1)]
    v = np.unique(np.array([x for x in vals if abs(x) < (1 << 51)], dtype=np.int64))
    kb, sb = key_bin(v), sub_bin(v)
    assert np.all(np.diff(kb) >= 0)
    same = np.diff(kb) == 0
    assert np.all(np.diff(sb)[same] >= 0)
    assert kb.min() >= 0 and kb.max() < KEY_BINS and sb.min() >= 0 and sb.max() < SUB_BINS


def test_bins_are_monotone_on_random_scores():
    rng = np.random.default_rng(7)
    v = np.sort(np.concatenate([rng.integers(-(1 << 50), 1 << 50, 20000), rng.integers(-(1 << 20), 1 << 20, 20000)]))
    kb, sb = key_bin(v), sub_bin(v)
    assert np.all(np.diff(kb) >= 0)
    assert np.all(np.diff(sb)[np.diff(kb) == 0] >= 0)


@pytest.mark.parametrize("case", ["gauss", "ties", "all_equal_small", "skewed", "tiny", "large"])
def test_placement_rule_gives_the_exact_topk(case):
    rng = np.random.default_rng(len(case))
    n, k = 16000, 512
    if case == "gauss":
        s = np.rint(rng.normal(0, 16 * 2 ** 20, n)).astype(np.int64)
    elif case == "ties":  # 97 distinct scores repeated: ties decide at the cut
        s = np.rint(rng.normal(0, 2 ** 24, 97)).astype(np.int64)[rng.integers(0, 97, n)]
    elif case == "all_equal_small":  # one bin, one sub-bin: pairwise ranking decides by position
        n = 200
        s = np.full(n, 12345, np.int64)
        k = 64
    elif case == "skewed":  # a few huge keys, the rest tightly packed
        s = rng.integers(-1000, 1000, n).astype(np.int64)
        s[rng.integers(0, n, 40)] = 1 << 45
    elif case == "tiny":
        s = rng.integers(-3, 4, n).astype(np.int64)
    else:
        s = rng.integers(-(1 << 50), 1 << 50, n).astype(np.int64)
    got = select_model(s, k)
    if got is None:  # the kernel settles such a row by radix select; the case must be a tie storm
        assert case == "tiny"
        return
    assert got == brute(s, k)


def test_tie_storms_leave_the_histogram_path():
    # more equal keys in the cut than the pairwise ranking holds, or more candidates than the list
    assert select_model(np.full(300, 7, np.int64), 64) is None
    assert select_model(np.zeros(20000, np.int64), 512) is None
    # exactly the capacity still ranks pairwise
    s = np.full(TIE_CAP, -5, np.int64)
    s = np.concatenate([s, np.full(600, -(1 << 40), np.int64)])
    assert select_model(s, 100) == list(range(100))
