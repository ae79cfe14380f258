"""The decode score kernel's integer arithmetic, modelled on the host and checked against the oracle.

The score kernel never converts a code to floating point. Each E2M1 code c becomes the integer
2 * value(c) in {0, +-1, +-2, +-3, +-4, +-6, +-8, +-12}. The magnitudes come from a byte permute of
the table {0, 1, 2, 3, 4, 6, 8, 12} whose sign-replicate mode returns 0 for codes with the sign bit
set, so one permute gives the positive channels and one permute of the sign-flipped codes gives the
negative ones. A 16-channel block's dot product is D = sum (2q)(2k), |D| <= 2304. An E4M3 scale
s = M * 2^(E - 10) enters as the integer f(s) = M * 2^(E - 1) = s * 2^9, and the int64 sum of
D * f(s_k) * f(s_q) over the blocks is S = score * 2^20 exactly. These tests model that arithmetic in
numpy integers and check that:
  * S equals the oracle's exact fp64 score times 2^20, on random, large-sigma and extreme inputs;
  * f(s) = s * 2^9 for every finite E4M3 scale (normal and subnormal);
  * the bounds that make the int32 and int64 steps safe hold at the largest inputs the format
    allows: |D| <= 2304, |D * f_k| < 2^31, each block term < 2^47, |S| < 2^51.
"""
import numpy as np
import pytest
import torch

TAB = np.array([0, 1, 2, 3, 4, 6, 8, 12], np.int64)  # 2 * E2M1 magnitude of codes 0..7


def twice_values(codes):
    """2 * value of E2M1 codes, as the kernel forms it: positive and negative permutes."""
    c = codes.astype(np.int64)
    pos = np.where(c < 8, TAB[c & 7], 0)          # sign-replicate: sign-bit codes give 0
    neg = np.where(c >= 8, TAB[(c ^ 8) & 7], 0)   # the same permute of the sign-flipped codes
    return pos - neg


def fixed_scale(byte):
    """f(s) = M * 2^(E - 1) for the E4M3 scale byte (sign bit 0): normal M = 8 + m, subnormal E = 1, M = m."""
    b = np.asarray(byte, np.int64)
    e, m = (b >> 3) & 15, b & 7
    M = np.where(e == 0, m, 8 + m)
    E = np.where(e == 0, 1, e)
    return M << (E - 1)


def unpack(data):
    d = data.astype(np.int64)
    return np.stack([d & 15, d >> 4], axis=-1).reshape(d.shape[0], -1)


def model_scores(qd, qs, kd, ks, hk=4, hi=4):
    """S[p] = sum over heads h and blocks b of D(h, b, p) * f(k scale) * f(q scale), in int64."""
    q2 = twice_values(unpack(qd))                  # [hi, 64]
    k2 = twice_values(unpack(kd)).reshape(-1, hk, 64)
    fq = fixed_scale(qs)                           # [hi, 4]
    fk = fixed_scale(ks).reshape(-1, hk, 4)
    S = np.zeros(k2.shape[0], np.int64)
    stats = {"D": 0, "Dfk": 0, "term": 0}
    for h in range(hi):
        g = h * hk // hi
        for b in range(4):
            D = (k2[:, g, 16 * b:16 * b + 16] * q2[h, 16 * b:16 * b + 16]).sum(axis=1)
            dfk = D * fk[:, g, b]
            term = dfk * fq[h, b]
            stats["D"] = max(stats["D"], int(np.abs(D).max()))
            stats["Dfk"] = max(stats["Dfk"], int(np.abs(dfk).max()))
            stats["term"] = max(stats["term"], int(np.abs(term).max()))
            S += term
    return S, stats


def test_fixed_scale_is_s_times_2_pow_9(orc):
    for b in range(0x7F):  # every finite non-negative E4M3 byte (0x7F is NaN)
        assert fixed_scale(b) == orc.e4m3_decode(b) * 2 ** 9, hex(b)
    assert fixed_scale(0x7E) == 229376  # the largest finite scale, 448 = 14 * 2^5, times 2^9


def test_twice_values_table(orc):
    for c in range(16):
        assert twice_values(np.array([c]))[0] == 2 * orc.e2m1_decode(c)


@pytest.mark.parametrize("sigma,seed", [(1.0, 1), (8.0, 2), (1e-3, 3)])
def test_integer_scores_equal_exact_scores(orc, sigma, seed):
    n = 256
    g = torch.Generator().manual_seed(seed)
    keys = (torch.randn(n, 256, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    q = (torch.randn(4, 64, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    c = orc.SeqCache(cap=n, swa_cap=128)
    c.append(0, idx_k=keys)
    ref = c.scores(q, np.arange(n))
    qd, qs = orc.quantize_rows(q, 64)
    S, st = model_scores(qd, qs, c.ik_data[:n], c.ik_scale[:n])
    assert np.array_equal(S, (np.asarray(ref) * 2.0 ** 20).astype(np.int64))
    assert np.array_equal(S.astype(np.float64) / 2 ** 20, np.asarray(ref))


def test_bounds_at_the_format_limits(orc):
    """Every code +-6 (2 * value = +-12) at the largest scale 448 in query and keys: the extremes."""
    n = 4
    six = torch.full((n, 256), 2688.0)  # 6 * 448: every block's scale is 448, every code 6
    six[1] = -2688.0
    six[2, ::2] = -2688.0
    qv = torch.full((4, 64), 2688.0)
    c = orc.SeqCache(cap=n, swa_cap=128)
    c.append(0, idx_k=six.to(torch.bfloat16))
    qd, qs = orc.quantize_rows(qv.to(torch.bfloat16), 64)
    assert (qs == 0x7E).all() and (c.ik_scale[:n] == 0x7E).all()
    S, st = model_scores(qd, qs, c.ik_data[:n], c.ik_scale[:n])
    assert st["D"] == 16 * 12 * 12 == 2304
    assert st["Dfk"] == 2304 * 229376 < 2 ** 31
    assert st["term"] == 2304 * 229376 * 229376 < 2 ** 47
    assert int(np.abs(S).max()) == 16 * st["term"] < 2 ** 51
    ref = c.scores(qv.to(torch.bfloat16), np.arange(n))
    assert np.array_equal(S.astype(np.float64) / 2 ** 20, np.asarray(ref))
    assert ref[0] == 4 * 64 * 2688.0 ** 2 and ref[1] == -ref[0] and ref[2] == 0.0
