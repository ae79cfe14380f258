"""Pins of the oracle's parts in the pages' own shapes (R13-R15; "Pushing KV Cache Compression to
890 Bytes per Token", sec. VII byte budget and the configuration list of its closing section):
the MXFP4 indexer key, the 32 x 128 MQA indexer and attention over the 512-channel latent.

* E8M0: every byte against 2.0 ** (byte - 127); 0xFF is NaN.
* MXFP4 codec: an independent route (the shared exponent from math.frexp, nearest E2M1 value
  by brute force in exact rationals, ties to the even code) for every block; error bounds;
  the identity on blocks that already are a power of two times E2M1 values with a 4 or a 6.
* Bytes: ch/2 + ch/32 (68 B for the 128-channel key) and the 890 B/token budget printed on the
  page: 2.5 entries per token x (288 B latent + 68 B indexer key) = 720 + 170.
* Indexer scores: exact rational arithmetic from codes decoded through the golden E2M1 table;
  the ReLU variant; a one-hot closed form; Top-k against a full sort.
* Latent attention: sparse == dense torch fp64 softmax with K = V = the decoded latent; a single
  key returns itself; order of the indices does not matter; the default scale is 1/sqrt(512).
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import golden_rows

E2M1 = {int(c, 16): float(v) for c, v in golden_rows("e2m1_values.txt")}


def bf16(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


def nearest_e2m1(y: Fraction):
    """Nearest E2M1 magnitude by brute force, ties to the even code, saturating at 6; sign kept."""
    a = abs(y)
    best = min((abs(a - Fraction(E2M1[c])), c & 1, c) for c in range(8))
    code = best[2] if a <= 6 else 7
    return code | (8 if (y < 0 or (y == 0 and math.copysign(1.0, float(y)) < 0)) else 0)


def mx_independent(x: torch.Tensor):
    """R13 written independently: rows [r, 32 * nb] -> (codes [r, 32 * nb], scale bytes [r, nb])."""
    xf = x.double().numpy()
    r, ch = xf.shape
    codes = np.zeros((r, ch), np.uint8)
    sb = np.zeros((r, ch // 32), np.uint8)
    for i in range(r):
        for b in range(ch // 32):
            blk = xf[i, 32 * b:32 * b + 32]
            amax = float(np.abs(blk).max())
            if amax == 0.0:
                continue
            m, e = math.frexp(amax)  # amax = m * 2^e, m in [0.5, 1): floor(log2 amax) = e - 1
            se = min(max(e - 1 - 2, -127), 127)
            sb[i, b] = se + 127
            for j, v in enumerate(blk):
                y = Fraction(v) / Fraction(2) ** se if se >= 0 else Fraction(v) * Fraction(2) ** (-se)
                code = nearest_e2m1(y)
                if v == 0.0 and math.copysign(1.0, v) < 0:
                    code |= 8
                codes[i, 32 * b + j] = code
    return codes, sb


def unpack(data):
    d = data.astype(np.int64)
    return np.stack([d & 15, d >> 4], axis=-1).reshape(d.shape[0], -1)


def test_e8m0_every_byte(orc):
    for b in range(255):
        assert orc.e8m0_decode(b) == 2.0 ** (b - 127)
    assert math.isnan(orc.e8m0_decode(255))


@pytest.mark.parametrize("sigma", [1.0, 8.0, 1e-3, 1e-30, 3e-39])
def test_mx_codec_independent_route(orc, sigma):
    """sigma 3e-39: block maxima below 2^-125, where the shared exponent is clamped at -127."""
    g = torch.Generator().manual_seed(int(sigma * 1000) % 97 + 1)
    x = (torch.randn(24, 128, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    x[2, 7] = -0.0
    x[3] = 0.0
    x[4, :32] = -0.0
    data, scale = orc.mx_quantize_rows(x, 128)
    codes, sb = mx_independent(x)
    assert np.array_equal(scale, sb)
    assert np.array_equal(unpack(data), codes)
    # packing: channel 2j in the low nibble of byte j
    assert np.array_equal(data, (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8))


def test_mx_error_bounds_and_identity(orc):
    g = torch.Generator().manual_seed(5)
    x = torch.randn(128, 128, generator=g).mul(3.0).clamp(-26, 26).to(torch.bfloat16)
    data, scale = orc.mx_quantize_rows(x, 128)
    deq = orc.mx_dequant_rows(data, scale, 128).reshape(128, 4, 32)
    xf = x.double().numpy().reshape(128, 4, 32)
    X = (2.0 ** (scale.astype(np.float64) - 127))[:, :, None]
    err = np.abs(xf - deq)
    # |x| / X < 8 always; up to 6 X the grid step is at most 2 X (error <= X), beyond it saturation
    assert np.all(np.abs(xf) < 8 * X)
    assert np.all(err[np.abs(xf) <= 6 * X] <= X.repeat(32, 2)[np.abs(xf) <= 6 * X])
    assert np.all(err <= 2 * X)
    # the identity on blocks that are 2^s times E2M1 values with a 4 or a 6 (their amax sets X = 2^s)
    vals = np.array([6, -4, 3, 2, 1.5, -1, 0.5, 0, 4, -6, 0.5, 1, 2, 3, 4, -0.5] * 2, dtype=np.float64)
    for s in (-9, -1, 0, 3, 20):
        xb = bf16((vals * 2.0 ** s).tolist()).reshape(1, 32)
        d, sc = orc.mx_quantize_rows(xb, 32)
        assert sc[0, 0] == s + 127
        assert np.array_equal(orc.mx_dequant_rows(d, sc, 32)[0], xb.double().numpy()[0])


def test_mx_zero_block(orc):
    x = torch.zeros(1, 64)
    x[0, 40] = 1.0
    data, scale = orc.mx_quantize_rows(x.to(torch.bfloat16), 64)
    assert scale[0, 0] == 0 and not data[0, :16].any()
    assert scale[0, 1] == 125  # amax 1 -> X = 2^-2
    code_of_4 = [c for c in range(8) if E2M1[c] == 4.0][0]
    assert unpack(data)[0, 40] == code_of_4  # 1 / 2^-2 = 4, an E2M1 value


def test_bytes_and_the_890_budget(orc):
    assert orc.mx_entry_bytes(128) == 68 and orc.mx_entry_bytes(32) == 17
    assert orc.mx_entry_bytes(48) == 0 and orc.mx_entry_bytes(0) == 0
    assert orc.entry_bytes(512) == 288
    # entries per token: 3 encoder caches at r = 2 plus 1 decoder cache at r = 1 = 2.5
    per_token = Fraction(3, 2) + 1
    main, idx = per_token * orc.entry_bytes(512), per_token * orc.mx_entry_bytes(128)
    assert (main, idx, main + idx) == (720, 170, 890)


def make_latent(orc, n, seed=0, sigma=1.0, swa_cap=256):
    g = torch.Generator().manual_seed(seed)
    c = orc.LatentCache(cap=n, swa_cap=swa_cap)
    lat = (torch.randn(n, 512, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    ik = (torch.randn(n, 128, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    sw = (torch.randn(n, 512, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    c.append(0, latent=lat, idx_k=ik, swa=sw)
    return c


def mx_decode_exact(data, scale):
    """Exact rationals of MXFP4 rows through the golden E2M1 table and 2^(byte - 127)."""
    codes = unpack(data)
    out = []
    for r in range(codes.shape[0]):
        out.append([Fraction(E2M1[int(c)]) * Fraction(2) ** (int(scale[r, j // 32]) - 127)
                    for j, c in enumerate(codes[r])])
    return out


@pytest.mark.parametrize("sigma,relu", [(1.0, False), (1.0, True), (8.0, False), (0.01, True)])
def test_indexer_scores_exact(orc, sigma, relu):
    n = 24
    c = make_latent(orc, n, seed=3, sigma=sigma)
    q = (torch.randn(32, 128, generator=torch.Generator().manual_seed(4)) * sigma).clamp(-26, 26).to(torch.bfloat16)
    idx, sc = c.index_topk_full(n - 1, q, k=8, relu=relu)
    qd, qs = orc.mx_quantize_rows(q, 128)
    qv = mx_decode_exact(qd, qs)
    kv = mx_decode_exact(c.kdata[:n], c.kscale[:n])
    for p in range(n):
        tot = Fraction(0)
        for h in range(32):
            dot = sum(a * b for a, b in zip(qv[h], kv[p]))
            tot += max(dot, Fraction(0)) if relu else dot
        assert Fraction(sc[p]) == tot, p
    ranked = sorted(range(n), key=lambda p: (-sc[p], p))[:8]
    assert idx.tolist() == sorted(ranked)


def test_indexer_one_hot_closed_form_and_causality(orc):
    n = 16
    c = make_latent(orc, n, seed=6)
    q = torch.zeros(32, 128)
    q[11, 70] = 3.0  # block amax 3 -> X = 2^-1, code value 6
    _, sc = c.index_topk_full(n - 1, q.to(torch.bfloat16), k=4)
    kv = orc.mx_dequant_rows(c.kdata, c.kscale, 128)
    assert np.array_equal(sc, 3.0 * kv[:, 70])
    idx, sc5 = c.index_topk_full(5, q.to(torch.bfloat16), k=16)
    assert sc5.size == 6 and idx.tolist() == list(range(6)) + [-1] * 10
    _, sc_r2 = c.index_topk_full(6, q.to(torch.bfloat16), k=4, ratio=2)
    assert sc_r2.size == 3  # tokens 0..6 complete entries 0, 1, 2 at ratio 2


def dense_latent(orc, c, q, rows, win_pos, scale):
    parts = []
    if len(rows):
        parts.append(torch.from_numpy(orc.dequant_rows(c.ldata[rows], c.lscale[rows], 512)))
    if len(win_pos):
        w = c.swa[[p & (c.swa_cap - 1) for p in win_pos]]
        parts.append(torch.from_numpy(np.ascontiguousarray(w)).view(torch.float8_e4m3fn).double())
    L = torch.cat(parts)
    lg = q.double() @ L.T * scale
    return (torch.softmax(lg, dim=-1) @ L).numpy(), torch.logsumexp(lg, dim=-1).numpy()


@pytest.mark.parametrize("sigma", [1.0, 0.25])
def test_latent_sparse_equals_dense(orc, sigma):
    n = 20
    c = make_latent(orc, n, seed=8, sigma=sigma)
    q = (torch.randn(64, 512, generator=torch.Generator().manual_seed(9)) * sigma).to(torch.bfloat16)
    idx = np.concatenate([np.arange(n), -np.ones(12)]).astype(np.int32)
    out, lse = c.attend(n - 1, q, idx, win=6)
    ref, rl = dense_latent(orc, c, q, list(range(n)), list(range(n - 6, n)), 1 / np.sqrt(512))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)
    out2, _ = c.attend(n - 1, q, np.random.default_rng(0).permutation(idx), win=6)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-12)


def test_latent_single_key_returns_it(orc):
    c = make_latent(orc, 8, seed=10)
    q = torch.randn(64, 512, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    out, lse = c.attend(7, q, np.array([3], np.int32), win=0)
    lat3 = orc.dequant_rows(c.ldata[3:4], c.lscale[3:4], 512)[0]
    assert np.array_equal(out, np.broadcast_to(lat3, (64, 512)))  # K = V: the one key comes back
    with pytest.raises(AssertionError):  # an entry the query cannot see yet
        c.attend(2, q, np.array([3], np.int32), win=0)
