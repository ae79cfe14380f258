"""Pins of the oracle's codec (R1, R8, R9) against things other than itself.

* E2M1 values: the OCP MX table in tests/golden/e2m1_values.txt (format named in
  "Pushing KV Cache Compression to 890 Bytes per Token", sec. XI).
* E4M3 values and RNE conversion: torch's float8_e4m3fn (a library routine).
* Rounding: brute-force nearest-value search in exact rational arithmetic, ties to the
  even code.
* Range: 448 x 6 = 2688 (sec. XI).
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import golden, golden_rows

E2M1 = {int(c, 16): float(v) for c, v in golden_rows("e2m1_values.txt")}


def e4m3_table():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def nearest_code(y: Fraction, values: dict, finite_max):
    """Brute force: nearest representable magnitude, ties to the even code, saturating."""
    neg = y < 0
    a = abs(y)
    best = None
    for code, v in values.items():
        if v < 0 or (v == 0 and math.copysign(1.0, v) < 0) or math.isnan(v):
            continue
        d = abs(a - Fraction(v))
        key = (d, code & 1, code)
        if best is None or key < best[0]:
            best = (key, code)
    code = best[1]
    if a > Fraction(finite_max):
        code = max(c for c, v in values.items() if v == finite_max)
    return code, neg


def test_e2m1_decode_matches_table(orc):
    for code, v in E2M1.items():
        got = orc.e2m1_decode(code)
        assert got == v and math.copysign(1, got) == math.copysign(1, v)


def test_e4m3_decode_matches_torch(orc):
    ref = e4m3_table()
    for b in range(256):
        got = orc.e4m3_decode(b)
        if b in (0x7F, 0xFF):
            assert math.isnan(got) and math.isnan(ref[b])
        else:
            assert got == ref[b], b


def test_range_2688(orc):
    g = golden("byte_budget.txt")
    mx = max(abs(orc.e2m1_decode(c)) * orc.e4m3_decode(s) for c in range(16) for s in range(0x7F))
    assert mx == g["fp4_no_global_scale_max"] == g["e4m3_max"] * g["e2m1_max"]


def _e2m1_sweep():
    ys = set()
    vals = sorted({abs(v) for v in E2M1.values()})
    for a, b in zip(vals, vals[1:]):
        m = (a + b) / 2
        ys.update([m, np.nextafter(m, 0), np.nextafter(m, 10)])
    ys.update(vals)
    ys.update([5.0, 6.0, 6.5, 7.0, 100.0, 1e30, 1e-30, 0.0])
    rng = np.random.default_rng(0)
    ys.update(rng.uniform(0, 8, 2000).tolist())
    out = []
    for y in ys:
        out += [y, -y]
    return out


def test_e2m1_encode_brute_force(orc):
    for y in _e2m1_sweep():
        got = orc.e2m1_encode(y)
        code, neg = nearest_code(Fraction(y), E2M1, 6.0)
        want = code | (8 if (neg or (y == 0 and math.copysign(1, y) < 0)) else 0)
        assert got == want, (y, got, want)


def test_e2m1_signed_zero_and_saturation(orc):
    assert orc.e2m1_encode(-0.0) == 0x8
    assert orc.e2m1_encode(-0.2) == 0x8
    assert orc.e2m1_encode(0.2) == 0x0
    assert orc.e2m1_encode(7.0) == 0x7
    assert orc.e2m1_encode(-1e9) == 0xF


def _e4m3_sweep():
    tab = e4m3_table()
    pos = sorted({float(v) for v in tab[:0x7F]})
    ys = set(pos)
    for a, b in zip(pos, pos[1:]):
        m = (a + b) / 2
        ys.update([m, float(np.nextafter(np.float32(m), np.float32(0))), float(np.nextafter(np.float32(m), np.float32(1e9)))])
    rng = np.random.default_rng(1)
    ys.update(np.float32(rng.uniform(0, 464, 3000)).astype(float).tolist())
    ys.update(np.float32(np.exp(rng.uniform(-16, 6, 3000))).astype(float).tolist())
    out = []
    for y in ys:
        out += [y, -y]
    return out


def test_e4m3_encode_matches_torch_rne(orc):
    ys = [y for y in _e4m3_sweep() if abs(y) <= 464.0]
    ref = torch.tensor(ys, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_encode(y) for y in ys], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(ys[i], got[i], ref[i]) for i in bad[:5]]


def test_e4m3_encode_brute_force_and_saturation(orc):
    tab = {c: float(v) for c, v in enumerate(e4m3_table())}
    for y in _e4m3_sweep()[::7] + [464.0, 465.0, 1e6, -1e6]:
        code, neg = nearest_code(Fraction(y), tab, 448.0)
        want = code | (0x80 if neg else 0)
        assert orc.e4m3_encode(y) == want, y
    assert orc.e4m3_encode(1e30) == 0x7E and orc.e4m3_encode(-1e30) == 0xFE


def _bf16(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


def independent_quantize(xb: torch.Tensor):
    """R1 by another route: the scale through torch's fp32 -> e4m3 RNE conversion of
    fp32(amax)/6, the codes by exact rational nearest search."""
    x = xb.float().reshape(-1, 16)
    amax = x.abs().amax(dim=1)
    sc = (amax / 6.0).to(torch.float8_e4m3fn)
    s = sc.double()
    codes = []
    for r in range(x.shape[0]):
        row = []
        for i in range(16):
            if s[r] == 0:
                row.append(0)
                continue
            y = Fraction(float(x[r, i])) / Fraction(float(s[r]))
            c, neg = nearest_code(y, E2M1, 6.0)
            neg = neg or (float(x[r, i]) == 0 and math.copysign(1, float(x[r, i])) < 0)
            row.append(c | (8 if neg else 0))
        codes.append(row)
    codes = np.array(codes, np.uint8)
    data = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return data, sc.view(torch.uint8).numpy()


@pytest.mark.parametrize("sigma", [1.0, 8.0, 1e-3, 3e-5])
def test_quantize_rows_independent_route(orc, sigma):
    g = torch.Generator().manual_seed(7)
    x = (torch.randn(64, 16, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    x[3, 5] = -0.0
    x[4] = 0.0
    x[5] = -0.0
    data, scale = orc.quantize_rows(x, 16)
    d2, s2 = independent_quantize(x)
    assert np.array_equal(scale.reshape(-1), s2)
    assert np.array_equal(data.reshape(-1, 8), d2)


def test_quantize_error_bound_and_roundtrip(orc):
    g = torch.Generator().manual_seed(3)
    x = torch.randn(256, 256, generator=g).mul(2.0).clamp(-26, 26).to(torch.bfloat16)
    data, scale = orc.quantize_rows(x, 256)
    deq = orc.dequant_rows(data, scale, 256)
    xf = x.double().numpy().reshape(256, 16, 16)
    s = np.array([[orc.e4m3_decode(int(b)) for b in r] for r in scale])
    amax = np.abs(xf).max(axis=2)
    bound = np.maximum(s, amax - 6 * s)[:, :, None]
    assert np.all(np.abs(xf - deq.reshape(256, 16, 16)) <= bound + 1e-12)
    # quantise o dequant is the identity on a block that already is s * E2M1 with a +-6 code
    vals = np.array([6, -4, 3, 2, 1.5, -1, 0.5, 0, 6, -6, 0.5, 1, 2, 3, 4, -0.5])
    for s_code in (0x38, 0x30, 0x41, 0x09, 0x66):
        sv = orc.e4m3_decode(s_code)
        xb = _bf16((vals * sv).tolist())
        d, sc = orc.quantize_rows(xb, 16)
        assert sc[0, 0] == s_code
        assert np.array_equal(orc.dequant_rows(d, sc, 16)[0], xb.double().numpy())


def test_packing_order(orc):
    """R9: channel 2j -> low nibble of byte j, 2j+1 -> high nibble; scale byte b <-> block b."""
    for c in (0, 1, 14, 15, 16, 33, 255):
        x = torch.zeros(256)
        x[c] = 6.0
        data, scale = orc.quantize_rows(x.to(torch.bfloat16), 256)
        nz = np.nonzero(data[0])[0]
        assert nz.tolist() == [c // 2]
        assert data[0, c // 2] == (0x7 << (4 * (c % 2)))
        assert np.nonzero(scale[0])[0].tolist() == [c // 16]
        assert scale[0, c // 16] == 0x38  # 6 / 6 = 1.0


def test_all_zero_and_tiny_blocks(orc):
    x = torch.zeros(2, 16)
    x[1] = 1e-30
    data, scale = orc.quantize_rows(x.to(torch.bfloat16), 16)
    assert not data.any() and not scale.any()


def test_fp8_rows_match_torch(orc):
    g = torch.Generator().manual_seed(11)
    x = torch.randn(4096, generator=g).mul(8).clamp(-26, 26).to(torch.bfloat16)
    got = orc.fp8_rows(x)
    ref = x.float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_exact_products_in_bf16_and_fp16(orc):
    """Every E2M1 x E4M3 product is exact in bf16 and in fp16 (dequantisation loses nothing)."""
    prods = np.array([orc.e2m1_decode(c) * orc.e4m3_decode(s) for c in range(8) for s in range(0x7F)])
    for dt in (torch.bfloat16, torch.float16):
        t = torch.tensor(prods, dtype=torch.float64)
        assert torch.equal(t.to(dt).double(), t)
