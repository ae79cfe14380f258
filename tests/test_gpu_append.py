"""Quantise-append on the GPU against the oracle, bit for bit.

The element and scale rounding are swept exhaustively: every finite positive bf16 value as a
block maximum (scale rounding), every bf16 value in [-6s, 6s] for every non-zero E4M3 scale s
(element rounding, ties and signed zeros included), and every finite bf16 value for the FP8
window codec.
"""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_append_b200 as csa
import oracle
from _gpu import DEV, bf16_np, gpu_fill, oracle_seq, values

pytestmark = pytest.mark.gpu


def _append_rows(rows_bf16: torch.Tensor):
    """Quantise rows of 256 channels through both planes of a 1-sequence cache."""
    t = rows_bf16.shape[0]
    shape = csa.make_shape()
    cache = csa.Cache(1, t, swa_cap=1 << max(7, (t - 1).bit_length()))
    pos = torch.zeros(1, dtype=torch.int64, device=DEV)
    x = rows_bf16.to(DEV).contiguous()
    ws = csa.Workspace(shape, 1, 1, 512, 8)
    csa.csa2_quantize_append(shape, cache, 1, t, pos, x, x, x, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    return cache


def _all_finite_bf16():
    b = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    return b[torch.isfinite(b.float())]


def test_scale_rounding_exhaustive(orc):
    v = _all_finite_bf16()
    v = v[v.float() > 0]
    n = v.numel()
    blocks = torch.zeros(n, 16, dtype=torch.bfloat16)
    blocks[:, 0] = v
    blocks[:, 7] = -v.float().mul(0.5).to(torch.bfloat16)
    rows = torch.cat([blocks.reshape(-1), torch.zeros((-blocks.numel()) % 256, dtype=torch.bfloat16)]).reshape(-1, 256)
    cache = _append_rows(rows)
    d, s = orc.quantize_rows(bf16_np(rows), 256)
    assert np.array_equal(cache.kv_scale[0].cpu().numpy(), s)
    assert np.array_equal(cache.kv_data[0].cpu().numpy(), d)
    assert np.array_equal(cache.ik_scale[0].cpu().numpy(), s)
    assert np.array_equal(cache.ik_data[0].cpu().numpy(), d)


def test_element_rounding_exhaustive(orc):
    allv = _all_finite_bf16()
    allf = allv.float()
    blocks = []
    for sc in range(1, 0x7F):
        s = orc.e4m3_decode(sc)
        amax = torch.tensor([6.0 * s], dtype=torch.float32).to(torch.bfloat16)
        assert float(amax) == 6.0 * s
        el = allv[allf.abs() <= 6.0 * s]
        el = torch.cat([el, torch.zeros((-el.numel()) % 15, dtype=torch.bfloat16)]).reshape(-1, 15)
        blk = torch.cat([amax.expand(el.shape[0], 1), el], dim=1)
        blocks.append(blk)
    blocks = torch.cat(blocks)
    rows = torch.cat([blocks.reshape(-1), torch.zeros((-blocks.numel()) % 256, dtype=torch.bfloat16)]).reshape(-1, 256)
    cache = _append_rows(rows)
    d, s = orc.quantize_rows(bf16_np(rows), 256)
    got_d = cache.kv_data[0].cpu().numpy()
    bad = np.nonzero((got_d != d).any(axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:3]}"
    assert np.array_equal(cache.kv_scale[0].cpu().numpy(), s)


def test_window_fp8_exhaustive(orc):
    v = _all_finite_bf16()
    rows = torch.cat([v, torch.zeros((-v.numel()) % 256, dtype=torch.bfloat16)]).reshape(-1, 256)
    cache = _append_rows(rows)
    ref = orc.fp8_rows(bf16_np(rows))
    n = rows.shape[0]
    assert np.array_equal(cache.swa[0, :n].cpu().numpy(), ref)


@pytest.mark.parametrize("sigma", [1.0, 8.0])
def test_append_ragged_positions_and_ring(orc, sigma):
    """Several sequences appended at different positions; the window ring wraps."""
    B, cap, swa_cap, t = 3, 700, 128, 37
    shape = csa.make_shape()
    cache = csa.Cache(B, cap, swa_cap)
    ws = csa.Workspace(shape, B, 1, 512, 8)
    starts = [0, 300, 663]
    pos = torch.tensor(starts, dtype=torch.int64, device=DEV)
    b = torch.arange(B, device=DEV)
    p = pos.unsqueeze(1) + torch.arange(t, device=DEV)
    kv = values(5, "kv", b, p, 256, DEV, sigma).contiguous()
    ik = values(5, "ik", b, p, 256, DEV, sigma).contiguous()
    sw = values(5, "swa", b, p, 256, DEV, sigma).contiguous()
    csa.csa2_quantize_append(shape, cache, B, t, pos, kv, ik, sw, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    for i in range(B):
        oc = oracle.SeqCache(cap, swa_cap)
        pp = torch.arange(starts[i], starts[i] + t)
        oc.append(starts[i], kv=values(5, "kv", [i], pp, 256, "cpu", sigma)[0],
                  idx_k=values(5, "ik", [i], pp, 256, "cpu", sigma)[0],
                  swa_kv=values(5, "swa", [i], pp, 256, "cpu", sigma)[0])
        for name in ("kv_data", "kv_scale", "ik_data", "ik_scale", "swa"):
            assert np.array_equal(getattr(cache, name)[i].cpu().numpy(), getattr(oc, name)), (i, name)


def test_append_past_capacity_sets_status_and_writes_nothing():
    shape = csa.make_shape()
    cache = csa.Cache(2, 64, 128)
    ws = csa.Workspace(shape, 2, 1, 512, 8)
    pos = torch.tensor([10, 60], dtype=torch.int64, device=DEV)
    x = values(1, "kv", torch.arange(2), torch.arange(8), 256, DEV).contiguous()
    csa.csa2_quantize_append(shape, cache, 2, 8, pos, x, x, None, ws=ws)
    assert csa.csa2_get_device_status(ws) == csa.CSA2_DEV_BAD_POS
    assert cache.kv_data[1].abs().sum() == 0 and cache.kv_data[0].abs().sum() > 0
    assert csa.csa2_get_device_status(ws) == 0  # cleared by the read


def test_full_cache_fill_matches_oracle():
    shape = csa.make_shape()
    cache = csa.Cache(2, 5000, 8192)
    gpu_fill(cache, shape, 9, 2, 5000, chunk=2048)
    torch.cuda.synchronize()
    oc = oracle_seq(9, 1, 5000, 5000, 8192)
    for name in ("kv_data", "kv_scale", "ik_data", "ik_scale"):
        assert np.array_equal(getattr(cache, name)[1].cpu().numpy(), getattr(oc, name))
    assert np.array_equal(cache.swa[1, :5000].cpu().numpy(), oc.swa[:5000])


def _mx_gpu(x_cpu, ch):
    rows = x_cpu.shape[0]
    data = torch.empty(rows, ch // 2, dtype=torch.uint8, device=DEV)
    scale = torch.empty(rows, ch // 32, dtype=torch.uint8, device=DEV)
    csa.csa2_mxfp4_quantize(x_cpu.to(DEV).contiguous(), data, scale)
    return data.cpu().numpy(), scale.cpu().numpy()


@pytest.mark.parametrize("ch,sigma", [(128, 1.0), (128, 8.0), (512, 1.0), (32, 1e-3), (128, 1e-38)])
def test_mxfp4_codec_matches_oracle(orc, ch, sigma):
    """The MXFP4 row codec of the pages' indexer key (E2M1 + E8M0 per 32 channels) against the
    oracle's R13 codec, byte for byte: unit, large (clipped), small and subnormal values."""
    rows = 2048
    x = values(21, "ik", [0], torch.arange(rows), ch, "cpu", sigma)[0]
    d, s = _mx_gpu(x, ch)
    rd, rs = oracle.mx_quantize_rows(bf16_np(x), ch)
    assert np.array_equal(s, rs)
    assert np.array_equal(d, rd)


def test_mxfp4_codec_every_value_at_many_scales(orc):
    """Every finite bf16 value of magnitude <= A, in blocks whose largest magnitude is A, for block
    maxima across the whole exponent range (subnormal and the largest included), so that every
    E8M0 byte the rule can give and every E2M1 rounding decision is taken on the GPU and in the
    oracle; plus all-zero and signed-zero blocks (byte 0, +0 codes)."""
    pats = np.arange(0x10000, dtype=np.uint32).astype(np.uint16)
    vals = pats.view(np.int16).astype(np.int32)
    finite = (pats & 0x7F80) != 0x7F80
    f32 = (pats.astype(np.uint32) << 16).view(np.float32)
    blocks = []
    for amax_bits in (0x0001, 0x0040, 0x0080, 0x00C0, 0x1234, 0x3F80, 0x3FC0, 0x40C0, 0x4B00, 0x7F7F):
        A = np.float32((np.uint32(amax_bits) << 16).view(np.float32))
        sel = pats[finite & (np.abs(f32) <= A)]
        n = (len(sel) + 30) // 31
        sel = np.resize(sel, n * 31)
        blk = np.concatenate([np.full((n, 1), amax_bits, np.uint16), sel.reshape(n, 31)], axis=1)
        blocks.append(blk)
    nb = sum(b.shape[0] for b in blocks)
    pad = (-(nb + 2)) % 4  # whole 128-channel rows
    blocks.append(np.full((pad + 1, 32), 0x0000, np.uint16))
    blocks.append(np.full((1, 32), 0x8000, np.uint16))
    x = np.concatenate(blocks, axis=0).reshape(-1, 128)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    d, s = _mx_gpu(xt, 128)
    rd, rs = oracle.mx_quantize_rows(x, 128)
    assert np.array_equal(s, rs)
    assert np.array_equal(d, rd)
    assert (s.reshape(-1)[-2:] == 0).all() and (d.reshape(-1, 16)[-2:] == 0).all()
