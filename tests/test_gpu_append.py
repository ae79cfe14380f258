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
