"""The latent attention kernel's arithmetic (latent.cu), modelled on the host in numpy and checked
against the oracle's fp64 LatentCache.attend.

Modelled: q rounded bf16 -> fp16; the dequantised latent exact in fp16; logits accumulated in fp32;
tiles of 128 keys (the selected entries, then the window); per head a running maximum m that moves
only when a tile's maximum exceeds it by more than 8 (log2 units), the accumulated output and sum
then rescaled by 2^(m_old - m_new); P = 2^(logit - m) rounded to fp16 for the output, unrounded for
the sum; out = O / l; lse = m ln 2 + ln l.

Checked: on workload-shaped inputs the model stays within a tenth (σ = 1) and a quarter (σ = 8) of
the GPU tests' tolerances; on rows whose maxima jump by more than the threshold at every tile (the rescale
path) and rows whose maxima creep up below it (probabilities up to 2^8), the error is no larger
than with a maximum kept exact at every tile; and without the rescale the error would be large,
so the rescale is what keeps the deferred maximum exact.
"""
import numpy as np
import pytest
import torch

import workloads as W

LN2 = 0.6931471805599453


def model_attend(q16, L, nsel, scale, lazy=8.0, rescale=True):
    """q16 [H, D] fp16 values (as float64), L [n, D] exact dequantised keys = values, the first nsel
    of them selected entries and the rest window rows; returns (out [H, D], lse [H])."""
    H, D = q16.shape
    s2 = np.float32(scale * 1.4426950408889634)
    tiles = [(a, min(nsel, a + 128)) for a in range(0, nsel, 128)] + ([(nsel, L.shape[0])] if L.shape[0] > nsel else [])
    m = np.full(H, -np.inf, np.float32)
    l = np.zeros(H, np.float32)
    O = np.zeros((H, D), np.float32)
    for a, b in tiles:
        S = (q16.astype(np.float32) @ L[a:b].astype(np.float32).T).astype(np.float32)  # fp32 logits [H, keys]
        tmax = (S * s2).max(axis=1)
        move = tmax > m + np.float32(lazy)
        al = np.where(move & np.isfinite(m), np.exp2(np.minimum(m - tmax, 0)).astype(np.float32), np.float32(1.0))
        al = np.where(move & ~np.isfinite(m), np.float32(0.0), al)
        m = np.where(move, tmax, m).astype(np.float32)
        if rescale:
            O *= al[:, None]
            l *= al
        p = np.exp2((S * s2 - m[:, None]).astype(np.float32)).astype(np.float32)
        l += p.sum(axis=1, dtype=np.float32)
        O += (p.astype(np.float16).astype(np.float32) @ L[a:b].astype(np.float32)).astype(np.float32)
    out = O / l[:, None]
    return out.astype(np.float64), (m.astype(np.float64) * LN2 + np.log(l.astype(np.float64)))


def _case(orc, seed, sigma, n=700, k=512):
    b = torch.tensor([0])
    lat = W.cache_values(seed, "lat", b, torch.arange(n), 512, sigma)[0]
    sw = W.cache_values(seed, "lsw", b, torch.arange(n), 512, sigma)[0]
    q = W.cache_values(seed, "lq", b, torch.tensor([[n - 1]]), 64 * 512, sigma)[0, 0].reshape(64, 512)
    oc = orc.LatentCache(1024, 128)
    oc.append(0, latent=lat, swa=sw)
    idx = W.distinct_sorted(seed, "sel", b, n - 1, k)[0].numpy().astype(np.int32)
    ro, rl = oc.attend(n - 1, q, idx)
    d = orc.dequant_rows(oc.ldata[idx], oc.lscale[idx], 512)
    win = np.stack([[orc.e4m3_decode(x) for x in oc.swa[p & 127]] for p in range(n - 128, n)])
    L = np.concatenate([d, win])
    q16 = q.float().numpy().astype(np.float16).astype(np.float64)
    return q16, L, k, ro, rl


@pytest.mark.parametrize("sigma,tol,margin", [(1.0, 2e-3, 10), (8.0, 1.6e-2, 4)])
def test_model_within_the_gpu_tolerance_with_margin(orc, sigma, tol, margin):
    """σ = 1: within a tenth of the 2e-3 tolerance. σ = 8: values reach |V| ~ 48, so the fp16
    rounding of P (relative 2^-12) allows ~1e-2 in the worst case; the model stays within a
    quarter of the 1.6e-2 tolerance."""
    q16, L, k, ro, rl = _case(orc, 41, sigma)
    out, lse = model_attend(q16, L, k, 1.0 / np.sqrt(512.0))
    assert np.abs(out - ro).max() <= tol / margin
    assert np.abs(lse - rl).max() <= tol / margin


def test_deferred_maximum_costs_no_accuracy(orc):
    """Rows whose logits grow by about 9.8 c (log2) per tile for head c-scales in [-1, 1.4]: the
    deferred maximum (threshold 8) is as accurate as the exact one (threshold 0), and dropping the
    rescale would be far off."""
    rng = np.random.default_rng(9)
    n, k = 640, 512
    v = rng.standard_normal(512)
    g = 0.3 * (np.arange(n) // 128)
    rows = (g[:, None] * v[None, :] + 0.25 * rng.standard_normal((n, 512)))
    L = rows.astype(np.float16).astype(np.float64)  # exact in fp16, as the kernel's tiles are
    c = np.linspace(-1.0, 1.4, 64)
    q16 = (c[:, None] * v[None, :]).astype(np.float16).astype(np.float64)
    scale = 1.0 / np.sqrt(512.0)
    logits = (q16 @ L.T) * scale
    mx = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - mx)
    ref = (w @ L) / w.sum(axis=1, keepdims=True)
    ref_lse = mx[:, 0] + np.log(w.sum(axis=1))
    lazy, lazy_lse = model_attend(q16, L, k, scale, lazy=8.0)
    exact, _ = model_attend(q16, L, k, scale, lazy=0.0)
    e_lazy, e_exact = np.abs(lazy - ref).max(), np.abs(exact - ref).max()
    assert e_lazy <= max(2.0 * e_exact, 1e-4) and e_lazy <= 4e-3
    assert np.abs(lazy_lse - ref_lse).max() <= 1e-3
    broken, _ = model_attend(q16, L, k, scale, lazy=8.0, rescale=False)
    assert np.abs(broken - ref).max() > 0.1
