"""Sparse attention and the four per-mode compositions on the GPU against the oracle.

Attention outputs (fp32) must be within 2e-3 at unit-variance inputs, scaled with sigma (the bound
of fp16 products of exact dequantised values with fp32 accumulation); the bf16 output must be the
round-to-nearest-even of the fp32 output; index outputs of the compositions must be identical to the oracle's.
"""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_append_b200 as csa
import workloads as W
from _gpu import DEV, attn_tol, gpu_fill, oracle_seq, query_values, values

pytestmark = pytest.mark.gpu


def _cache(B, n, seed, sigma=1.0, swa_cap=None):
    shape = csa.make_shape()
    swa_cap = swa_cap or (1 << max(7, (n - 1).bit_length()))
    cache = csa.Cache(B, n, swa_cap)
    gpu_fill(cache, shape, seed, B, n, sigma)
    return shape, cache, swa_cap


def _check_rows(out, out_f32, lse, refs, tol):
    assert torch.equal(out, out_f32.to(torch.bfloat16))
    for r, (ro, rl) in enumerate(refs):
        got = out_f32[r].double().cpu().numpy()
        err = np.abs(got - ro).max()
        assert err <= tol, (r, err)
        gl = lse[r].double().cpu().numpy()
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(gl), fin)
        if fin.any():
            assert np.abs(gl[fin] - rl[fin]).max() <= tol


@pytest.mark.parametrize("B,n,k,sigma,swa_begin", [
    (3, 300, 64, 1.0, None),
    (4, 100, 64, 1.0, None),  # 50 selected keys: a tile mixes FP4 rows and FP8 window rows
    (2, 5000, 512, 1.0, [4900, 0]),
    (300, 700, 512, 1.0, None),
    (2, 3000, 512, 8.0, None),
    (1, 2100, 2048, 1.0, None),
])
def test_sparse_attend_matches_oracle(orc, B, n, k, sigma, swa_begin):
    seed = 31 + n + B
    shape, cache, swa_cap = _cache(B, n, seed, sigma)
    qpos = [n - 1 - (i % 7) * 3 for i in range(B)]
    qp = torch.tensor(qpos, dtype=torch.int64, device=DEV)
    q = query_values(seed, "q", torch.arange(B), qp, 2048, DEV, sigma).reshape(B, 16, 128).contiguous()
    nsel = min(k, n // 2)
    idx = W.distinct_sorted(seed, "sel", torch.arange(B, device=DEV), n - 30, nsel).to(torch.int32)
    idx = torch.cat([idx, torch.full((B, k - nsel), -1, dtype=torch.int32, device=DEV)], 1)
    perm = torch.argsort(torch.rand(B, k, generator=torch.Generator().manual_seed(seed)), dim=1).to(DEV)
    idx = torch.gather(idx, 1, perm).contiguous()  # any order, -1 anywhere
    sb = None if swa_begin is None else torch.tensor(swa_begin, dtype=torch.int64, device=DEV)
    out = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=DEV)
    of = torch.empty(B, 16, 128, dtype=torch.float32, device=DEV)
    lse = torch.empty(B, 16, dtype=torch.float32, device=DEV)
    ws = csa.Workspace(csa.make_shape(), B, 1, k, 8)
    csa.csa2_sparse_attend(shape, cache, B, 1, qp, q, idx, k, out, swa_begin=sb, out_f32=of, lse=lse, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    check = range(B) if B <= 4 else [0, 1, B // 2, B - 1]
    refs = []
    for b in check:
        oc = oracle_seq(seed, b, n, n, swa_cap, sigma)
        qb = query_values(seed, "q", [b], [qpos[b]], 2048, "cpu", sigma)[0]
        refs.append(oc.sparse_attend(qpos[b], qb, idx[b].cpu().numpy(), swa_begin=0 if sb is None else swa_begin[b]))
    rows = list(check)
    _check_rows(out[rows], of[rows], lse[rows], refs, attn_tol(None, sigma))


def test_bad_index_and_empty_row(orc):
    B, n, k = 2, 400, 16
    shape, cache, swa_cap = _cache(B, n, 7)
    qp = torch.tensor([200, 399], dtype=torch.int64, device=DEV)
    q = query_values(7, "q", torch.arange(B), qp, 2048, DEV).reshape(B, 16, 128).contiguous()
    idx = torch.full((B, k), -1, dtype=torch.int32, device=DEV)
    idx[0, :5] = torch.tensor([3, 250, 17, -5, 100])  # 250 > qpos, -5 invalid
    sb = torch.tensor([0, 1000], dtype=torch.int64, device=DEV)  # row 1: window empty, no selection
    out = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=DEV)
    of = torch.empty(B, 16, 128, dtype=torch.float32, device=DEV)
    lse = torch.empty(B, 16, dtype=torch.float32, device=DEV)
    ws = csa.Workspace(shape, B, 1, k, 8)
    csa.csa2_sparse_attend(shape, cache, B, 1, qp, q, idx, k, out, swa_begin=sb, out_f32=of, lse=lse, ws=ws)
    assert csa.csa2_get_device_status(ws) == csa.CSA2_DEV_BAD_INDEX
    oc = oracle_seq(7, 0, n, n, swa_cap)
    ro, rl = oc.sparse_attend(200, query_values(7, "q", [0], [200], 2048, "cpu")[0], np.array([3, 17, 100], np.int32))
    _check_rows(out[:1], of[:1], lse[:1], [(ro, rl)], 2e-3)
    assert torch.all(of[1] == 0) and torch.all(torch.isneginf(lse[1]))


def test_decode_modes_match_oracle(orc):
    """decode_full (with pool), decode_reindex on that pool, decode_minimal on inherited indices."""
    B, n, k, P = 2, 6000, 512, 128
    seed = 41
    shape = csa.make_shape()
    swa_cap = 8192
    cache = csa.Cache(B, n, swa_cap)
    gpu_fill(cache, shape, seed, B, n - 1)  # positions 0..n-2; the step appends n-1
    b = torch.arange(B, device=DEV)
    qp = torch.full((B,), n - 1, dtype=torch.int64, device=DEV)
    kv = values(seed, "kv", b, qp.unsqueeze(1), 256, DEV)[:, 0].contiguous()
    ik = values(seed, "ik", b, qp.unsqueeze(1), 256, DEV)[:, 0].contiguous()
    sw = values(seed, "swa", b, qp.unsqueeze(1), 256, DEV)[:, 0].contiguous()
    iq = query_values(seed, "iq", b, qp, 256, DEV).contiguous()
    q = query_values(seed, "q", b, qp, 2048, DEV).reshape(B, 16, 128).contiguous()
    out_idx = torch.empty(B, k, dtype=torch.int32, device=DEV)
    pool = torch.empty(B, P, dtype=torch.int32, device=DEV)
    pool_n = torch.empty(B, dtype=torch.int32, device=DEV)
    out = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=DEV)
    of = torch.empty(B, 16, 128, dtype=torch.float32, device=DEV)
    lse = torch.empty(B, 16, dtype=torch.float32, device=DEV)
    ws = csa.Workspace(shape, B, 1, k, n, P)
    csa.csa2_decode_full(shape, cache, B, qp, kv, ik, sw, iq, q, k, out_idx, out, pool_blocks=P, out_pool=pool,
                         out_pool_n=pool_n, max_ctx=n, out_f32=of, lse=lse, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    # Reindex layer: its own indexer query and query, same pool
    iq2 = query_values(seed + 1, "iq", b, qp, 256, DEV).contiguous()
    q2 = query_values(seed + 1, "q", b, qp, 2048, DEV).reshape(B, 16, 128).contiguous()
    sw2 = values(seed + 1, "swa", b, qp.unsqueeze(1), 256, DEV)[:, 0].contiguous()
    idx2 = torch.empty(B, k, dtype=torch.int32, device=DEV)
    out2 = torch.empty_like(out)
    of2 = torch.empty_like(of)
    lse2 = torch.empty_like(lse)
    csa.csa2_decode_reindex(shape, cache, B, qp, sw2, iq2, q2, pool, pool_n, k, idx2, out2, out_f32=of2, lse=lse2, ws=ws)
    # Minimal layer: inherits idx2, own query and window entry
    q3 = query_values(seed + 2, "q", b, qp, 2048, DEV).reshape(B, 16, 128).contiguous()
    sw3 = values(seed + 2, "swa", b, qp.unsqueeze(1), 256, DEV)[:, 0].contiguous()
    out3 = torch.empty_like(out)
    of3 = torch.empty_like(of)
    lse3 = torch.empty_like(lse)
    csa.csa2_decode_minimal(shape, cache, B, qp, sw3, q3, idx2, k, out3, out_f32=of3, lse=lse3, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    for bb in range(B):
        oc = oracle_seq(seed, bb, n, n, swa_cap)
        ridx, rpool, rpn = oc.index_topk_full(n - 1, query_values(seed, "iq", [bb], [n - 1], 256, "cpu")[0], k=k,
                                              pool_blocks=P)
        assert np.array_equal(out_idx[bb].cpu().numpy(), ridx)
        assert np.array_equal(pool[bb].cpu().numpy(), rpool) and int(pool_n[bb]) == rpn
        r1 = oc.sparse_attend(n - 1, query_values(seed, "q", [bb], [n - 1], 2048, "cpu")[0], ridx)
        _check_rows(out[bb:bb + 1], of[bb:bb + 1], lse[bb:bb + 1], [r1], 2e-3)
        # the Reindex layer writes its own window entry at n-1 (the oracle ring too)
        oc.append(n - 1, swa_kv=values(seed + 1, "swa", [bb], [n - 1], 256, "cpu")[0])
        ridx2 = oc.index_topk_reindex(n - 1, query_values(seed + 1, "iq", [bb], [n - 1], 256, "cpu")[0], rpool, rpn, k=k)
        assert np.array_equal(idx2[bb].cpu().numpy(), ridx2)
        r2 = oc.sparse_attend(n - 1, query_values(seed + 1, "q", [bb], [n - 1], 2048, "cpu")[0], ridx2)
        _check_rows(out2[bb:bb + 1], of2[bb:bb + 1], lse2[bb:bb + 1], [r2], 2e-3)
        oc.append(n - 1, swa_kv=values(seed + 2, "swa", [bb], [n - 1], 256, "cpu")[0])
        r3 = oc.sparse_attend(n - 1, query_values(seed + 2, "q", [bb], [n - 1], 2048, "cpu")[0], ridx2)
        _check_rows(out3[bb:bb + 1], of3[bb:bb + 1], lse3[bb:bb + 1], [r3], 2e-3)


@pytest.mark.parametrize("p0,t", [(3000, 64), (0, 200)])
def test_prefill_chunk_matches_oracle(orc, p0, t):
    seed, k = 51, 512
    cap = p0 + t
    shape = csa.make_shape()
    swa_cap = 1 << (t + 128 - 1).bit_length()
    cache = csa.Cache(1, cap, swa_cap)
    if p0:
        gpu_fill(cache, shape, seed, 1, p0)
    p = torch.arange(p0, p0 + t, device=DEV)
    kv = values(seed, "kv", [0], p, 256, DEV)[0].contiguous()
    ik = values(seed, "ik", [0], p, 256, DEV)[0].contiguous()
    sw = values(seed, "swa", [0], p, 256, DEV)[0].contiguous()
    iq = values(seed, "iq", [0], p, 256, DEV)[0].contiguous()
    q = values(seed, "q", [0], p, 2048, DEV)[0].reshape(t, 16, 128).contiguous()
    out_idx = torch.empty(t, k, dtype=torch.int32, device=DEV)
    out = torch.empty(t, 16, 128, dtype=torch.bfloat16, device=DEV)
    of = torch.empty(t, 16, 128, dtype=torch.float32, device=DEV)
    lse = torch.empty(t, 16, dtype=torch.float32, device=DEV)
    ws = csa.Workspace(shape, 1, t, k, cap)
    csa.csa2_prefill_chunk(shape, cache, p0, t, kv, ik, sw, iq, q, k, out_idx, out, out_f32=of, lse=lse, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    oc = oracle_seq(seed, 0, cap, cap, swa_cap)
    iqc = values(seed, "iq", [0], p.cpu(), 256, "cpu")[0]
    qc = values(seed, "q", [0], p.cpu(), 2048, "cpu")[0]
    rows = list(range(0, t, max(1, t // 16))) + [t - 1]
    refs = []
    for r in rows:
        ridx = oc.index_topk_full(p0 + r, iqc[r], k=k)
        assert np.array_equal(out_idx[r].cpu().numpy(), ridx), r
        refs.append(oc.sparse_attend(p0 + r, qc[r], ridx))
    _check_rows(out[rows], of[rows], lse[rows], refs, 2e-3)


def test_ratio_two_attention(orc):
    """Compression ratio 2: a query at token i may use entries 0 .. floor((i + 1) / 2) - 1; the window
    stays per token. Entry floor((i + 1) / 2) is not visible yet: flagged and skipped."""
    B, n, k = 2, 3000, 256
    seed = 57
    _, cache, swa_cap = _cache(B, n, seed)
    shape = csa.make_shape(ratio=2)
    qpos = [2999, 2500]  # visible entries 1500 and 1250
    qp = torch.tensor(qpos, dtype=torch.int64, device=DEV)
    q = query_values(seed, "q", torch.arange(B), qp, 2048, DEV).reshape(B, 16, 128).contiguous()
    vis = [(p + 1) // 2 for p in qpos]
    idx = torch.stack([W.distinct_sorted(seed, "sel", torch.tensor([b], device=DEV), vis[b], k)[0]
                       for b in range(B)]).to(torch.int32).contiguous()
    out = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=DEV)
    of = torch.empty(B, 16, 128, dtype=torch.float32, device=DEV)
    lse = torch.empty(B, 16, dtype=torch.float32, device=DEV)
    ws = csa.Workspace(shape, B, 1, k, 8)
    csa.csa2_sparse_attend(shape, cache, B, 1, qp, q, idx, k, out, out_f32=of, lse=lse, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    refs = []
    for b in range(B):
        oc = oracle_seq(seed, b, n, n, swa_cap)
        qb = query_values(seed, "q", [b], [qpos[b]], 2048, "cpu")[0]
        refs.append(oc.sparse_attend(qpos[b], qb, idx[b].cpu().numpy(), ratio=2))
    _check_rows(out, of, lse, refs, attn_tol(None, 1.0))
    # the first entry that is not visible yet
    idx2 = idx.clone()
    idx2[:, 0] = torch.tensor(vis, dtype=torch.int32, device=DEV)
    csa.csa2_sparse_attend(shape, cache, B, 1, qp, q, idx2, k, out, out_f32=of, lse=lse, ws=ws)
    assert csa.csa2_get_device_status(ws) == csa.CSA2_DEV_BAD_INDEX
