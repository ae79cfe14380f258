"""csa2_sparse_attend_noalloc: the attention entry point for callers that cannot allocate device
memory where they run attention (its scratch lives in a static device array inside libcsa2).

Called through the C ABI several times in a row, it must give what csa2_sparse_attend gives with a
caller workspace, and what the oracle gives, within the attention tolerance. The calls change the
batch, the rows per sequence and so the split count between them, so that each call finds the
shared tickets where the call before left them. The first call runs on a non-blocking stream (the
array must need no clearing that the caller's stream does not order). This file is collected last
so that a failure here never hides the other tests; it passes alone in a fresh process too.
"""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_append_b200 as csa
import workloads as W
from _gpu import DEV, attn_tol, gpu_fill, oracle_seq, query_values

pytestmark = pytest.mark.gpu

# (batch, tq, context n, k, ratio): 3 rows are split many ways, 200 rows a few, 1000 rows not at all
CALLS = [(3, 1, 700, 512, 1), (40, 5, 1200, 256, 2), (200, 1, 400, 64, 1), (1000, 1, 300, 32, 1), (2, 5, 900, 512, 2)]


def _inputs(B, tq, n, k, ratio, seed):
    swa_cap = 1 << max(7, (n + 8).bit_length())
    cache = csa.Cache(B, n, swa_cap)
    gpu_fill(cache, csa.make_shape(), seed, B, n)
    # row i of sequence b sits at token n - 1 - 3 * (b % 3) - (tq - 1 - i)
    qpos = [n - 1 - 3 * (b % 3) - (tq - 1 - i) for b in range(B) for i in range(tq)]
    qp = torch.tensor(qpos, dtype=torch.int64, device=DEV)
    rows = torch.arange(B * tq)
    q = query_values(seed, "q", rows, qp, 2048, DEV).reshape(B * tq, 16, 128).contiguous()
    vis = (n - 1 - 3 * 2 - (tq - 1) + 1) // ratio  # entries every row may use
    nsel = min(k, vis // 2)
    idx = W.distinct_sorted(seed, "sel", torch.arange(B * tq, device=DEV), vis, nsel).to(torch.int32)
    idx = torch.cat([idx, torch.full((B * tq, k - nsel), -1, dtype=torch.int32, device=DEV)], 1).contiguous()
    return cache, swa_cap, qpos, qp, q, idx


def test_noalloc_matches_workspace_entry_point_and_oracle(orc):
    side = torch.cuda.Stream()  # non-blocking with respect to the legacy default stream
    for c, (B, tq, n, k, ratio) in enumerate(CALLS):
        seed = 97 + c
        shape = csa.make_shape(ratio=ratio)
        cache, swa_cap, qpos, qp, q, idx = _inputs(B, tq, n, k, ratio, seed)
        R = B * tq
        ref = torch.empty(R, 16, 128, dtype=torch.float32, device=DEV)
        ref_bf = torch.empty(R, 16, 128, dtype=torch.bfloat16, device=DEV)
        ref_lse = torch.empty(R, 16, dtype=torch.float32, device=DEV)
        ws = csa.Workspace(shape, B, tq, k, 8)
        csa.csa2_sparse_attend(shape, cache, B, tq, qp, q, idx, k, ref_bf, out_f32=ref, lse=ref_lse, ws=ws)
        assert csa.csa2_get_device_status(ws) == 0
        torch.cuda.synchronize()
        of = torch.full((R, 16, 128), float("nan"), dtype=torch.float32, device=DEV)
        out = torch.empty(R, 16, 128, dtype=torch.bfloat16, device=DEV)
        lse = torch.full((R, 16), float("nan"), dtype=torch.float32, device=DEV)
        if c == 0:
            with torch.cuda.stream(side):
                csa.csa2_sparse_attend_noalloc(shape, cache, B, tq, qp, q, idx, k, out, out_f32=of, lse=lse)
            side.synchronize()
        else:
            csa.csa2_sparse_attend_noalloc(shape, cache, B, tq, qp, q, idx, k, out, out_f32=of, lse=lse)
        torch.cuda.synchronize()
        err = float((of - ref).abs().max())
        assert err <= 2e-3, (c, err)
        assert float((lse - ref_lse).abs().max()) <= 2e-3, c
        assert torch.equal(out, of.to(torch.bfloat16)), c
        # the oracle on the first and the last row
        for r in (0, R - 1):
            b = r // tq
            oc = oracle_seq(seed, b, n, n, swa_cap)
            qr = query_values(seed, "q", [r], [qpos[r]], 2048, "cpu")[0]
            ro, rl = oc.sparse_attend(qpos[r], qr, idx[r].cpu().numpy(), ratio=ratio)
            assert np.abs(of[r].double().cpu().numpy() - ro).max() <= attn_tol(ro), (c, r)
            assert np.abs(lse[r].double().cpu().numpy() - rl).max() <= attn_tol(ro), (c, r)


def test_noalloc_rejects_too_many_rows():
    shape = csa.make_shape()
    cache = csa.Cache(1, 64, 128)
    B = 1025
    qpos = torch.zeros(B, dtype=torch.int64, device=DEV)
    q = torch.zeros(B, 16, 128, dtype=torch.bfloat16, device=DEV)
    idx = torch.full((B, 16), -1, dtype=torch.int32, device=DEV)
    out = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(csa.Csa2Error) as e:
        csa.csa2_sparse_attend_noalloc(shape, cache, B, 1, qpos, q, idx, 16, out)
    assert e.value.status == csa.CSA2_ERR_CAPACITY
