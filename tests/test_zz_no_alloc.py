"""csa2_sparse_attend_noalloc: the attention entry point for callers that cannot allocate device
memory where they run attention (its scratch lives in a static device array inside libcsa2).

Called through the C ABI twice in a row, it must give what csa2_sparse_attend gives with a caller
workspace, within the attention tolerance. The second call checks that the shared scratch was left
ready (split tickets back at zero). This file is collected last so that a failure here never hides
the other tests; it passes alone in a fresh process too.
"""
import pytest
import torch

import compressed_sparse_attention_append_b200 as csa
import workloads as W
from _gpu import DEV, gpu_fill, query_values

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,n,k", [(3, 700, 512), (200, 400, 64)])
def test_noalloc_matches_workspace_entry_point(B, n, k):
    seed = 97 + B
    shape = csa.make_shape()
    swa_cap = 1 << max(7, (n - 1).bit_length())
    cache = csa.Cache(B, n, swa_cap)
    gpu_fill(cache, shape, seed, B, n)
    qpos = torch.tensor([n - 1 - 5 * (i % 3) for i in range(B)], dtype=torch.int64, device=DEV)
    q = query_values(seed, "q", torch.arange(B), qpos, 2048, DEV).reshape(B, 16, 128).contiguous()
    nsel = min(k, n // 2 - 3)
    idx = W.distinct_sorted(seed, "sel", torch.arange(B, device=DEV), n - 20, nsel).to(torch.int32)
    idx = torch.cat([idx, torch.full((B, k - nsel), -1, dtype=torch.int32, device=DEV)], 1).contiguous()

    ref = torch.empty(B, 16, 128, dtype=torch.float32, device=DEV)
    ref_bf = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=DEV)
    ws = csa.Workspace(shape, B, 1, k, 8)
    csa.csa2_sparse_attend(shape, cache, B, 1, qpos, q, idx, k, ref_bf, out_f32=ref, ws=ws)
    for call in range(2):
        of = torch.full((B, 16, 128), float("nan"), dtype=torch.float32, device=DEV)
        out = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=DEV)
        csa.csa2_sparse_attend_noalloc(shape, cache, B, 1, qpos, q, idx, k, out, out_f32=of)
        torch.cuda.synchronize()
        err = float((of - ref).abs().max())
        assert err <= 2e-3, (call, err)
        assert torch.equal(out, of.to(torch.bfloat16))


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
