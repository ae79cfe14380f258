"""GPU parity of the indexer of the pages' own shape ("Pushing KV Cache Compression to 890 Bytes per
Token", sec. VII: one 128-channel MXFP4 key per entry; the configuration list: 32 indexer heads of
128 channels) against the oracle's LatentCache.index_topk_full: index sets identical (score
descending, ties to the lower position, ascending output, -1 padding) for plain and ReLU scores,
8 and 32 heads, k up to 2048, ratio 2, several rows per sequence, σ = 8, rows with fewer visible
entries than k, an all-zero query (every score ties), an empty row, a row past the workspace bound,
and sampled rows of the full-size workload in bench.py's launch configuration."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_append_b200 as csa
import oracle
from _gpu import DEV, values
from _oracle_pool import oracle_steps
from workloads import gpu as G

pytestmark = pytest.mark.gpu


def _gpu_keys(B, n, seed, sigma=1.0, chunk=4096):
    c = csa.LatentCache(B, n, 128, latent=False)
    ws = G.StatusWs(DEV)
    b = torch.arange(B, device=DEV)
    for p0 in range(0, n, chunk):
        t = min(chunk, n - p0)
        ik = values(seed, "lik", b, torch.arange(p0, p0 + t, device=DEV), 128, DEV, sigma)
        csa.csa2_latent_append(c, B, t, torch.full((B,), p0, dtype=torch.int64, device=DEV), idx_k=ik.contiguous(),
                               ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    return c


def _oracle_keys(b, n, seed, sigma=1.0):
    oc = oracle.LatentCache(n, 128)
    for p0 in range(0, n, 8192):
        oc.append(p0, idx_k=values(seed, "lik", [b], torch.arange(p0, min(n, p0 + 8192)), 128, "cpu", sigma)[0])
    return oc


def _queries(seed, rows, qpos, hi, sigma=1.0):
    p = torch.tensor([[max(x, 0)] for x in qpos])
    return values(seed, "liq", torch.arange(rows), p, hi * 128, "cpu", sigma)[:, 0].reshape(rows, hi, 128).contiguous()


@pytest.mark.parametrize("B,tq,n,hi,k,relu,ratio,sigma", [
    (2, 1, 5000, 32, 512, False, 1, 1.0),
    (2, 1, 5000, 32, 512, True, 1, 1.0),
    (1, 3, 20000, 32, 2048, True, 1, 1.0),
    (2, 2, 3000, 8, 256, False, 2, 8.0),
    (1, 2, 400, 32, 512, True, 1, 1.0),   # fewer visible entries than k
])
def test_latent_index_matches_oracle(orc, B, tq, n, hi, k, relu, ratio, sigma):
    seed = 307 + n + hi + k
    c = _gpu_keys(B, n, seed, sigma)
    rows = B * tq
    qpos = [n - 1 - 37 * (r % tq) - 5 * (r // tq) for r in range(rows)]
    iq = _queries(seed, rows, qpos, hi, sigma)
    out = torch.empty(rows, k, dtype=torch.int32, device=DEV)
    ws = csa.LatentIndexWorkspace(rows, hi, n)
    csa.csa2_latent_index_topk(c, B, tq, torch.tensor(qpos, dtype=torch.int64, device=DEV), iq.to(DEV), k, out, ws,
                               ratio=ratio, max_ctx=n, flags=csa.CSA2_SCORE_RELU if relu else 0)
    assert csa.csa2_get_device_status(ws) == 0
    caches = {}
    for r in range(rows):
        b = r // tq
        if b not in caches:
            caches[b] = _oracle_keys(b, n, seed, sigma)
        ref, _ = caches[b].index_topk_full(qpos[r], iq[r], k=k, relu=relu, ratio=ratio)
        assert np.array_equal(out[r].cpu().numpy(), ref), r


def test_latent_index_ties_empty_row_and_bound(orc):
    """Row 0: an all-zero query, so every score is 0 and the k lowest positions win. Row 1: qpos -1,
    nothing visible. Row 2: an ordinary row. Row 3: more visible entries than max_ctx: reported,
    all -1."""
    B, n, hi, k, seed = 4, 3000, 32, 256, 911
    c = _gpu_keys(B, n, seed)
    max_ctx = n - 50
    qpos = [n - 100, -1, n - 60, n - 1]
    iq = _queries(seed, B, qpos, hi)
    iq[0] = 0
    out = torch.empty(B, k, dtype=torch.int32, device=DEV)
    ws = csa.LatentIndexWorkspace(B, hi, max_ctx)
    csa.csa2_latent_index_topk(c, B, 1, torch.tensor(qpos, dtype=torch.int64, device=DEV), iq.to(DEV), k, out, ws,
                               max_ctx=max_ctx, flags=csa.CSA2_SCORE_RELU)
    assert csa.csa2_get_device_status(ws) == csa.CSA2_DEV_BAD_POS
    got = out.cpu().numpy()
    assert np.array_equal(got[0], np.arange(k))
    assert (got[1] == -1).all() and (got[3] == -1).all()
    ref, _ = _oracle_keys(2, n, seed).index_topk_full(qpos[2], iq[2], k=k, relu=True)
    assert np.array_equal(got[2], ref)
    ref0, _ = _oracle_keys(0, n, seed).index_topk_full(qpos[0], iq[0], k=k, relu=True)
    assert np.array_equal(got[0], ref0)


def test_latent_index_workload_full_size_sampled(orc):
    """128 rows at N = 131,072 (every position filled, as bench.py builds it), ReLU scores, Top-512;
    rows spread over the batch against the oracle, and a repeated step giving the same indices."""
    name = "latent_index_b128_n131072"
    step = G.build(name)
    step.run()
    assert csa.csa2_get_device_status(step.ws) == 0
    seqs = [0, 1, 2, 31, 64, 100, 126, 127]
    ref = oracle_steps(name, seqs)
    for b in seqs:
        assert np.array_equal(step.outputs["idx"][b].cpu().numpy(), ref[b]["idx"]), b
    prev = step.outputs["idx"].clone()
    step.run()
    assert torch.equal(step.outputs["idx"], prev)
    del step
    torch.cuda.empty_cache()
