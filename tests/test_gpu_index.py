"""Index scoring, exact Top-k, block pool and Reindex on the GPU against the oracle: index sets
must be identical (the scores are exact on both sides and the ranking is a total order)."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_append_b200 as csa
import oracle
import workloads as W
from _gpu import DEV, bf16_np, gpu_fill, oracle_seq, query_values, values

pytestmark = pytest.mark.gpu


def _setup(B, n, seed, sigma=1.0, cap=None):
    cap = cap or n
    shape = csa.make_shape()
    swa_cap = 1 << max(7, (n - 1).bit_length())
    cache = csa.Cache(B, cap, swa_cap)
    gpu_fill(cache, shape, seed, B, n, sigma)
    return shape, cache, swa_cap


@pytest.mark.parametrize("B,n,k,pool,sigma,ragged", [
    (1, 37, 16, 4, 1.0, False),
    (3, 600, 64, 16, 1.0, True),
    (2, 4099, 512, 0, 1.0, True),
    (2, 9000, 512, 2048, 8.0, True),
    (1, 20000, 512, 600, 1.0, False),
])
def test_full_mode_matches_oracle(orc, B, n, k, pool, sigma, ragged):
    seed = 11 + n
    shape, cache, swa_cap = _setup(B, n, seed, sigma)
    qpos = [n - 1 - (37 * i if ragged else 0) for i in range(B)]
    qp = torch.tensor(qpos, dtype=torch.int64, device=DEV)
    iq = query_values(seed, "iq", torch.arange(B), qp, 256, DEV, sigma).contiguous()
    out = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
    opool = torch.full((B, max(pool, 1)), -7, dtype=torch.int32, device=DEV)
    opn = torch.zeros(B, dtype=torch.int32, device=DEV)
    ws = csa.Workspace(shape, B, 1, k, n, pool)
    refs = []
    for b in range(B):
        oc = oracle_seq(seed, b, n, n, swa_cap, sigma)
        qb = query_values(seed, "iq", [b], [qpos[b]], 256, "cpu", sigma)[0]
        refs.append(oc.index_topk_full(qpos[b], qb, k=k, pool_blocks=pool) if pool else
                    (oc.index_topk_full(qpos[b], qb, k=k), None, None))
    for rep in range(2):  # the second call checks that the counters were left cleared
        csa.csa2_index_topk_full(shape, cache, B, 1, qp, iq, k, out, pool, opool if pool else None,
                                 opn if pool else None, max_ctx=n, ws=ws)
        assert csa.csa2_get_device_status(ws) == 0
        for b in range(B):
            ridx, rpool, rpn = refs[b]
            if pool:
                assert int(opn[b]) == rpn
                assert np.array_equal(opool[b].cpu().numpy(), rpool)
            assert np.array_equal(out[b].cpu().numpy(), ridx), (rep, b)


@pytest.mark.parametrize("tq,ratio", [(3, 1), (5, 1), (3, 2)])
def test_full_mode_multi_row_queries(orc, tq, ratio):
    """tq > 1 query rows per sequence (the prefill form, and 5 draft positions verified together):
    every row ranks its own visible prefix (with ratio 2: the entries whose two tokens precede it)."""
    B, n, k = 2, 5000, 256
    seed = 91
    _, cache, swa_cap = _setup(B, n, seed)
    shape = csa.make_shape(ratio=ratio)
    qpos = [[n - 1 - 700 * b - 13 * t for t in range(tq)] for b in range(B)]
    qp = torch.tensor(qpos, dtype=torch.int64, device=DEV).reshape(-1)
    rows_b = torch.arange(B).repeat_interleave(tq)
    iq = query_values(seed, "iq", rows_b.to(DEV), qp, 256, DEV).contiguous()
    out = torch.full((B * tq, k), -7, dtype=torch.int32, device=DEV)
    ws = csa.Workspace(shape, B, tq, k, n)
    csa.csa2_index_topk_full(shape, cache, B, tq, qp, iq, k, out, max_ctx=n, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    for b in range(B):
        oc = oracle_seq(seed, b, n, n, swa_cap)
        for t in range(tq):
            qb = query_values(seed, "iq", [b], [qpos[b][t]], 256, "cpu")[0]
            ref = oc.index_topk_full(qpos[b][t], qb, k=k, ratio=ratio)
            assert np.array_equal(out[b * tq + t].cpu().numpy(), ref), (b, t)


@pytest.mark.parametrize("B,tq,n,k", [(1, 300, 20000, 512), (3, 5, 20000, 512), (2, 40, 9000, 256)])
def test_full_mode_multi_row_tensor_core(orc, B, tq, n, k):
    """Several rows per sequence at a context that takes the tensor-core filter (approximate MMA
    scores, exact rescoring of the survivors): index sets identical to the oracle's. The rows mix
    the cases of that path: the usual sampled threshold, a row whose visible prefix fits the
    candidate list (every position admitted), a row seeing fewer than k positions, and an all-zero
    query (every score equal: the candidate list overflows and the exact scan takes the row)."""
    seed = 17 + tq
    shape, cache, swa_cap = _setup(B, n, seed)
    rng = np.random.default_rng(seed)
    qpos = [[n - 1 - int(rng.integers(0, n // 4)) for _ in range(tq)] for _ in range(B)]
    qpos[0][0] = n - 1
    if tq > 2:
        qpos[0][1] = 3000          # visible prefix within the candidate list
        qpos[0][2] = k // 2        # fewer than k visible positions
    qp = torch.tensor(qpos, dtype=torch.int64, device=DEV).reshape(-1)
    rows_b = torch.arange(B).repeat_interleave(tq)
    iq = query_values(seed, "iq", rows_b.to(DEV), qp, 256, DEV).contiguous()
    zero_row = B * tq - 1
    iq[zero_row] = 0
    out = torch.full((B * tq, k), -7, dtype=torch.int32, device=DEV)
    ws = csa.Workspace(shape, B, tq, k, n)
    for rep in range(2):
        csa.csa2_index_topk_full(shape, cache, B, tq, qp, iq, k, out, max_ctx=n, ws=ws)
        assert csa.csa2_get_device_status(ws) == 0
        for b in range(B):
            oc = oracle_seq(seed, b, n, n, swa_cap)
            for t in range(tq):
                r = b * tq + t
                qb = iq[r].cpu() if r == zero_row else query_values(seed, "iq", [b], [qpos[b][t]], 256, "cpu")[0]
                ref = oc.index_topk_full(qpos[b][t], bf16_np(qb), k=k)
                assert np.array_equal(out[r].cpu().numpy(), ref), (rep, b, t)


def test_prefill_chunk_tensor_core_blind_sample(orc):
    """A prefill chunk over a context where every 5th key is 8x larger: the sampled tile maxima see
    mostly those keys; the selection must still be exact (through the filter, or the exact scan for
    rows whose threshold admitted fewer than k keys)."""
    n, t, k = 12000, 64, 512
    p = torch.arange(n)
    ik = values(8, "ik", [0], p, 256, "cpu")[0].float()
    ik[p % 5 == 0] *= 8.0
    ik = ik.to(torch.bfloat16)
    shape = csa.make_shape()
    cache = csa.Cache(1, n, 1 << 14)
    ws = csa.Workspace(shape, 1, t, k, n)
    pos = torch.zeros(1, dtype=torch.int64, device=DEV)
    csa.csa2_quantize_append(shape, cache, 1, n, pos, None, ik[None].to(DEV).contiguous(), None, ws=ws)
    qpos = torch.arange(n - t, n, dtype=torch.int64)
    iq = query_values(8, "iq", torch.zeros(t, dtype=torch.int64), qpos, 256, "cpu").contiguous()
    out = torch.full((t, k), -7, dtype=torch.int32, device=DEV)
    csa.csa2_index_topk_full(shape, cache, 1, t, qpos.to(DEV), iq.to(DEV), k, out, max_ctx=n, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    oc = oracle.SeqCache(n, 1 << 14)
    oc.append(0, idx_k=bf16_np(ik))
    for r in range(0, t, 7):
        ref = oc.index_topk_full(int(qpos[r]), bf16_np(iq[r]), k=k)
        assert np.array_equal(out[r].cpu().numpy(), ref), r


def test_full_mode_long_pool(orc):
    """More pool blocks than fit on chip (17,500 blocks of 8): the pool ranking reads from memory."""
    B, n, k, P = 1, 140000, 64, 256
    seed = 17
    shape, cache, swa_cap = _setup(B, n, seed, cap=n)
    qp = torch.tensor([n - 1], dtype=torch.int64, device=DEV)
    iq = query_values(seed, "iq", [0], qp, 256, DEV).contiguous()
    out = torch.empty(B, k, dtype=torch.int32, device=DEV)
    opool = torch.empty(B, P, dtype=torch.int32, device=DEV)
    opn = torch.empty(B, dtype=torch.int32, device=DEV)
    ws = csa.Workspace(shape, B, 1, k, n, P)
    csa.csa2_index_topk_full(shape, cache, B, 1, qp, iq, k, out, P, opool, opn, max_ctx=n, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    oc = oracle_seq(seed, 0, n, n, swa_cap)
    qb = query_values(seed, "iq", [0], [n - 1], 256, "cpu")[0]
    ridx, rpool, rpn = oc.index_topk_full(n - 1, qb, k=k, pool_blocks=P)
    assert int(opn[0]) == rpn
    assert np.array_equal(opool[0].cpu().numpy(), rpool)
    assert np.array_equal(out[0].cpu().numpy(), ridx)


def _full_from_rows(ik_cpu, kv_cpu, k, pool=0):
    """Full mode over one sequence whose indexer keys are the given bf16 rows (made on the host)."""
    n = ik_cpu.shape[0]
    shape = csa.make_shape()
    cache = csa.Cache(1, n, 1 << max(7, (n - 1).bit_length()))
    csa.csa2_quantize_append(shape, cache, 1, n, torch.zeros(1, dtype=torch.int64, device=DEV),
                             kv_cpu[None].to(DEV).contiguous(), ik_cpu[None].to(DEV).contiguous(),
                             kv_cpu[None].to(DEV).contiguous())
    iq = query_values(5, "iq", [0], [n - 1], 256, "cpu")
    qp = torch.tensor([n - 1], dtype=torch.int64, device=DEV)
    out = torch.empty(1, k, dtype=torch.int32, device=DEV)
    opool = torch.empty(1, max(pool, 1), dtype=torch.int32, device=DEV)
    opn = torch.empty(1, dtype=torch.int32, device=DEV)
    ws = csa.Workspace(shape, 1, 1, k, n, pool)
    csa.csa2_index_topk_full(shape, cache, 1, 1, qp, iq.to(DEV).contiguous(), k, out, pool,
                             opool if pool else None, opn if pool else None, max_ctx=n, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    oc = oracle.SeqCache(n, 1 << max(7, (n - 1).bit_length()))
    oc.append(0, kv=bf16_np(kv_cpu), idx_k=bf16_np(ik_cpu))
    if pool:
        ridx, rpool, rpn = oc.index_topk_full(n - 1, bf16_np(iq[0]), k=k, pool_blocks=pool)
        assert int(opn[0]) == rpn
        assert np.array_equal(opool[0].cpu().numpy(), rpool)
    else:
        ridx = oc.index_topk_full(n - 1, bf16_np(iq[0]), k=k)
    got = out[0].cpu().numpy()
    assert np.array_equal(got, ridx)
    return got


def test_full_mode_all_keys_equal(orc):
    """Every position has the same indexer key: one score for all, so the k lowest positions win."""
    n, k = 5000, 256
    p = torch.arange(n)
    ik = values(6, "ik", [0], torch.zeros(n, dtype=torch.int64), 256, "cpu")[0]
    kv = values(6, "kv", [0], p, 256, "cpu")[0]
    got = _full_from_rows(ik, kv, k, pool=64)
    assert np.array_equal(got, np.arange(k))


def test_full_mode_sample_blind_to_most_keys(orc):
    """Keys at every 5th position are 8x larger: a regular sample of the keys sees only those, so the
    threshold it suggests admits fewer than k keys and the ranking must run over every key."""
    n, k = 20000, 512
    p = torch.arange(n)
    ik = values(8, "ik", [0], p, 256, "cpu")[0].float()
    ik[p % 5 == 0] *= 8.0
    ik = ik.to(torch.bfloat16)
    kv = values(8, "kv", [0], p, 256, "cpu")[0]
    _full_from_rows(ik, kv, k, pool=300)


def test_full_mode_relu_and_ties(orc):
    """Identical indexer keys at many positions force exact score ties: the lower position wins."""
    B, n, k = 1, 3000, 512
    shape = csa.make_shape()
    cache = csa.Cache(B, n, 4096)
    p = torch.arange(n, device=DEV)
    ik = values(3, "ik", [0], p % 97, 256, DEV).contiguous()  # 97 distinct keys, repeated
    kv = values(3, "kv", [0], p, 256, DEV).contiguous()
    csa.csa2_quantize_append(shape, cache, 1, n, torch.zeros(1, dtype=torch.int64, device=DEV), kv, ik, kv)
    iq = query_values(3, "iq", [0], [n - 1], 256, DEV).contiguous()
    qp = torch.tensor([n - 1], dtype=torch.int64, device=DEV)
    oc = oracle.SeqCache(n, 4096)
    oc.append(0, kv=bf16_np(kv[0]), idx_k=bf16_np(ik[0]))
    qb = bf16_np(iq[0])
    for flags, relu in ((0, False), (csa.CSA2_SCORE_RELU, True)):
        out = torch.empty(B, k, dtype=torch.int32, device=DEV)
        ws = csa.Workspace(shape, B, 1, k, n)
        csa.csa2_index_topk_full(shape, cache, B, 1, qp, iq, k, out, max_ctx=n, flags=flags, ws=ws)
        ref = oc.index_topk_full(n - 1, qb, k=k, relu=relu)
        assert np.array_equal(out[0].cpu().numpy(), ref), relu


@pytest.mark.parametrize("B,n,P,k,shuffled", [
    (2, 4096, 40, 128, False),
    (3, 50000, 2000, 512, False),
    (1, 1000, 125, 512, False),
    (3, 1000, 125, 64, False),   # 125 units per row: the last scoring step reaches past each row
    (2, 5000, 301, 64, True),    # pool blocks listed out of order: the output is still ascending
])
def test_reindex_matches_oracle(orc, B, n, P, k, shuffled):
    seed = 23 + P
    shape, cache, swa_cap = _setup(B, n, seed)
    nblk = (n + 7) // 8
    pool = W.distinct_sorted(seed, "pool", torch.arange(B, device=DEV), nblk, P).to(torch.int32)
    if shuffled:
        g = torch.Generator().manual_seed(seed)
        pool = torch.stack([r[torch.randperm(P, generator=g).to(DEV)] for r in pool])
    pool = pool.contiguous()
    pool_n = torch.tensor([P - 3 * i for i in range(B)], dtype=torch.int32, device=DEV)
    qpos = [n - 1 - 101 * i for i in range(B)]
    qp = torch.tensor(qpos, dtype=torch.int64, device=DEV)
    iq = query_values(seed, "iq", torch.arange(B), qp, 256, DEV).contiguous()
    out = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
    ws = csa.Workspace(shape, B, 1, k, P * 8)
    csa.csa2_index_topk_reindex(shape, cache, B, qp, iq, pool, pool_n, k, out, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    for b in range(B):
        oc = oracle_seq(seed, b, n, n, swa_cap)
        qb = query_values(seed, "iq", [b], [qpos[b]], 256, "cpu")[0]
        pl = pool[b].cpu().numpy()
        ref = oc.index_topk_reindex(qpos[b], qb, pl, int(pool_n[b]), k=k)
        assert np.array_equal(out[b].cpu().numpy(), ref), b


def test_reindex_with_full_query_reproduces_full_topk(orc):
    """Pool built by Full mode, then Reindex with the same query: the same Top-k."""
    B, n, k, P = 2, 30000, 512, 2048
    shape, cache, _ = _setup(B, n, 77)
    qp = torch.tensor([n - 1, n - 500], dtype=torch.int64, device=DEV)
    iq = query_values(77, "iq", torch.arange(B), qp, 256, DEV).contiguous()
    out = torch.empty(B, k, dtype=torch.int32, device=DEV)
    opool = torch.empty(B, P, dtype=torch.int32, device=DEV)
    opn = torch.empty(B, dtype=torch.int32, device=DEV)
    ws = csa.Workspace(shape, B, 1, k, n, P)
    csa.csa2_index_topk_full(shape, cache, B, 1, qp, iq, k, out, P, opool, opn, max_ctx=n, ws=ws)
    out2 = torch.empty(B, k, dtype=torch.int32, device=DEV)
    csa.csa2_index_topk_reindex(shape, cache, B, qp, iq, opool, opn, k, out2, ws=ws)
    assert torch.equal(out, out2)
    for b in range(B):
        sel = out[b][out[b] >= 0]
        blocks = set(opool[b][: int(opn[b])].tolist())
        assert all(int(x) // 8 in blocks for x in sel)


def test_bad_pool_id_sets_status():
    shape, cache, _ = _setup(1, 256, 5)
    pool = torch.tensor([[0, 3, 1000]], dtype=torch.int32, device=DEV)
    pool_n = torch.tensor([3], dtype=torch.int32, device=DEV)
    qp = torch.tensor([255], dtype=torch.int64, device=DEV)
    iq = query_values(5, "iq", [0], qp, 256, DEV).contiguous()
    out = torch.empty(1, 16, dtype=torch.int32, device=DEV)
    ws = csa.Workspace(shape, 1, 1, 16, 24)
    csa.csa2_index_topk_reindex(shape, cache, 1, qp, iq, pool, pool_n, 16, out, ws=ws)
    assert csa.csa2_get_device_status(ws) == csa.CSA2_DEV_BAD_POOL
    got = out[0].cpu().numpy()
    assert set(got[got >= 0].tolist()) == set(range(0, 8)) | set(range(24, 32))


def test_ratio_two_full_and_reindex(orc):
    """Compression ratio 2: the rows at tokens 2n - 1 and 2n - 6 see the first n and n - 3 entries
    (entry e summarises tokens 2e, 2e + 1). Full (with its pool) and Reindex against the oracle."""
    B, n, k, P = 2, 6000, 256, 300
    seed = 63
    _, cache, swa_cap = _setup(B, n, seed)
    shape = csa.make_shape(ratio=2)
    qpos = [2 * n - 1, 2 * n - 6]
    qp = torch.tensor(qpos, dtype=torch.int64, device=DEV)
    iq = query_values(seed, "iq", torch.arange(B), qp, 256, DEV).contiguous()
    out = torch.empty(B, k, dtype=torch.int32, device=DEV)
    opool = torch.empty(B, P, dtype=torch.int32, device=DEV)
    opn = torch.empty(B, dtype=torch.int32, device=DEV)
    ws = csa.Workspace(shape, B, 1, k, n, P)
    csa.csa2_index_topk_full(shape, cache, B, 1, qp, iq, k, out, P, opool, opn, max_ctx=n, ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    pool = W.distinct_sorted(seed, "pool", torch.arange(B, device=DEV), n // 8, 400).to(torch.int32).contiguous()
    pool_n = torch.tensor([400, 390], dtype=torch.int32, device=DEV)
    out2 = torch.empty(B, k, dtype=torch.int32, device=DEV)
    ws2 = csa.Workspace(shape, B, 1, k, 400 * 8)
    csa.csa2_index_topk_reindex(shape, cache, B, qp, iq, pool, pool_n, k, out2, ws=ws2)
    assert csa.csa2_get_device_status(ws2) == 0
    for b in range(B):
        oc = oracle_seq(seed, b, n, n, swa_cap)
        qb = query_values(seed, "iq", [b], [qpos[b]], 256, "cpu")[0]
        ridx, rpool, rpn = oc.index_topk_full(qpos[b], qb, k=k, pool_blocks=P, ratio=2)
        assert int(opn[b]) == rpn
        assert np.array_equal(opool[b].cpu().numpy(), rpool)
        assert np.array_equal(out[b].cpu().numpy(), ridx)
        rr = oc.index_topk_reindex(qpos[b], qb, pool[b].cpu().numpy(), int(pool_n[b]), k=k, ratio=2)
        assert np.array_equal(out2[b].cpu().numpy(), rr)
