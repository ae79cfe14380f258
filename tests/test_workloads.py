"""The seeded input generator: its definition (splitmix64 + Irwin-Hall(12)) checked against an
independent numpy uint64 implementation, its distribution, and its position sets."""
import numpy as np
import torch

import workloads as W


def np_splitmix(x):
    with np.errstate(over="ignore"):
        z = (x + np.uint64(0x9E3779B97F4A7C15))
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def np_gauss(seed, stream, n, sigma=1.0, clip=26.0):
    base = np.uint64(W.splitmix64_int(((seed << 32) + W.STREAM[stream]) & W.M64))
    with np.errstate(over="ignore"):
        c = n.astype(np.uint64) * np.uint64(3) + base
        s = np.zeros(n.shape, np.int64)
        for j in range(3):
            h = np_splitmix(c + np.uint64(j))
            for i in range(4):
                s += ((h >> np.uint64(16 * i)) & np.uint64(0xFFFF)).astype(np.int64)
    z = (s - 393210).astype(np.float32) * np.float32(1 / 65536)
    z = np.clip(z * np.float32(sigma), -clip, clip).astype(np.float32)
    return torch.from_numpy(z).to(torch.bfloat16)


def test_generator_matches_numpy_definition():
    n = np.arange(0, 200000, 7, dtype=np.int64)
    for seed, stream, sigma in [(0, "kv", 1.0), (3, "swa", 8.0), (4, "q", 1.0)]:
        a = W.gaussian_bf16(seed, stream, torch.from_numpy(n), sigma)
        b = np_gauss(seed, stream, n, sigma)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    big = torch.tensor([(127 << 21) * 256 + 255, (1 << 48) + 5], dtype=torch.int64)
    assert torch.equal(W.gaussian_bf16(2, "ik", big).view(torch.int16),
                       np_gauss(2, "ik", big.numpy()).view(torch.int16))


def test_distribution():
    v = W.gaussian_bf16(1, "kv", torch.arange(1 << 20)).double()
    assert abs(v.mean()) < 5e-3 and abs(v.std() - 1) < 5e-3
    assert v.abs().max() <= 6.0
    big = W.gaussian_bf16(1, "kv", torch.arange(1 << 16), sigma=8.0).double()
    assert big.abs().max() <= 26.0 and (big.abs() == 26.0).any()


def test_distinct_sorted_sets():
    b = torch.arange(5)
    s = W.distinct_sorted(2, "pool", b, 131072 // 64, 200)
    assert s.shape == (5, 200)
    for r in s:
        assert torch.all(r[1:] > r[:-1]) and r.min() >= 0 and r.max() < 2048
    assert not torch.equal(s[0], s[1])
    s2 = W.distinct_sorted(2, "pool", torch.tensor([3]), 131072 // 64, 200)
    assert torch.equal(s2[0], s[3])  # a sequence's set does not depend on the batch it came in


def test_cache_counters_layout():
    c = W.cache_counters(torch.tensor([0, 2]), torch.tensor([[5], [7]]), 4)
    assert c.tolist() == [[[20, 21, 22, 23]], [[((2 << 21) + 7) * 4 + i for i in range(4)]]]


def test_draft_rows_are_causal_in_the_oracle_driver(orc):
    """Multi-token decode on the oracle side, at a small context: row t of a step that appended all 5
    draft tokens equals row t of a step whose cache holds only the tokens up to N-5+t, and every
    selected position of row t is visible to it."""
    from oracle import workload as OW

    wl = OW.workload("draft_b64_n131072_tq5", context=2048)
    p0 = wl.context - wl.tq
    c, inp = OW.build_sequence(wl, 3)
    r = OW.run_step(c, wl, inp)
    assert sorted(r["rows"]) == list(range(wl.tq))
    for t in range(wl.tq):
        idx, out, lse = r["rows"][t]
        sel = idx[idx >= 0]
        assert sel.size == wl.k and sel.max() <= p0 + t and np.all(np.diff(sel) > 0)
        c2, inp2 = OW.build_sequence(wl, 3)
        c2.append(p0, kv=inp2["kv"][:t + 1], idx_k=inp2["idx_k"][:t + 1], swa_kv=inp2["swa_kv"][:t + 1])
        idx2 = c2.index_topk_full(p0 + t, inp2["idx_q"][t], k=wl.k)
        out2, lse2 = c2.sparse_attend(p0 + t, inp2["q"][t], idx2)
        assert np.array_equal(idx, idx2)
        assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    # the rows differ: each sees one more token and has its own query
    assert not np.array_equal(r["rows"][0][1], r["rows"][wl.tq - 1][1])


def test_inputs_never_saturate_a_scale(orc):
    """Headroom ([C] sec. XI): the FP4 range reaches 6 x 448 = 2688, while post-RoPE values stay near
    sqrt(512) ~ 22.6 and the generator clips at 26. So a block scale amax / 6 <= 26 / 6 never comes
    near the E4M3 limit 448: no generated block saturates its scale, at sigma 1 or at sigma 8."""
    for sigma in (1.0, 8.0):
        b = torch.arange(4)
        p = torch.arange(2048)
        x = W.cache_values(7, "kv", b, p, 256, sigma).reshape(-1, 256)
        assert float(x.float().abs().max()) <= 26.0
        data, scale = orc.quantize_rows(x, 256)
        smax = max(orc.e4m3_decode(int(v)) for v in np.unique(scale))
        assert smax <= 4.5  # 26 / 6 = 4.33 rounds to the E4M3 value 4.5 at most
        assert 448 / smax >= 99  # about two orders of magnitude of headroom below saturation
