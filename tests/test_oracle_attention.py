"""Pins of the oracle's sparse attention (R7, R8; "Pushing KV Cache Compression to 890 Bytes
per Token", sec. VI "What one layer looks like", sec. XII SWA Bounded Replay).

* sparse == dense torch fp64 softmax attention when the selection covers every row;
* a single key returns its V exactly;
* the result does not depend on the order of the selected indices;
* softmax over A u B equals the log-sum-exp combination of A and B;
* the window follows [max(s, i - win + 1), i] (tests/golden/swa_window.txt).
FP4 rows are decoded through the golden E2M1 table and torch's E4M3 decoder, FP8 rows
through torch's float8_e4m3fn, not through the oracle.
"""
import numpy as np
import pytest
import torch

from conftest import golden_rows

E2M1 = torch.tensor([float(v) for _, v in golden_rows("e2m1_values.txt")], dtype=torch.float64)


def e4m3(t: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(t)).view(torch.float8_e4m3fn).double()


def fp4_rows(data: np.ndarray, scale: np.ndarray) -> torch.Tensor:
    d = torch.from_numpy(data.astype(np.int64))
    codes = torch.stack([d & 15, d >> 4], dim=-1).reshape(d.shape[0], -1)
    s = e4m3(scale).repeat_interleave(16, dim=1)
    return E2M1[codes] * s


def build(orc, n, seed=0, win=128, swa_cap=256, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    c = orc.SeqCache(cap=n, swa_cap=swa_cap)
    kv = (torch.randn(n, 256, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    sw = (torch.randn(n, 256, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    c.append(0, kv=kv, swa_kv=sw)
    q = (torch.randn(16, 128, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    return c, q


def dense(c, q, main_rows, swa_pos, scale):
    rows = fp4_rows(c.kv_data[main_rows], c.kv_scale[main_rows]) if len(main_rows) else torch.zeros(0, 256, dtype=torch.float64)
    sw = e4m3(c.swa[[p & (c.swa_cap - 1) for p in swa_pos]]) if len(swa_pos) else torch.zeros(0, 256, dtype=torch.float64)
    kvr = torch.cat([rows, sw])
    K, V = kvr[:, :128], kvr[:, 128:]
    lg = q.double() @ K.T * scale
    out = torch.softmax(lg, dim=-1) @ V
    return out.numpy(), torch.logsumexp(lg, dim=-1).numpy()


@pytest.mark.parametrize("sigma", [1.0, 4.0])
def test_sparse_equals_dense_when_selection_covers_all(orc, sigma):
    n = 40
    c, q = build(orc, n, seed=1, sigma=sigma)
    qpos, win = n - 1, 8
    idx = np.concatenate([np.arange(n), -np.ones(24)]).astype(np.int32)
    out, lse = c.sparse_attend(qpos, q, idx, win=win)
    ref, rl = dense(c, q, list(range(n)), list(range(qpos - win + 1, qpos + 1)), 1 / np.sqrt(128))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_single_key_returns_v(orc):
    c, q = build(orc, 10, seed=2)
    idx = np.array([4, -1, -1, -1], np.int32)
    out, lse = c.sparse_attend(9, q, idx, win=0)
    v = fp4_rows(c.kv_data[[4]], c.kv_scale[[4]])[0, 128:].numpy()
    assert np.array_equal(out, np.broadcast_to(v, out.shape))
    k = fp4_rows(c.kv_data[[4]], c.kv_scale[[4]])[0, :128]
    np.testing.assert_allclose(lse, (q.double() @ k / np.sqrt(128)).numpy(), atol=1e-12)


def test_permutation_invariance(orc):
    c, q = build(orc, 300, seed=3)
    rng = np.random.default_rng(0)
    idx = np.sort(rng.choice(300, 64, replace=False)).astype(np.int32)
    a, la = c.sparse_attend(299, q, idx)
    b, lb = c.sparse_attend(299, q, rng.permutation(idx))
    np.testing.assert_allclose(a, b, atol=1e-12)
    np.testing.assert_allclose(la, lb, atol=1e-12)


def test_lse_combination_of_two_splits(orc):
    c, q = build(orc, 200, seed=4)
    sel = np.arange(0, 200, 3).astype(np.int32)
    A, B = sel[:30], sel[30:]
    oa, la = c.sparse_attend(199, q, A, win=0)
    ob, lb = c.sparse_attend(199, q, B, win=0)
    o, l = c.sparse_attend(199, q, sel, win=128)  # window included on the whole side
    ow, lw = c.sparse_attend(199, q, np.array([-1], np.int32), win=128)
    m = np.maximum(np.maximum(la, lb), lw)
    wa, wb, ww = np.exp(la - m), np.exp(lb - m), np.exp(lw - m)
    comb = (oa * wa[:, None] + ob * wb[:, None] + ow * ww[:, None]) / (wa + wb + ww)[:, None]
    np.testing.assert_allclose(o, comb, atol=1e-12)
    np.testing.assert_allclose(l, m + np.log(wa + wb + ww), atol=1e-12)


def test_window_golden_cases(orc):
    for s, i, win, lo, hi in [[int(v) for v in r] for r in golden_rows("swa_window.txt")]:
        c = orc.SeqCache(cap=1, swa_cap=256)
        g = torch.Generator().manual_seed(i)
        q = torch.randn(16, 128, generator=g).to(torch.bfloat16)
        sw = torch.randn(256, 256, generator=g).to(torch.bfloat16)
        # write the ring directly through the oracle's FP8 codec: slot = p & 255
        base = max(0, i - 255)
        for p in range(base, i + 1):
            c.swa[p & 255] = orc.fp8_rows(sw[p - base])
        out, lse = c.sparse_attend(i, q, np.array([-1], np.int32), swa_begin=s, win=win)
        want = list(range(lo, hi + 1))
        if not want:
            assert np.all(out == 0) and np.all(np.isneginf(lse))
            continue
        ref, rl = dense(c, q, [], want, 1 / np.sqrt(128))
        np.testing.assert_allclose(out, ref, atol=1e-12)
        np.testing.assert_allclose(lse, rl, atol=1e-12)


def test_default_scale_is_inverse_sqrt_d(orc):
    c, q = build(orc, 20, seed=6)
    idx = np.arange(20, dtype=np.int32)
    a, la = c.sparse_attend(19, q, idx, sm_scale=0.0)
    b, lb = c.sparse_attend(19, q, idx, sm_scale=1 / np.sqrt(128))
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_ratio_two_selected_rows_must_be_complete(orc):
    """R12 with r = 2: a query at token 150 may use entries 0..74 (entry 74 covers tokens 148, 149);
    entry 75 covers token 151, which is in the future. The window stays per token."""
    c, q = build(orc, 200, seed=12)
    qpos, scale = 150, 1.0 / np.sqrt(128.0)
    idx = np.array([0, 10, 74, -1], np.int32)
    out, lse = c.sparse_attend(qpos, q, idx, ratio=2)
    want, wl = dense(c, q, [0, 10, 74], list(range(qpos - 127, qpos + 1)), scale)
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, wl, rtol=0, atol=1e-12)
    with pytest.raises(ValueError):
        c.sparse_attend(qpos, q, np.array([75], np.int32), ratio=2)
    c.sparse_attend(qpos, q, np.array([75], np.int32), ratio=1)  # visible without compression
