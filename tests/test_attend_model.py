"""The attention kernel's floating-point arithmetic, modelled on the host, against the oracle.

The kernel feeds exact operands to fp16 tensor-core products: dequantised FP4 and FP8 rows are
exact in fp16, and the bf16 query is rounded to fp16. Logits accumulate in fp32 and are scaled by
sm_scale * log2(e). The softmax is online in fp32 with exp2; the weights P that multiply V are
rounded to fp16, while the running denominator keeps the fp32 values. So the output differs from
the exact one by at most about 2^-11 * max|V| (from the P rounding) plus fp32 terms. These tests
run that arithmetic in numpy (fp32 accumulation, fp16 rounding of q and P), on inputs shaped like
the workloads, and check:
  * the error against the oracle's fp64 attention stays well inside the 2e-3 tolerance at sigma 1
    (and 2e-3 * sigma at sigma 8), which the GPU parity tests use;
  * the error is of the size the P rounding predicts (below 2^-11 * max|V| plus a small fp32 term).
"""
import numpy as np
import pytest
import torch

LOG2E = 1.4426950408889634


def kernel_model(q_bf16, K, V, scale):
    """out [H, 128] and lse [H] as the kernel computes them (fp16 P numerator, fp32 denominator)."""
    q = q_bf16.float().numpy().astype(np.float16).astype(np.float32)
    K32, V32 = K.astype(np.float32), V.astype(np.float32)
    s = (q @ K32.T).astype(np.float32) * np.float32(scale * LOG2E)
    m = s.max(axis=1, keepdims=True)
    p = np.exp2(s - m).astype(np.float32)
    p16 = p.astype(np.float16).astype(np.float32)
    out = (p16 @ V32) / p.sum(axis=1, keepdims=True, dtype=np.float32)
    lse = m[:, 0] / np.float32(LOG2E) + np.log(p.sum(axis=1, dtype=np.float32))
    return out, lse


def rows(orc, c, idx, qpos, win=128):
    """Exact K and V of the selected FP4 rows and the FP8 window rows (decoded by the oracle)."""
    main = orc.dequant_rows(c.kv_data[idx], c.kv_scale[idx], 256)
    lo = max(0, qpos - win + 1)
    w = c.swa[[p & (c.swa_cap - 1) for p in range(lo, qpos + 1)]]
    win_rows = torch.from_numpy(np.ascontiguousarray(w)).view(torch.float8_e4m3fn).double().numpy()
    kv = np.concatenate([main, win_rows])
    return kv[:, :128], kv[:, 128:]


@pytest.mark.parametrize("sigma,n,k", [(1.0, 2048, 512), (1.0, 600, 512), (8.0, 2048, 512), (1.0, 300, 50)])
def test_model_error_is_well_inside_the_tolerance(orc, sigma, n, k):
    g = torch.Generator().manual_seed(int(sigma) * 100 + k)
    c = orc.SeqCache(cap=n, swa_cap=256)
    kv = (torch.randn(n, 256, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    sw = (torch.randn(n, 256, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
    c.append(0, kv=kv, swa_kv=sw)
    worst, worst_bound = 0.0, 0.0
    for trial in range(4):
        q = (torch.randn(16, 128, generator=g) * sigma).clamp(-26, 26).to(torch.bfloat16)
        qpos = n - 1 - 7 * trial
        idx = np.sort(torch.randperm(qpos + 1, generator=g)[:k].numpy()).astype(np.int32)
        ref, rlse = c.sparse_attend(qpos, q, idx)
        K, V = rows(orc, c, idx, qpos)
        out, lse = kernel_model(q, K, V, 1 / np.sqrt(128))
        err = float(np.abs(out - ref).max())
        worst = max(worst, err)
        # P rounding: |sum (p16 - p) V| / sum p <= 2^-11 max|V|; plus fp32 logits and sums
        bound = 2.0 ** -11 * float(np.abs(V).max()) + 1e-5 * sigma
        worst_bound = max(worst_bound, bound)
        assert err <= bound, (trial, err, bound)
        assert float(np.abs(lse - rlse).max()) <= 1e-4 * sigma
    tol = 2e-3 * max(1.0, sigma)
    assert worst <= 0.5 * tol, (worst, tol)
