"""GPU parity of the pages' own attention shape ("Pushing KV Cache Compression to 890 Bytes per
Token", sec. VII and its configuration list: 64 query heads of 512 channels over ONE 512-channel
latent per entry, which is both key and value; sec. XII for the window) against the oracle's
LatentCache (fp64):

* csa2_latent_append: latent (E2M1 + E4M3 per 16), indexer key (MXFP4) and window (E4M3) planes
  byte for byte, the ring wrapping, an append past the capacity reported and skipped;
* csa2_latent_attend (tensor cores): fp32 output within the tolerance of fp16 probabilities,
  bf16 = RNE of fp32, lse; full, ragged and -1-padded selections in any order, 16 key tiles,
  several rows per sequence, ratio 2, a cut window, window-only and empty rows, a bad index;
* a constructed row whose per-head maxima jump by more than the lazy-rescale threshold from tile
  to tile on some heads and creep up below it on others, so that both the in-place rescale of the
  accumulated output and the deferred maximum are exercised;
* the full-size workload (128 sequences at N = 131,072) in bench.py's launch configuration, every
  sequence, and a repeated step giving identical bytes.
"""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_append_b200 as csa
import oracle
import workloads as W
from _gpu import DEV, attn_tol, values
from _oracle_pool import oracle_steps
from workloads import gpu as G

pytestmark = pytest.mark.gpu


def _planes(seed, b, p, device, sigma):
    """bf16 latent [.., 512], indexer key [.., 128] and window rows [.., 512] of sequences b at p."""
    return (values(seed, "lat", b, p, 512, device, sigma), values(seed, "lik", b, p, 128, device, sigma),
            values(seed, "lsw", b, p, 512, device, sigma))


def _gpu_cache(B, n, cap, swa_cap, seed, sigma=1.0, chunk=1024):
    c = csa.LatentCache(B, cap, swa_cap)
    ws = G.StatusWs(DEV)
    b = torch.arange(B, device=DEV)
    for p0 in range(0, n, chunk):
        t = min(chunk, n - p0)
        lat, ik, sw = _planes(seed, b, torch.arange(p0, p0 + t, device=DEV), DEV, sigma)
        csa.csa2_latent_append(c, B, t, torch.full((B,), p0, dtype=torch.int64, device=DEV), lat.contiguous(),
                               ik.contiguous(), sw.contiguous(), ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    return c


def _oracle_cache(b, n, cap, swa_cap, seed, sigma=1.0):
    oc = oracle.LatentCache(cap, swa_cap)
    for p0 in range(0, n, 4096):
        lat, ik, sw = _planes(seed, [b], torch.arange(p0, min(n, p0 + 4096)), "cpu", sigma)
        oc.append(p0, latent=lat[0], idx_k=ik[0], swa=sw[0])
    return oc


def _check(out, of, lse, ref_out, ref_lse, tol):
    assert torch.equal(out, of.to(torch.bfloat16))
    err = np.abs(of.double().cpu().numpy() - ref_out).max()
    assert err <= tol, err
    gl = lse.double().cpu().numpy()
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(gl), fin)
    if fin.any():
        assert np.abs(gl[fin] - ref_lse[fin]).max() <= tol


def test_latent_append_matches_oracle(orc):
    B, n, cap, swa_cap, seed = 2, 700, 1024, 256, 71
    c = _gpu_cache(B, n, cap, swa_cap, seed)
    for b in range(B):
        oc = _oracle_cache(b, n, cap, swa_cap, seed)
        assert np.array_equal(c.l_data[b, :n].cpu().numpy(), oc.ldata[:n])
        assert np.array_equal(c.l_scale[b, :n].cpu().numpy(), oc.lscale[:n])
        assert np.array_equal(c.k_data[b, :n].cpu().numpy(), oc.kdata[:n])
        assert np.array_equal(c.k_scale[b, :n].cpu().numpy(), oc.kscale[:n])
        assert np.array_equal(c.swa[b].cpu().numpy(), oc.swa)  # the ring wrapped: the last 256 tokens
        assert not c.l_data[b, n:].any()
    # an append that would run past the capacity: reported, and that sequence is left untouched
    ws = G.StatusWs(DEV)
    before = c.l_data.clone()
    lat, ik, _ = _planes(seed, torch.arange(B, device=DEV), torch.arange(cap - 1, cap + 1, device=DEV), DEV, 1.0)
    csa.csa2_latent_append(c, B, 2, torch.tensor([cap - 1, 0], dtype=torch.int64, device=DEV), lat.contiguous(),
                           ik.contiguous(), None, ws=ws)
    assert csa.csa2_get_device_status(ws) & csa.CSA2_DEV_BAD_POS
    assert torch.equal(c.l_data[0], before[0])
    assert not torch.equal(c.l_data[1, :2], before[1, :2])


@pytest.mark.parametrize("B,tq,n,k,sigma,swa_begin,ratio", [
    (3, 1, 2000, 512, 1.0, None, 1),
    (2, 1, 1500, 300, 8.0, None, 1),        # ragged last tile, peaked softmax
    (2, 1, 4300, 2048, 1.0, [4250, 0], 1),  # 16 selected tiles; sequence 0's window cut to 50 tokens
    (2, 2, 1200, 512, 1.0, None, 2),        # one entry per 2 tokens, two rows per sequence
    (1, 1, 900, 100, 1.0, None, 1),
])
def test_latent_attend_matches_oracle(orc, B, tq, n, k, sigma, swa_begin, ratio):
    seed = 101 + n + B + k
    cap, swa_cap = 1 << (n - 1).bit_length(), 256
    c = _gpu_cache(B, n, cap, swa_cap, seed, sigma)
    rows = B * tq
    # tokens below n: the window rows were appended for tokens 0..n-1 (with ratio 2 the first
    # (qpos + 1) / 2 entries are visible)
    qpos = [n - 1 - 3 * (r // tq) - 5 * (r % tq) for r in range(rows)]
    qp = torch.tensor(qpos, dtype=torch.int64, device=DEV)
    vis = min((p + 1) // ratio for p in qpos)
    q = values(seed, "lq", torch.arange(rows), qp.cpu().unsqueeze(1), 64 * 512, "cpu", sigma)[:, 0]
    q = q.reshape(rows, 64, 512).to(DEV).contiguous()
    nsel = min(k, vis - 8, k - k // 7)
    idx = W.distinct_sorted(seed, "sel", torch.arange(rows, device=DEV), vis - 4, nsel).to(torch.int32)
    idx = torch.cat([idx, torch.full((rows, k - nsel), -1, dtype=torch.int32, device=DEV)], 1)
    perm = torch.argsort(torch.rand(rows, k, generator=torch.Generator().manual_seed(seed)), dim=1).to(DEV)
    idx = torch.gather(idx, 1, perm).contiguous()  # any order, -1 anywhere
    sb = None if swa_begin is None else torch.tensor(swa_begin, dtype=torch.int64, device=DEV)
    out = torch.empty(rows, 64, 512, dtype=torch.bfloat16, device=DEV)
    of = torch.empty(rows, 64, 512, dtype=torch.float32, device=DEV)
    lse = torch.empty(rows, 64, dtype=torch.float32, device=DEV)
    ws = G.StatusWs(DEV)
    csa.csa2_latent_attend(c, B, tq, qp, q, idx, k, out, swa_begin=sb, win=128, ratio=ratio, out_f32=of, lse=lse,
                           ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    for r in range(rows):
        b = r // tq
        oc = _oracle_cache(b, n, cap, swa_cap, seed, sigma)
        ro, rl = oc.attend(qpos[r], q[r].cpu(), idx[r].cpu().numpy(), swa_begin=0 if sb is None else swa_begin[b],
                           win=128, ratio=ratio)
        _check(out[r], of[r], lse[r], ro, rl, attn_tol(None, sigma))


def test_latent_rescale_of_the_running_maximum(orc):
    """Latent rows L_p = g(p) v + noise with g growing by tile and queries q_h = c_h v: the logits of
    head h grow by about 9.8 c_h (log2 units) per 128-key tile. Heads with c_h > 0.82 exceed the
    running maximum by more than 8 at every tile (rescale of the accumulated output in tensor memory),
    heads with smaller c_h creep up below the threshold (probabilities up to 2^8 before one rescale),
    heads with c_h < 0 peak in the first tile."""
    n, cap, swa_cap, seed = 640, 1024, 128, 977
    p = torch.arange(n)
    v = values(seed, "lat", [0], [n], 512, "cpu")[0, 0].float()  # a direction not used as a row
    noise = values(seed, "lsw", [0], p, 512, "cpu")[0].float()
    g = 0.3 * (p // 128).float()
    rows = (g[:, None] * v[None, :] + 0.25 * noise).to(torch.bfloat16)
    ch = torch.linspace(-1.0, 1.4, 64)
    q = (ch[:, None] * v[None, :]).to(torch.bfloat16).reshape(1, 64, 512)
    c = csa.LatentCache(1, cap, swa_cap)
    ws = G.StatusWs(DEV)
    zero = torch.zeros(1, dtype=torch.int64, device=DEV)
    csa.csa2_latent_append(c, 1, 512, zero, latent=rows[:512].reshape(1, 512, 512).to(DEV).contiguous(), ws=ws)
    csa.csa2_latent_append(c, 1, 128, zero + 512, swa=rows[512:].reshape(1, 128, 512).to(DEV).contiguous(), ws=ws)
    oc = oracle.LatentCache(cap, swa_cap)
    oc.append(0, latent=rows[:512])
    oc.append(512, swa=rows[512:])
    idx = torch.arange(512, dtype=torch.int32).reshape(1, 512)
    qp = torch.tensor([n - 1], dtype=torch.int64, device=DEV)
    out = torch.empty(1, 64, 512, dtype=torch.bfloat16, device=DEV)
    of = torch.empty(1, 64, 512, dtype=torch.float32, device=DEV)
    lse = torch.empty(1, 64, dtype=torch.float32, device=DEV)
    csa.csa2_latent_attend(c, 1, 1, qp, q.to(DEV).contiguous(), idx.to(DEV), 512, out, win=128, out_f32=of, lse=lse,
                           ws=ws)
    assert csa.csa2_get_device_status(ws) == 0
    ro, rl = oc.attend(n - 1, q[0], idx[0].numpy(), win=128)
    # the rows reach |L| ~ 5: the fp16 probability rounding bounds the error by 2^-11 max|L|
    _check(out[0], of[0], lse[0], ro, rl, 4e-3)
    # the heads that rescale put almost all weight on the window tile, the others spread it
    assert np.abs(rl[-1] - rl[0]) > 10


def test_latent_window_only_empty_row_and_bad_index(orc):
    n, cap, swa_cap, seed, k = 1000, 1024, 128, 55, 256
    B = 4
    c = _gpu_cache(B, n, cap, swa_cap, seed)
    qpos = [n - 1, -1, n - 11, n - 1]
    qp = torch.tensor(qpos, dtype=torch.int64, device=DEV)
    sb = torch.tensor([0, 0, 0, n], dtype=torch.int64, device=DEV)  # sequence 3: no window token
    q = values(seed, "lq", torch.arange(B), torch.tensor([[max(x, 0)] for x in qpos]), 64 * 512, "cpu")[:, 0]
    q = q.reshape(B, 64, 512).to(DEV).contiguous()
    idx = W.distinct_sorted(seed, "sel", torch.arange(B, device=DEV), n - 20, k).to(torch.int32)
    idx[0] = -1                       # window only
    idx[2, 5] = qpos[2] + 3           # not visible yet: reported and skipped
    idx = idx.contiguous()
    out = torch.empty(B, 64, 512, dtype=torch.bfloat16, device=DEV)
    of = torch.empty(B, 64, 512, dtype=torch.float32, device=DEV)
    lse = torch.empty(B, 64, dtype=torch.float32, device=DEV)
    ws = G.StatusWs(DEV)
    csa.csa2_latent_attend(c, B, 1, qp, q, idx, k, out, swa_begin=sb, win=128, out_f32=of, lse=lse, ws=ws)
    assert csa.csa2_get_device_status(ws) == csa.CSA2_DEV_BAD_INDEX
    assert not of[1].any() and torch.isinf(lse[1]).all() and (lse[1] < 0).all()
    for r in (0, 2, 3):
        oc = _oracle_cache(r, n, cap, swa_cap, seed)
        ir = idx[r].cpu().numpy().copy()
        ir[ir > qpos[r]] = -1
        ro, rl = oc.attend(qpos[r], q[r].cpu(), ir, swa_begin=int(sb[r]), win=128)
        _check(out[r], of[r], lse[r], ro, rl, attn_tol(None))


def test_latent_workload_full_size_every_sequence(orc):
    """128 sequences at N = 131,072 (the selected rows and the window filled, as bench.py builds it),
    one decode row each, in bench.py's launch configuration; every sequence against the oracle."""
    name = "latent_b128_n131072"
    step = G.build(name)
    of = torch.empty(step.batch, 64, 512, dtype=torch.float32, device=DEV)
    lse = torch.empty(step.batch, 64, dtype=torch.float32, device=DEV)
    step.run(out_f32=of, lse=lse)
    assert csa.csa2_get_device_status(step.ws) == 0
    ref = oracle_steps(name, list(range(step.batch)))
    for b in range(step.batch):
        assert np.array_equal(step.inputs["idx"][b].cpu().numpy(), ref[b]["idx"])
        _check(step.outputs["out"][b], of[b], lse[b], ref[b]["out"], ref[b]["lse"], attn_tol(None))
    prev = step.outputs["out"].clone()
    step.run()
    assert torch.equal(step.outputs["out"], prev)
    del step
    torch.cuda.empty_cache()
