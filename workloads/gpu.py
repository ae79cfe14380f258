"""Builds the workloads on a GPU through libcsa2's C ABI (bench.py and the full-size parity
tests use it). Inputs come from the seeded generator in workloads/__init__.py, made on the device;
the cache is filled with libcsa2's own quantise-append. Only the positions a step can read are
filled (a Reindex step reads only its pool, a Minimal step only its inherited rows); the rest of
each allocated plane stays zero.
"""
from __future__ import annotations

import dataclasses

import torch

import compressed_sparse_attention_append_b200 as csa
from . import WORKLOADS, Workload, cache_values, distinct_sorted


def _vals(seed, stream, b, p, width):
    return cache_values(seed, stream, b, p, width)


@dataclasses.dataclass
class Step:
    wl: Workload
    shape: object
    cache: csa.Cache
    ws: csa.Workspace
    inputs: dict            # per-step device inputs
    outputs: dict           # per-step device outputs
    batch: int
    max_ctx: int

    # ---- one pass of the hot path, through the composed entry point ----
    def run(self, stream=None, ws=None, out_f32=None, lse=None):
        wl, I, O = self.wl, self.inputs, self.outputs
        ws = ws or self.ws
        if wl.mode == "full":
            csa.csa2_decode_full(self.shape, self.cache, self.batch, I["qpos"], I["kv"], I["idx_k"], I["swa_kv"],
                                 I["idx_q"], I["q"], wl.k, O["idx"], O["out"], pool_blocks=wl.pool_blocks,
                                 out_pool=O.get("pool"), out_pool_n=O.get("pool_n"), max_ctx=self.max_ctx,
                                 out_f32=out_f32, lse=lse, ws=ws, stream=stream)
        elif wl.mode == "reindex":
            csa.csa2_decode_reindex(self.shape, self.cache, self.batch, I["qpos"], I["swa_kv"], I["idx_q"], I["q"],
                                    I["pool"], I["pool_n"], wl.k, O["idx"], O["out"], out_f32=out_f32, lse=lse,
                                    ws=ws, stream=stream)
        elif wl.mode == "minimal":
            csa.csa2_decode_minimal(self.shape, self.cache, self.batch, I["qpos"], I["swa_kv"], I["q"], I["idx"],
                                    wl.k, O["out"], out_f32=out_f32, lse=lse, ws=ws, stream=stream)
        elif wl.mode == "draft":
            self._draft(lambda n, ph: None, stream, ws, out_f32, lse)
        else:
            csa.csa2_prefill_chunk(self.shape, self.cache, wl.context - wl.tq, wl.tq, I["kv"], I["idx_k"],
                                   I["swa_kv"], I["idx_q"], I["q"], wl.k, O["idx"], O["out"], out_f32=out_f32,
                                   lse=lse, ws=ws, stream=stream)

    def _draft(self, hooks, stream, ws, out_f32=None, lse=None):
        """Multi-token decode: append the tq draft tokens, index tq rows, attend tq rows (there is no
        composed entry point for tq > 1: these are the three calls a user makes)."""
        wl, I, O, b, t = self.wl, self.inputs, self.outputs, self.batch, self.wl.tq
        hooks("append", 0)
        csa.csa2_quantize_append(self.shape, self.cache, b, t, I["pos"], I["kv"], I["idx_k"], I["swa_kv"], ws=ws,
                                 stream=stream)
        hooks("append", 1)
        hooks("index", 0)
        csa.csa2_index_topk_full(self.shape, self.cache, b, t, I["qpos"], I["idx_q"], wl.k, O["idx"],
                                 max_ctx=self.max_ctx, ws=ws, stream=stream)
        hooks("index", 1)
        hooks("attend", 0)
        csa.csa2_sparse_attend(self.shape, self.cache, b, t, I["qpos"], I["q"], O["idx"], wl.k, O["out"],
                               out_f32=out_f32, lse=lse, ws=ws, stream=stream)
        hooks("attend", 1)

    def _prefill_parts(self, hooks, stream):
        """The prefill chunk as the three calls csa2_prefill_chunk makes: append the chunk at
        p0 = context - tq, index its tq rows (row i at position p0 + i), attend them."""
        wl, I, O, t = self.wl, self.inputs, self.outputs, self.wl.tq
        p0 = wl.context - t
        dev = I["idx_q"].device
        if not hasattr(self, "_pp"):
            self._pp = (torch.full((1,), p0, dtype=torch.int64, device=dev),
                        torch.arange(p0, wl.context, dtype=torch.int64, device=dev))
        pos, qpos = self._pp
        hooks("append", 0)
        csa.csa2_quantize_append(self.shape, self.cache, 1, t, pos, I["kv"], I["idx_k"], I["swa_kv"], ws=self.ws,
                                 stream=stream)
        hooks("append", 1)
        hooks("index", 0)
        csa.csa2_index_topk_full(self.shape, self.cache, 1, t, qpos, I["idx_q"], wl.k, O["idx"], max_ctx=wl.context,
                                 ws=self.ws, stream=stream)
        hooks("index", 1)
        hooks("attend", 0)
        csa.csa2_sparse_attend(self.shape, self.cache, 1, t, qpos, I["q"], O["idx"], wl.k, O["out"], ws=self.ws,
                               stream=stream)
        hooks("attend", 1)

    # ---- the same pass as separate entry points (kernel-level timing) ----
    def run_parts(self, hooks, stream=None):
        """hooks(name) is called before and after each kernel's entry point: ('append'|'index'|'attend')."""
        wl, I, O = self.wl, self.inputs, self.outputs
        b = self.batch
        if wl.mode == "prefill":
            return self._prefill_parts(hooks, stream)
        if wl.mode == "draft":
            return self._draft(hooks, stream, self.ws)
        hooks("append", 0)
        if wl.mode == "full":
            csa.csa2_quantize_append(self.shape, self.cache, b, 1, I["qpos"], I["kv"], I["idx_k"], I["swa_kv"],
                                     ws=self.ws, stream=stream)
        else:
            csa.csa2_quantize_append(self.shape, self.cache, b, 1, I["qpos"], None, None, I["swa_kv"], ws=self.ws,
                                     stream=stream)
        hooks("append", 1)
        idx = I.get("idx")
        if wl.mode in ("full", "reindex"):
            hooks("index", 0)
            if wl.mode == "full":
                csa.csa2_index_topk_full(self.shape, self.cache, b, 1, I["qpos"], I["idx_q"], wl.k, O["idx"],
                                         wl.pool_blocks, O.get("pool"), O.get("pool_n"), max_ctx=self.max_ctx,
                                         ws=self.ws, stream=stream)
            else:
                csa.csa2_index_topk_reindex(self.shape, self.cache, b, I["qpos"], I["idx_q"], I["pool"], I["pool_n"],
                                            wl.k, O["idx"], ws=self.ws, stream=stream)
            hooks("index", 1)
            idx = O["idx"]
        hooks("attend", 0)
        csa.csa2_sparse_attend(self.shape, self.cache, b, 1, I["qpos"], I["q"], idx, wl.k, O["out"], ws=self.ws,
                               stream=stream)
        hooks("attend", 1)


class StatusWs:
    """The 256-byte workspace csa2_latent_attend / csa2_latent_append take (its status word)."""

    def __init__(self, device):
        self.buf = torch.zeros(256, dtype=torch.uint8, device=device)

    @property
    def ptr(self):
        return self.buf.data_ptr()

    @property
    def nbytes(self):
        return self.buf.numel()


@dataclasses.dataclass
class LatentStep:
    """A decode row per sequence in the pages' own attention shape (64 heads x 512 over the
    512-channel latent, K = V): one csa2_latent_attend call per step."""
    wl: Workload
    cache: csa.LatentCache
    ws: StatusWs
    inputs: dict
    outputs: dict
    batch: int

    def run(self, stream=None, ws=None, out_f32=None, lse=None):
        I, O = self.inputs, self.outputs
        csa.csa2_latent_attend(self.cache, self.batch, 1, I["qpos"], I["q"], I["idx"], self.wl.k, O["out"],
                               win=self.wl.win, out_f32=out_f32, lse=lse, ws=ws or self.ws, stream=stream)

    def run_parts(self, hooks, stream=None):
        hooks("attend", 0)
        self.run(stream)
        hooks("attend", 1)


def _build_latent(wl, seqs, B, device):
    N = wl.context
    cache = csa.LatentCache(B, N, 128, device=device, indexer=False)
    ws = StatusWs(device)
    idx = distinct_sorted(wl.seed, "sel", seqs, N - 1, wl.k).to(torch.int32).contiguous()
    lat = _vals(wl.seed, "lat", seqs, idx.to(torch.int64), 512)
    for j in range(wl.k):  # the selected rows only: the step reads nothing else of the latent plane
        csa.csa2_latent_append(cache, B, 1, idx[:, j].to(torch.int64).contiguous(), latent=lat[:, j:j + 1].contiguous(),
                               ws=ws)
    pw = torch.arange(N - wl.win, N, device=device)
    csa.csa2_latent_append(cache, B, wl.win, torch.full((B,), N - wl.win, dtype=torch.int64, device=device),
                           swa=_vals(wl.seed, "lsw", seqs, pw, 512).contiguous(), ws=ws)
    qpos = torch.full((B,), N - 1, dtype=torch.int64, device=device)
    q = _vals(wl.seed, "lq", seqs, qpos.unsqueeze(1), 64 * 512)[:, 0].reshape(B, 64, 512).contiguous()
    out = torch.empty(B, 64, 512, dtype=torch.bfloat16, device=device)
    torch.cuda.synchronize()
    return LatentStep(wl, cache, ws, {"qpos": qpos, "q": q, "idx": idx}, {"out": out}, B)


@dataclasses.dataclass
class LatentIndexStep:
    """A decode row per sequence scored by the indexer of the pages' own shape (32 heads x 128 over
    one MXFP4 key per entry, ReLU scores) against every visible entry: one csa2_latent_index_topk."""
    wl: Workload
    cache: csa.LatentCache
    ws: csa.LatentIndexWorkspace
    inputs: dict
    outputs: dict
    batch: int

    def run(self, stream=None, ws=None, out_f32=None, lse=None):
        I, O = self.inputs, self.outputs
        csa.csa2_latent_index_topk(self.cache, self.batch, 1, I["qpos"], I["idx_q"], self.wl.k, O["idx"], ws or self.ws,
                                   max_ctx=self.wl.context, flags=csa.CSA2_SCORE_RELU, stream=stream)

    def run_parts(self, hooks, stream=None):
        hooks("index", 0)
        self.run(stream)
        hooks("index", 1)


def _build_latent_index(wl, seqs, B, device, chunk=4096):
    N = wl.context
    cache = csa.LatentCache(B, N, 128, device=device, latent=False)
    st = StatusWs(device)
    for p0 in range(0, N, chunk):  # every position: the step scans them all
        t = min(chunk, N - p0)
        p = torch.arange(p0, p0 + t, device=device)
        csa.csa2_latent_append(cache, B, t, torch.full((B,), p0, dtype=torch.int64, device=device),
                               idx_k=_vals(wl.seed, "lik", seqs, p, 128).contiguous(), ws=st)
    qpos = torch.full((B,), N - 1, dtype=torch.int64, device=device)
    iq = _vals(wl.seed, "liq", seqs, qpos.unsqueeze(1), wl.hi * 128)[:, 0].reshape(B, wl.hi, 128).contiguous()
    out = torch.empty(B, wl.k, dtype=torch.int32, device=device)
    ws = csa.LatentIndexWorkspace(B, wl.hi, N, device=device)
    torch.cuda.synchronize()
    return LatentIndexStep(wl, cache, ws, {"qpos": qpos, "idx_q": iq}, {"idx": out}, B)


def build(name: str, batch: int | None = None, seq_offset: int = 0, device="cuda", context=None) -> Step:
    """Allocate and fill the cache of workload `name` (optionally a smaller batch, or the sequences
    seq_offset .. seq_offset+batch-1 of it, as a data-parallel rank would; optionally another context
    length, for profiling small cases) and its step inputs."""
    wl = WORKLOADS[name]
    if context:
        wl = dataclasses.replace(wl, context=context)
    B = wl.batch if batch is None else batch
    seqs = torch.arange(seq_offset, seq_offset + B, device=device)
    if wl.mode == "latent":
        return _build_latent(wl, seqs, B, device)
    if wl.mode == "latent_index":
        return _build_latent_index(wl, seqs, B, device)
    shape = csa.make_shape(wl.win)
    N = wl.context
    I, O = {}, {}
    if wl.mode == "prefill":
        p0 = N - wl.tq
        cache = csa.Cache(B, N, 1 << (wl.tq + wl.win - 1).bit_length(), device=device)
        _fill_range(cache, shape, wl.seed, seqs, 0, p0, device)
        p = torch.arange(p0, N, device=device)
        I["kv"] = _vals(wl.seed, "kv", seqs, p, 256)[0].contiguous()
        I["idx_k"] = _vals(wl.seed, "ik", seqs, p, 256)[0].contiguous()
        I["swa_kv"] = _vals(wl.seed, "swa", seqs, p, 256)[0].contiguous()
        I["idx_q"] = _vals(wl.seed, "iq", seqs, p, 256)[0].contiguous()
        I["q"] = _vals(wl.seed, "q", seqs, p, 2048)[0].reshape(wl.tq, 16, 128).contiguous()
        O["idx"] = torch.empty(wl.tq, wl.k, dtype=torch.int32, device=device)
        O["out"] = torch.empty(wl.tq, 16, 128, dtype=torch.bfloat16, device=device)
        ws = csa.Workspace(shape, 1, wl.tq, wl.k, N)
        return Step(wl, shape, cache, ws, I, O, 1, N)

    if wl.mode == "draft":
        T = wl.tq
        p0 = N - T
        cache = csa.Cache(B, N, 1 << (T + wl.win - 1).bit_length(), device=device)
        _fill_range(cache, shape, wl.seed, seqs, 0, p0, device)
        p = torch.arange(p0, N, device=device)
        I["pos"] = torch.full((B,), p0, dtype=torch.int64, device=device)
        I["qpos"] = p.unsqueeze(0).repeat(B, 1).contiguous()
        I["kv"] = _vals(wl.seed, "kv", seqs, p, 256).contiguous()
        I["idx_k"] = _vals(wl.seed, "ik", seqs, p, 256).contiguous()
        I["swa_kv"] = _vals(wl.seed, "swa", seqs, p, 256).contiguous()
        I["idx_q"] = _vals(wl.seed, "iq", seqs, p, 256).contiguous()
        I["q"] = _vals(wl.seed, "q", seqs, p, 2048).reshape(B, T, 16, 128).contiguous()
        O["idx"] = torch.empty(B, T, wl.k, dtype=torch.int32, device=device)
        O["out"] = torch.empty(B, T, 16, 128, dtype=torch.bfloat16, device=device)
        ws = csa.Workspace(shape, B, T, wl.k, N)
        torch.cuda.synchronize()
        return Step(wl, shape, cache, ws, I, O, B, N)

    qpos = torch.full((B,), N - 1, dtype=torch.int64, device=device)
    I["qpos"] = qpos
    qp = qpos.unsqueeze(1)
    I["swa_kv"] = _vals(wl.seed, "swa", seqs, qp, 256)[:, 0].contiguous()
    I["q"] = _vals(wl.seed, "q", seqs, qp, 2048)[:, 0].reshape(B, 16, 128).contiguous()
    O["out"] = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=device)
    if wl.mode != "minimal":
        I["idx_q"] = _vals(wl.seed, "iq", seqs, qp, 256)[:, 0].contiguous()
        O["idx"] = torch.empty(B, wl.k, dtype=torch.int32, device=device)
    if wl.mode == "full":
        cache = csa.Cache(B, N, 128, device=device)
        _fill_range(cache, shape, wl.seed, seqs, 0, N - 1, device)
        I["kv"] = _vals(wl.seed, "kv", seqs, qp, 256)[:, 0].contiguous()
        I["idx_k"] = _vals(wl.seed, "ik", seqs, qp, 256)[:, 0].contiguous()
        if wl.pool_blocks:
            O["pool"] = torch.empty(B, wl.pool_blocks, dtype=torch.int32, device=device)
            O["pool_n"] = torch.empty(B, dtype=torch.int32, device=device)
        ws = csa.Workspace(shape, B, 1, wl.k, N, wl.pool_blocks)
    elif wl.mode == "reindex":
        cache = csa.Cache(B, N, 128, device=device)
        nblk = N // wl.bs
        pool = distinct_sorted(wl.seed, "pool", seqs, nblk, wl.pool_blocks).to(torch.int32).contiguous()
        I["pool"] = pool
        I["pool_n"] = torch.full((B,), wl.pool_blocks, dtype=torch.int32, device=device)
        _fill_blocks(cache, shape, wl.seed, seqs, pool, wl.bs, device)
        _fill_window(cache, shape, wl.seed, seqs, N - wl.win, N - 1, device)
        ws = csa.Workspace(shape, B, 1, wl.k, wl.pool_blocks * wl.bs)
    else:  # minimal
        cache = csa.Cache(B, N, 128, device=device, indexer=False)
        idx = distinct_sorted(wl.seed, "sel", seqs, N - 1, wl.k).to(torch.int32).contiguous()
        I["idx"] = idx
        _fill_rows(cache, shape, wl.seed, seqs, idx, device)
        _fill_window(cache, shape, wl.seed, seqs, N - wl.win, N - 1, device)
        ws = csa.Workspace(shape, B, 1, wl.k, 8)
    torch.cuda.synchronize()
    return Step(wl, shape, cache, ws, I, O, B, N)


def _fill_range(cache, shape, seed, seqs, p0, p1, device, chunk=2048):
    B = seqs.numel()
    for a in range(p0, p1, chunk):
        t = min(chunk, p1 - a)
        p = torch.arange(a, a + t, device=device)
        pos = torch.full((B,), a, dtype=torch.int64, device=device)
        kv = _vals(seed, "kv", seqs, p, 256).contiguous()
        ik = _vals(seed, "ik", seqs, p, 256).contiguous() if cache.ik_data is not None else None
        sw = _vals(seed, "swa", seqs, p, 256).contiguous()
        csa.csa2_quantize_append(shape, cache, B, t, pos, kv, ik, sw)


def _fill_window(cache, shape, seed, seqs, p0, p1, device):
    B = seqs.numel()
    p = torch.arange(p0, p1, device=device)
    pos = torch.full((B,), p0, dtype=torch.int64, device=device)
    sw = _vals(seed, "swa", seqs, p, 256).contiguous()
    csa.csa2_quantize_append(shape, cache, B, p1 - p0, pos, None, None, sw)


def _fill_blocks(cache, shape, seed, seqs, pool, bs, device, group=125):
    B, P = pool.shape
    off = torch.arange(bs, device=device)
    for g0 in range(0, P, group):
        g1 = min(P, g0 + group)
        p = (pool[:, g0:g1].to(torch.int64).unsqueeze(-1) * bs + off).reshape(B, -1)
        kv = _vals(seed, "kv", seqs, p, 256)
        ik = _vals(seed, "ik", seqs, p, 256)
        for j in range(g1 - g0):
            pos = pool[:, g0 + j].to(torch.int64) * bs
            csa.csa2_quantize_append(shape, cache, B, bs, pos, kv[:, j * bs:(j + 1) * bs].contiguous(),
                                     ik[:, j * bs:(j + 1) * bs].contiguous(), None)


def _fill_rows(cache, shape, seed, seqs, idx, device):
    B, K = idx.shape
    p = idx.to(torch.int64)
    kv = _vals(seed, "kv", seqs, p, 256)
    for j in range(K):
        csa.csa2_quantize_append(shape, cache, B, 1, p[:, j].contiguous(), kv[:, j:j + 1].contiguous(), None, None)
