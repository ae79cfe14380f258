"""Thin Python binding of libcsa2 (include/csa2.h): argument marshalling only.

Every function below has the name of the C entry point it calls, takes torch tensors where the C
call takes device pointers, passes the current CUDA stream, and raises Csa2Error on a non-zero
status. No step of the CSA2 layer runs here: quantise-append, scoring, Top-k, pool, gather,
dequantisation and attention all run in the CUDA kernels of libcsa2.so. There is no CPU
fallback: if the library is not built, loading fails loudly.

Plumbing helpers (`Cache`, `Workspace`) allocate device memory with torch and fill the C structs.

A Reindex decode step for a batch of B sequences (tensors on the GPU, bf16 unless noted):

    shape = make_shape()                                  # 16 x 128 heads, indexer 4 x 64, window 128
    cache = Cache(B, cap, swa_cap)                        # FP4 main / indexer planes + FP8 window ring
    ws = Workspace(shape, B, 1, 512, pool_stride * 8)     # sized for the largest pool
    csa2_quantize_append(shape, cache, B, t, pos, kv, idx_k, swa_kv)     # new entries (any plane may be None)
    csa2_decode_reindex(shape, cache, B, qpos, swa_kv, idx_q, q, pool, pool_n, 512, idx, out, ws=ws)
    status = csa2_get_device_status(ws)                   # bad indices / positions / pool ids, if any

`out` [B, 16, 128] holds the attention output, `idx` [B, 512] the selected positions (ascending,
-1 padded). The Full and Minimal modes, the separate index / attention calls and the prefill chunk
follow the same pattern (include/csa2.h documents every argument).

The pages' own shapes use a `LatentCache` (one 512-channel latent per entry that is both key and
value, a 128-channel MXFP4 indexer key, 512-channel FP8 window rows):

    lc = LatentCache(B, cap, swa_cap)
    csa2_latent_append(lc, B, t, pos, latent, idx_k, swa)                 # any plane may be None
    ws = LatentIndexWorkspace(B, 32, cap)
    csa2_latent_index_topk(lc, B, 1, qpos, idx_q, 512, idx, ws, flags=CSA2_SCORE_RELU)   # 32 x 128 heads
    csa2_latent_attend(lc, B, 1, qpos, q, idx, 512, out)                 # 64 heads x 512, tensor cores
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

CSA2_OK = 0
CSA2_ERR_INVALID_ARG = 1
CSA2_ERR_UNSUPPORTED_SHAPE = 2
CSA2_ERR_CAPACITY = 3
CSA2_ERR_WORKSPACE = 4
CSA2_ERR_CUDA = 5
CSA2_ERR_DEVICE = 6
CSA2_DEV_BAD_INDEX = 0x1
CSA2_DEV_BAD_POS = 0x2
CSA2_DEV_BAD_POOL = 0x4
CSA2_DEV_TIMEOUT = 0x8
CSA2_SCORE_RELU = 0x1

EXPORTS = (
    "csa2_entry_bytes", "csa2_status_string", "csa2_version", "csa2_workspace_size", "csa2_workspace_init",
    "csa2_quantize_append", "csa2_index_topk_full", "csa2_index_topk_reindex", "csa2_sparse_attend",
    "csa2_decode_full", "csa2_decode_reindex", "csa2_decode_minimal", "csa2_prefill_chunk",
    "csa2_get_device_status", "csa2_sparse_attend_noalloc", "csa2_mx_entry_bytes", "csa2_mxfp4_quantize",
    "csa2_latent_append", "csa2_latent_attend", "csa2_latent_index_workspace_size", "csa2_latent_index_topk",
)


class Csa2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_string(status)} (status {status})")
        self.status = status


class csa2_shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("hq", "d", "hi", "di", "hk", "win", "bs", "ratio")]


class csa2_cache(ctypes.Structure):
    _fields_ = [
        ("kv_data", ctypes.c_void_p), ("kv_scale", ctypes.c_void_p), ("ik_data", ctypes.c_void_p),
        ("ik_scale", ctypes.c_void_p), ("swa", ctypes.c_void_p), ("cap", ctypes.c_int64),
        ("swa_cap", ctypes.c_int64),
    ]


class csa2_latent_cache(ctypes.Structure):
    _fields_ = [
        ("l_data", ctypes.c_void_p), ("l_scale", ctypes.c_void_p), ("k_data", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p), ("swa", ctypes.c_void_p), ("cap", ctypes.c_int64),
        ("swa_cap", ctypes.c_int64),
    ]


_lib = None


def lib():
    """Load libcsa2.so (built in-tree by build.py). Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libcsa2.so is not built at {LIB_PATH}; run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, i64, u32, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint32, ctypes.c_float, ctypes.c_size_t
        S, C = ctypes.POINTER(csa2_shape), ctypes.POINTER(csa2_cache)
        LC = ctypes.POINTER(csa2_latent_cache)
        sig = {
            "csa2_entry_bytes": (sz, [i]),
            "csa2_status_string": (ctypes.c_char_p, [i]),
            "csa2_version": (i, []),
            "csa2_workspace_size": (i, [S, i, i, i, i64, i, ctypes.POINTER(sz)]),
            "csa2_workspace_init": (i, [vp, sz, vp]),
            "csa2_quantize_append": (i, [S, C, i, i, vp, vp, vp, vp, vp, sz, vp]),
            "csa2_index_topk_full": (i, [S, C, i, i, vp, vp, i, vp, i, vp, vp, i64, u32, vp, sz, vp]),
            "csa2_index_topk_reindex": (i, [S, C, i, vp, vp, vp, vp, i, i, vp, u32, vp, sz, vp]),
            "csa2_sparse_attend": (i, [S, C, i, i, vp, vp, vp, i, vp, f, vp, vp, vp, vp, sz, vp]),
            "csa2_decode_full": (i, [S, C, i, vp, vp, vp, vp, vp, vp, i, vp, i, vp, vp, i64, vp, f, vp, vp, vp, u32, vp, sz, vp]),
            "csa2_decode_reindex": (i, [S, C, i, vp, vp, vp, vp, vp, vp, i, i, vp, vp, f, vp, vp, vp, u32, vp, sz, vp]),
            "csa2_decode_minimal": (i, [S, C, i, vp, vp, vp, vp, i, vp, f, vp, vp, vp, vp, sz, vp]),
            "csa2_prefill_chunk": (i, [S, C, i64, i, vp, vp, vp, vp, vp, i, vp, i64, f, vp, vp, vp, u32, vp, sz, vp]),
            "csa2_get_device_status": (i, [vp, vp, ctypes.POINTER(ctypes.c_int32)]),
            "csa2_sparse_attend_noalloc": (i, [S, C, i, i, vp, vp, vp, i, vp, f, vp, vp, vp, vp]),
            "csa2_mx_entry_bytes": (sz, [i]),
            "csa2_mxfp4_quantize": (i, [vp, i64, i, vp, vp, vp]),
            "csa2_latent_append": (i, [LC, i, i, vp, vp, vp, vp, vp, sz, vp]),
            "csa2_latent_attend": (i, [LC, i, i, vp, vp, vp, i, vp, i, i, f, vp, vp, vp, vp, sz, vp]),
            "csa2_latent_index_workspace_size": (i, [i, i, i64, ctypes.POINTER(sz)]),
            "csa2_latent_index_topk": (i, [LC, i, i, vp, vp, i, i, i, i64, u32, vp, vp, sz, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().csa2_status_string(int(s)).decode()


def _check(fn: str, s: int) -> int:
    if s != CSA2_OK:
        raise Csa2Error(fn, s)
    return s


def _p(t):
    if t is None:
        return None
    assert isinstance(t, torch.Tensor) and t.is_cuda and t.is_contiguous(), "expected a contiguous CUDA tensor"
    return t.data_ptr()


def _typed(t, dtype):
    if t is None:
        return None
    assert isinstance(t, torch.Tensor) and t.dtype == dtype, f"expected a {dtype} tensor"
    return _p(t)


def _i64(t):
    """int64 arrays of include/csa2.h (positions): pointer only, after a dtype check."""
    return _typed(t, torch.int64)


def _i32(t):
    """int32 arrays of include/csa2.h (indices, pools, counts): pointer only, after a dtype check."""
    return _typed(t, torch.int32)


def _f32(t):
    """fp32 outputs of include/csa2.h (out_f32, lse): pointer only, after a dtype check."""
    return _typed(t, torch.float32)


def _u8(t):
    """byte outputs (codes, E8M0 scales): pointer only, after a dtype check."""
    return _typed(t, torch.uint8)


def _bits(t):
    """bf16 tensors travel as their 16-bit patterns; pointer only."""
    if t is None:
        return None
    assert t.dtype == torch.bfloat16, "expected bf16"
    return _p(t)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_shape(win: int = 128, ratio: int = 1) -> csa2_shape:
    return csa2_shape(hq=16, d=128, hi=4, di=64, hk=4, win=win, bs=8, ratio=ratio)


class Cache:
    """Cache planes of `batch` sequences in the layout of include/csa2.h, allocated with torch."""

    def __init__(self, batch: int, cap: int, swa_cap: int = 128, device="cuda", main=True, indexer=True):
        assert swa_cap & (swa_cap - 1) == 0
        self.batch, self.cap, self.swa_cap = batch, cap, swa_cap
        z = lambda *s: torch.zeros(*s, dtype=torch.uint8, device=device)
        self.kv_data = z(batch, cap, 128) if main else None
        self.kv_scale = z(batch, cap, 16) if main else None
        self.ik_data = z(batch, cap, 128) if indexer else None
        self.ik_scale = z(batch, cap, 16) if indexer else None
        self.swa = z(batch, swa_cap, 256)
        self.c = csa2_cache(_p(self.kv_data), _p(self.kv_scale), _p(self.ik_data), _p(self.ik_scale),
                            _p(self.swa), cap, swa_cap)

    @property
    def ref(self):
        return ctypes.byref(self.c)


class LatentCache:
    """Cache planes of the pages' own shape (include/csa2.h, csa2_latent_cache) for `batch`
    sequences: the 512-channel latent (E2M1 + E4M3 per 16), the 128-channel MXFP4 indexer key and
    a ring of 512-channel E4M3 window rows, allocated with torch."""

    def __init__(self, batch: int, cap: int, swa_cap: int = 128, device="cuda", indexer=True, latent=True):
        assert swa_cap & (swa_cap - 1) == 0
        self.batch, self.cap, self.swa_cap = batch, cap, swa_cap
        z = lambda *s: torch.zeros(*s, dtype=torch.uint8, device=device)
        self.l_data = z(batch, cap, 256) if latent else None
        self.l_scale = z(batch, cap, 32) if latent else None
        self.k_data = z(batch, cap, 64) if indexer else None
        self.k_scale = z(batch, cap, 4) if indexer else None
        self.swa = z(batch, swa_cap, 512)
        self.c = csa2_latent_cache(_p(self.l_data), _p(self.l_scale), _p(self.k_data), _p(self.k_scale),
                                   _p(self.swa), cap, swa_cap)

    @property
    def ref(self):
        return ctypes.byref(self.c)


def csa2_latent_append(cache: LatentCache, batch, t, pos, latent=None, idx_k=None, swa=None, ws=None, stream=None):
    """latent [B, t, 512], idx_k [B, t, 128], swa [B, t, 512] bf16 (any may be None) at pos [B] int64."""
    _check("csa2_latent_append", lib().csa2_latent_append(
        cache.ref, batch, t, _i64(pos), _bits(latent), _bits(idx_k), _bits(swa), ws.ptr if ws else None,
        ws.nbytes if ws else 0, _stream(stream)))


def csa2_latent_attend(cache: LatentCache, batch, tq, qpos, q, idx, k, out, swa_begin=None, win=128, ratio=1,
                       sm_scale=0.0, out_f32=None, lse=None, ws=None, stream=None):
    """q [B*tq, 64, 512] bf16, idx [B*tq, k] int32 -> out [B*tq, 64, 512] bf16 (tensor cores)."""
    _check("csa2_latent_attend", lib().csa2_latent_attend(
        cache.ref, batch, tq, _i64(qpos), _bits(q), _i32(idx), k, _i64(swa_begin), win, ratio, sm_scale, _bits(out),
        _f32(out_f32), _f32(lse), ws.ptr if ws else None, ws.nbytes if ws else 0, _stream(stream)))


def csa2_latent_index_workspace_size(rows, hi, max_ctx) -> int:
    out = ctypes.c_size_t(0)
    _check("csa2_latent_index_workspace_size",
           lib().csa2_latent_index_workspace_size(rows, hi, max_ctx, ctypes.byref(out)))
    return out.value


class LatentIndexWorkspace:
    """Workspace of csa2_latent_index_topk for `rows` query rows of `hi` heads and at most `max_ctx`
    visible entries per row (zeroed: its first word is the status word)."""

    def __init__(self, rows, hi, max_ctx, device="cuda"):
        self.buf = torch.zeros(csa2_latent_index_workspace_size(rows, hi, max_ctx), dtype=torch.uint8, device=device)
        assert self.buf.data_ptr() % 256 == 0

    @property
    def ptr(self):
        return self.buf.data_ptr()

    @property
    def nbytes(self):
        return self.buf.numel()


def csa2_latent_index_topk(cache: LatentCache, batch, tq, qpos, idx_q, k, out_idx, ws, ratio=1, max_ctx=None,
                           flags=0, stream=None):
    """idx_q [B*tq, hi, 128] bf16 -> out_idx [B*tq, k] int32 (the indexer of the pages' own shape)."""
    if max_ctx is None:
        max_ctx = cache.cap
    _check("csa2_latent_index_topk", lib().csa2_latent_index_topk(
        cache.ref, batch, tq, _i64(qpos), _bits(idx_q), idx_q.shape[-2], k, ratio, max_ctx, flags, _i32(out_idx),
        ws.ptr, ws.nbytes, _stream(stream)))


def csa2_entry_bytes(channels: int) -> int:
    return lib().csa2_entry_bytes(int(channels))


def csa2_mx_entry_bytes(channels: int) -> int:
    return lib().csa2_mx_entry_bytes(int(channels))


def csa2_mxfp4_quantize(x, data, scale, stream=None):
    """MXFP4 rows: x [rows, channels] bf16 -> data [rows, channels/2] u8, scale [rows, channels/32] u8."""
    rows, ch = x.shape
    _check("csa2_mxfp4_quantize", lib().csa2_mxfp4_quantize(_bits(x), rows, ch, _u8(data), _u8(scale), _stream(stream)))


def csa2_status_string(s: int) -> str:
    return status_string(s)


def csa2_version() -> int:
    return lib().csa2_version()


def csa2_workspace_size(shape, batch, tq, k, max_scan, pool_blocks=0) -> int:
    out = ctypes.c_size_t(0)
    _check("csa2_workspace_size", lib().csa2_workspace_size(ctypes.byref(shape), batch, tq, k, max_scan, pool_blocks,
                                                            ctypes.byref(out)))
    return out.value


def csa2_workspace_init(ws: torch.Tensor, stream=None):
    _check("csa2_workspace_init", lib().csa2_workspace_init(_p(ws), ws.numel(), _stream(stream)))


class Workspace:
    """A workspace sized by csa2_workspace_size and cleared once by csa2_workspace_init."""

    def __init__(self, shape, batch, tq, k, max_scan, pool_blocks=0, device="cuda", stream=None):
        n = csa2_workspace_size(shape, batch, tq, k, max_scan, pool_blocks)
        self.buf = torch.empty(n, dtype=torch.uint8, device=device)
        assert self.buf.data_ptr() % 256 == 0
        csa2_workspace_init(self.buf, stream)

    @property
    def ptr(self):
        return self.buf.data_ptr()

    @property
    def nbytes(self):
        return self.buf.numel()


def csa2_quantize_append(shape, cache: Cache, batch, t, pos, kv=None, idx_k=None, swa_kv=None, ws=None, stream=None):
    _check("csa2_quantize_append", lib().csa2_quantize_append(
        ctypes.byref(shape), cache.ref, batch, t, _i64(pos), _bits(kv), _bits(idx_k), _bits(swa_kv),
        ws.ptr if ws else None, ws.nbytes if ws else 0, _stream(stream)))


def csa2_index_topk_full(shape, cache: Cache, batch, tq, qpos, idx_q, k, out_idx, pool_blocks=0, out_pool=None,
                         out_pool_n=None, max_ctx=None, flags=0, ws=None, stream=None):
    if max_ctx is None:
        max_ctx = cache.cap
    _check("csa2_index_topk_full", lib().csa2_index_topk_full(
        ctypes.byref(shape), cache.ref, batch, tq, _i64(qpos), _bits(idx_q), k, _i32(out_idx), pool_blocks, _i32(out_pool),
        _i32(out_pool_n), max_ctx, flags, ws.ptr, ws.nbytes, _stream(stream)))


def csa2_index_topk_reindex(shape, cache: Cache, batch, qpos, idx_q, pool, pool_n, k, out_idx, flags=0, ws=None,
                            stream=None):
    _check("csa2_index_topk_reindex", lib().csa2_index_topk_reindex(
        ctypes.byref(shape), cache.ref, batch, _i64(qpos), _bits(idx_q), _i32(pool), _i32(pool_n), pool.shape[-1], k,
        _i32(out_idx), flags, ws.ptr, ws.nbytes, _stream(stream)))


def csa2_sparse_attend(shape, cache: Cache, batch, tq, qpos, q, idx, k, out, swa_begin=None, sm_scale=0.0,
                       out_f32=None, lse=None, ws=None, stream=None):
    _check("csa2_sparse_attend", lib().csa2_sparse_attend(
        ctypes.byref(shape), cache.ref, batch, tq, _i64(qpos), _bits(q), _i32(idx), k, _i64(swa_begin), sm_scale,
        _bits(out), _f32(out_f32), _f32(lse), ws.ptr, ws.nbytes, _stream(stream)))


def csa2_sparse_attend_noalloc(shape, cache: Cache, batch, tq, qpos, q, idx, k, out, swa_begin=None, sm_scale=0.0,
                               out_f32=None, lse=None, stream=None):
    """csa2_sparse_attend without a workspace (scratch in a static device array inside libcsa2)."""
    _check("csa2_sparse_attend_noalloc", lib().csa2_sparse_attend_noalloc(
        ctypes.byref(shape), cache.ref, batch, tq, _i64(qpos), _bits(q), _i32(idx), k, _i64(swa_begin), sm_scale,
        _bits(out), _f32(out_f32), _f32(lse), _stream(stream)))


def csa2_decode_full(shape, cache: Cache, batch, qpos, kv, idx_k, swa_kv, idx_q, q, k, out_idx, out, pool_blocks=0,
                     out_pool=None, out_pool_n=None, max_ctx=None, swa_begin=None, sm_scale=0.0, out_f32=None,
                     lse=None, flags=0, ws=None, stream=None):
    if max_ctx is None:
        max_ctx = cache.cap
    _check("csa2_decode_full", lib().csa2_decode_full(
        ctypes.byref(shape), cache.ref, batch, _i64(qpos), _bits(kv), _bits(idx_k), _bits(swa_kv), _bits(idx_q),
        _bits(q), k, _i32(out_idx), pool_blocks, _i32(out_pool), _i32(out_pool_n), max_ctx, _i64(swa_begin), sm_scale,
        _bits(out), _f32(out_f32), _f32(lse), flags, ws.ptr, ws.nbytes, _stream(stream)))


def csa2_decode_reindex(shape, cache: Cache, batch, qpos, swa_kv, idx_q, q, pool, pool_n, k, out_idx, out,
                        swa_begin=None, sm_scale=0.0, out_f32=None, lse=None, flags=0, ws=None, stream=None):
    _check("csa2_decode_reindex", lib().csa2_decode_reindex(
        ctypes.byref(shape), cache.ref, batch, _i64(qpos), _bits(swa_kv), _bits(idx_q), _bits(q), _i32(pool), _i32(pool_n),
        pool.shape[-1], k, _i32(out_idx), _i64(swa_begin), sm_scale, _bits(out), _f32(out_f32), _f32(lse), flags, ws.ptr,
        ws.nbytes, _stream(stream)))


def csa2_decode_minimal(shape, cache: Cache, batch, qpos, swa_kv, q, idx, k, out, swa_begin=None, sm_scale=0.0,
                        out_f32=None, lse=None, ws=None, stream=None):
    _check("csa2_decode_minimal", lib().csa2_decode_minimal(
        ctypes.byref(shape), cache.ref, batch, _i64(qpos), _bits(swa_kv), _bits(q), _i32(idx), k, _i64(swa_begin), sm_scale,
        _bits(out), _f32(out_f32), _f32(lse), ws.ptr, ws.nbytes, _stream(stream)))


def csa2_prefill_chunk(shape, cache: Cache, pos0, t, kv, idx_k, swa_kv, idx_q, q, k, out_idx, out, swa_begin=0,
                       sm_scale=0.0, out_f32=None, lse=None, flags=0, ws=None, stream=None):
    _check("csa2_prefill_chunk", lib().csa2_prefill_chunk(
        ctypes.byref(shape), cache.ref, pos0, t, _bits(kv), _bits(idx_k), _bits(swa_kv), _bits(idx_q), _bits(q), k,
        _i32(out_idx), swa_begin, sm_scale, _bits(out), _f32(out_f32), _f32(lse), flags, ws.ptr, ws.nbytes,
        _stream(stream)))


def csa2_get_device_status(ws: Workspace, stream=None) -> int:
    """Synchronises the stream and returns (and clears) the CSA2_DEV_* bits."""
    v = ctypes.c_int32(0)
    s = lib().csa2_get_device_status(ws.ptr, _stream(stream), ctypes.byref(v))
    if s not in (CSA2_OK, CSA2_ERR_DEVICE):
        raise Csa2Error("csa2_get_device_status", s)
    return v.value
