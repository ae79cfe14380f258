"""CPU oracle for the CSA2 layer step over an FP4 KV cache (ctypes wrapper of csa2_oracle.c).

TEST INFRASTRUCTURE. Only tests/, ``__graft_entry__.smoke()`` and ``bench.py``'s
cpu_baseline / reference leg may import this package. It shares no code with the CUDA
path and never consumes anything the CUDA path produced.

Sources (tags as in csa2_oracle.c):
  [A] "DeepSeek-V4.1-Flash: Shrinking KV Cache at 552B Scale" (visualisation captions)
  [B] "DeepSeek Cuts KV Cache Footprint Fourfold", "Technical Approach"
  [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token"

Each wrapper below names the passage its C function follows. Arrays are numpy; bf16
inputs are passed as their raw uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa2_oracle.c")
_LIB = os.path.join(_HERE, "libcsa2_oracle.so")

GCC_FLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile csa2_oracle.c with gcc into oracle/libcsa2_oracle.so (plain C, -lm)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


class _SeqCache(ctypes.Structure):
    _fields_ = [
        ("kv_data", ctypes.c_void_p),
        ("kv_scale", ctypes.c_void_p),
        ("ik_data", ctypes.c_void_p),
        ("ik_scale", ctypes.c_void_p),
        ("swa", ctypes.c_void_p),
        ("cap", ctypes.c_int64),
        ("swa_cap", ctypes.c_int64),
        ("hk", ctypes.c_int),
    ]


def lib():
    """The loaded oracle library: oracle/libcsa2_oracle.so, or the build of csa2_oracle.c that the
    environment variable CSA2_ORACLE_LIB names (the planted-mistake tests load copies of the source
    with one mistake planted in each)."""
    global _lib
    if _lib is None:
        L = ctypes.CDLL(os.environ.get("CSA2_ORACLE_LIB") or build())
        d, i, i64, vp = ctypes.c_double, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
        sig = {
            "orc_e2m1_decode": (d, [i]),
            "orc_e4m3_decode": (d, [i]),
            "orc_e2m1_encode": (i, [d]),
            "orc_e4m3_encode": (i, [d]),
            "orc_bf16_to_double": (d, [ctypes.c_uint16]),
            "orc_entry_bytes": (i64, [i]),
            "orc_quantize_rows": (None, [vp, i64, i, vp, vp]),
            "orc_fp8_rows": (None, [vp, i64, vp]),
            "orc_dequant_rows": (None, [vp, vp, i64, i, vp]),
            "orc_quantize_append": (i, [vp, i64, i, vp, vp, vp]),
            "orc_quantize_index_query": (None, [vp, i, vp, vp]),
            "orc_scores": (None, [vp, vp, i, vp, i64, i, vp]),
            "orc_topk": (i, [vp, vp, i64, i, vp]),
            "orc_pool": (i, [vp, i64, i, i, vp]),
            "orc_index_topk_full": (i, [vp, i64, vp, i, i, i, vp, i, i, vp, vp, i]),
            "orc_index_topk_reindex": (i, [vp, i64, vp, i, vp, i, i, i, i, vp, i]),
            "orc_sparse_attend": (i, [vp, i64, vp, i, vp, i, i64, i, d, vp, vp, i]),
            "orc_e8m0_decode": (d, [i]),
            "orc_mx_entry_bytes": (i64, [i]),
            "orc_mx_quantize_rows": (None, [vp, i64, i, vp, vp]),
            "orc_mx_dequant_rows": (None, [vp, vp, i64, i, vp]),
            "orc_mx_index_topk_full": (i, [vp, vp, i64, i64, vp, i, i, i, vp, vp, i]),
            "orc_latent_attend": (i, [vp, vp, i64, vp, i64, i64, vp, i, vp, i, i64, i, d, vp, vp, i]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(x) -> np.ndarray:
    """Accept a numpy uint16 array of bf16 bit patterns or a torch bf16 tensor."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # plain CPU view of the bit pattern

    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


# ---- element formats: [C] sec. XI; [A] FP4 caption -------------------------------------------
def e2m1_decode(code: int) -> float:
    return lib().orc_e2m1_decode(int(code))


def e4m3_decode(byte: int) -> float:
    return lib().orc_e4m3_decode(int(byte))


def e2m1_encode(y: float) -> int:
    return lib().orc_e2m1_encode(float(y))


def e4m3_encode(y: float) -> int:
    return lib().orc_e4m3_encode(float(y))


def entry_bytes(ch: int) -> int:
    """[C] sec. VII: bytes per entry of ch channels = ch/2 + ch/16 (0 if ch % 16)."""
    return lib().orc_entry_bytes(int(ch))


def quantize_rows(x, ch: int):
    """R1 codec over rows of `ch` channels -> (packed data [rows, ch/2], scales [rows, ch/16])."""
    xb = _bf16_bits(x).reshape(-1, ch)
    rows = xb.shape[0]
    data = np.zeros((rows, ch // 2), np.uint8)
    scale = np.zeros((rows, ch // 16), np.uint8)
    lib().orc_quantize_rows(_p(xb), rows, ch, _p(data), _p(scale))
    return data, scale


def fp8_rows(x) -> np.ndarray:
    """R8: elementwise E4M3 (RNE, satfinite) of bf16 values."""
    xb = _bf16_bits(x)
    out = np.zeros(xb.shape, np.uint8)
    lib().orc_fp8_rows(_p(xb.reshape(-1)), xb.size, _p(out.reshape(-1)))
    return out


def dequant_rows(data: np.ndarray, scale: np.ndarray, ch: int) -> np.ndarray:
    data = np.ascontiguousarray(data, np.uint8).reshape(-1, ch // 2)
    scale = np.ascontiguousarray(scale, np.uint8).reshape(-1, ch // 16)
    out = np.zeros((data.shape[0], ch), np.float64)
    lib().orc_dequant_rows(_p(data), _p(scale), data.shape[0], ch, _p(out))
    return out


def topk(scores: np.ndarray, pos: np.ndarray, k: int):
    """R5/R6: Top-k by (score desc, position asc), emitted ascending, padded with -1."""
    s = np.ascontiguousarray(scores, np.float64)
    p = np.ascontiguousarray(pos, np.int64)
    out = np.zeros(k, np.int32)
    m = lib().orc_topk(_p(s), _p(p), s.size, k, _p(out))
    return out, m


def pool(scores: np.ndarray, bs: int, pool_blocks: int):
    """R10 block pool over scores of positions 0..n-1 -> (ascending block ids padded -1, count)."""
    s = np.ascontiguousarray(scores, np.float64)
    out = np.zeros(pool_blocks, np.int32)
    m = lib().orc_pool(_p(s), s.size, bs, pool_blocks, _p(out))
    return out, m


class SeqCache:
    """One sequence's cache planes in the R9 layout (numpy, owned here)."""

    def __init__(self, cap: int, swa_cap: int, hk: int = 4):
        assert swa_cap & (swa_cap - 1) == 0, "SWA ring capacity must be a power of two"
        self.cap, self.swa_cap, self.hk = cap, swa_cap, hk
        self.kv_data = np.zeros((cap, 128), np.uint8)
        self.kv_scale = np.zeros((cap, 16), np.uint8)
        self.ik_data = np.zeros((cap, hk * 32), np.uint8)
        self.ik_scale = np.zeros((cap, hk * 4), np.uint8)
        self.swa = np.zeros((swa_cap, 256), np.uint8)
        self._c = _SeqCache(
            _p(self.kv_data).value, _p(self.kv_scale).value, _p(self.ik_data).value,
            _p(self.ik_scale).value, _p(self.swa).value, cap, swa_cap, hk,
        )

    @property
    def ref(self):
        return ctypes.byref(self._c)

    def append(self, pos: int, kv=None, idx_k=None, swa_kv=None):
        """Quantise-append t tokens at pos..pos+t-1 ([C] sec. XI; [B] Technical Approach)."""
        arrs = [None if a is None else _bf16_bits(a) for a in (kv, idx_k, swa_kv)]
        t = None
        for a, w in zip(arrs, (256, self.hk * 64, 256)):
            if a is not None:
                a2 = a.reshape(-1, w)
                t = a2.shape[0] if t is None else t
                assert a2.shape[0] == t
        if t is None:
            return
        ptrs = [None if a is None else _p(a) for a in arrs]
        rc = lib().orc_quantize_append(self.ref, pos, t, *ptrs)
        if rc != 0:
            raise ValueError("append out of capacity")

    def scores(self, idx_q, positions) -> np.ndarray:
        q = _bf16_bits(idx_q).reshape(-1)
        hi = q.size // 64
        p = np.ascontiguousarray(positions, np.int64)
        out = np.zeros(p.size, np.float64)
        lib().orc_scores(self.ref, _p(q), hi, _p(p), p.size, 0, _p(out))
        return out

    def scores_relu(self, idx_q, positions) -> np.ndarray:
        q = _bf16_bits(idx_q).reshape(-1)
        p = np.ascontiguousarray(positions, np.int64)
        out = np.zeros(p.size, np.float64)
        lib().orc_scores(self.ref, _p(q), q.size // 64, _p(p), p.size, 1, _p(out))
        return out

    def index_topk_full(self, qpos: int, idx_q, k: int = 512, pool_blocks: int = 0, bs: int = 8, relu=False,
                        ratio: int = 1):
        """Full mode at token qpos; with compression ratio `ratio` the first (qpos + 1) // ratio
        entries are visible (R12)."""
        q = _bf16_bits(idx_q).reshape(-1)
        out = np.zeros(k, np.int32)
        pool_out = np.zeros(max(pool_blocks, 1), np.int32)
        pool_n = np.zeros(1, np.int32)
        lib().orc_index_topk_full(self.ref, qpos, _p(q), q.size // 64, k, int(relu), _p(out),
                                  pool_blocks, bs, _p(pool_out), _p(pool_n), int(ratio))
        if pool_blocks > 0:
            return out, pool_out, int(pool_n[0])
        return out

    def index_topk_reindex(self, qpos: int, idx_q, pool_ids, pool_n: int, k: int = 512, bs: int = 8, relu=False,
                           ratio: int = 1):
        q = _bf16_bits(idx_q).reshape(-1)
        pl = np.ascontiguousarray(pool_ids, np.int32)
        out = np.zeros(k, np.int32)
        lib().orc_index_topk_reindex(self.ref, qpos, _p(q), q.size // 64, _p(pl), int(pool_n), bs, k,
                                     int(relu), _p(out), int(ratio))
        return out

    def sparse_attend(self, qpos: int, q, idx, swa_begin: int = 0, win: int = 128, sm_scale: float = 0.0,
                      ratio: int = 1):
        """R7/R8: one softmax over selected FP4 rows and the FP8 window; fp64 out [hq,128], lse [hq].
        Selected entries must be visible at token qpos (R12); the window is per token."""
        qb = _bf16_bits(q).reshape(-1)
        hq = qb.size // 128
        ix = np.ascontiguousarray(idx, np.int32).reshape(-1)
        if sm_scale == 0.0:
            sm_scale = 1.0 / np.sqrt(128.0)
        out = np.zeros((hq, 128), np.float64)
        lse = np.zeros(hq, np.float64)
        nk = lib().orc_sparse_attend(self.ref, qpos, _p(qb), hq, _p(ix), ix.size, swa_begin, win,
                                     float(sm_scale), _p(out), _p(lse), int(ratio))
        if nk < 0:
            raise ValueError("index out of range")
        return out, lse


# ---- the pages' own shapes: MXFP4 indexer key, 512-channel latent ([C] sec. VII, config list) ----
def e8m0_decode(byte: int) -> float:
    """E8M0 shared scale: 2^(byte - 127); 0xFF is NaN."""
    return lib().orc_e8m0_decode(int(byte))


def mx_entry_bytes(ch: int) -> int:
    """[C] sec. VII: bytes of an MXFP4 entry of ch channels = ch/2 + ch/32 (0 if ch % 32)."""
    return lib().orc_mx_entry_bytes(int(ch))


def mx_quantize_rows(x, ch: int):
    """R13 MXFP4 codec over rows of `ch` channels -> (packed data [rows, ch/2], E8M0 [rows, ch/32])."""
    xb = _bf16_bits(x).reshape(-1, ch)
    rows = xb.shape[0]
    data = np.zeros((rows, ch // 2), np.uint8)
    scale = np.zeros((rows, ch // 32), np.uint8)
    lib().orc_mx_quantize_rows(_p(xb), rows, ch, _p(data), _p(scale))
    return data, scale


def mx_dequant_rows(data: np.ndarray, scale: np.ndarray, ch: int) -> np.ndarray:
    data = np.ascontiguousarray(data, np.uint8).reshape(-1, ch // 2)
    scale = np.ascontiguousarray(scale, np.uint8).reshape(-1, ch // 32)
    out = np.zeros((data.shape[0], ch), np.float64)
    lib().orc_mx_dequant_rows(_p(data), _p(scale), data.shape[0], ch, _p(out))
    return out


class LatentCache:
    """One sequence's cache in the pages' own shapes: the 512-channel latent (K = V) in the R1 codec
    (256 B of codes + 32 B of E4M3 scales per entry), the ONE 128-channel indexer key in MXFP4 (64 B
    + 4 B of E8M0 scales per entry) and a power-of-two ring of 512-channel FP8 window rows."""

    def __init__(self, cap: int, swa_cap: int):
        assert swa_cap & (swa_cap - 1) == 0, "window ring capacity must be a power of two"
        self.cap, self.swa_cap = cap, swa_cap
        self.ldata = np.zeros((cap, 256), np.uint8)
        self.lscale = np.zeros((cap, 32), np.uint8)
        self.kdata = np.zeros((cap, 64), np.uint8)
        self.kscale = np.zeros((cap, 4), np.uint8)
        self.swa = np.zeros((swa_cap, 512), np.uint8)

    def append(self, pos: int, latent=None, idx_k=None, swa=None):
        """Quantise-append entries pos..pos+t-1 of any of the three planes (bf16 inputs)."""
        if latent is not None:
            xb = _bf16_bits(latent).reshape(-1, 512)
            assert 0 <= pos and pos + xb.shape[0] <= self.cap
            d, s = quantize_rows(xb, 512)
            self.ldata[pos:pos + xb.shape[0]], self.lscale[pos:pos + xb.shape[0]] = d, s
        if idx_k is not None:
            xb = _bf16_bits(idx_k).reshape(-1, 128)
            assert 0 <= pos and pos + xb.shape[0] <= self.cap
            d, s = mx_quantize_rows(xb, 128)
            self.kdata[pos:pos + xb.shape[0]], self.kscale[pos:pos + xb.shape[0]] = d, s
        if swa is not None:
            xb = _bf16_bits(swa).reshape(-1, 512)
            for i in range(xb.shape[0]):
                self.swa[(pos + i) & (self.swa_cap - 1)] = fp8_rows(xb[i])

    def index_topk_full(self, qpos: int, idx_q, k: int = 512, relu=False, ratio: int = 1):
        """R14: Top-k of the entries visible at token qpos for a 32 x 128 (any hi <= 64) query ->
        (ascending positions padded with -1, scores of entries 0..visible-1)."""
        qb = _bf16_bits(idx_q).reshape(-1, 128)
        n = max(0, (qpos + 1) // ratio) if qpos >= 0 else 0
        out = np.zeros(k, np.int32)
        sc = np.zeros(max(n, 1), np.float64)
        m = lib().orc_mx_index_topk_full(_p(self.kdata), _p(self.kscale), self.cap, int(qpos), _p(qb), qb.shape[0],
                                         int(k), int(bool(relu)), _p(out), _p(sc), int(ratio))
        assert m >= 0, "query outside the cache"
        return out, sc[:n]

    def attend(self, qpos: int, q, idx, swa_begin: int = 0, win: int = 128, sm_scale: float = 0.0, ratio: int = 1):
        """R15: one softmax over the selected latent entries and the window rows, K = V = the latent;
        sm_scale 0 means 1/sqrt(512). -> (out [hq, 512], lse [hq])."""
        qb = _bf16_bits(q).reshape(-1, 512)
        hq = qb.shape[0]
        idx = np.ascontiguousarray(idx, np.int32)
        if sm_scale == 0.0:
            sm_scale = 1.0 / np.sqrt(512.0)
        out = np.zeros((hq, 512), np.float64)
        lse = np.zeros(hq, np.float64)
        nk = lib().orc_latent_attend(_p(self.ldata), _p(self.lscale), self.cap, _p(self.swa), self.swa_cap, int(qpos),
                                     _p(qb), hq, _p(idx), idx.size, int(swa_begin), int(win), float(sm_scale),
                                     _p(out), _p(lse), int(ratio))
        assert nk >= 0, "a selected entry is not visible or outside the cache"
        return out, lse
