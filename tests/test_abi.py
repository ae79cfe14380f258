"""The C-ABI library loads and exports every symbol include/csa2.h declares; host-only calls and
argument validation (which returns before anything touches a GPU) behave as documented."""
import ctypes
import os
import re

import pytest
import torch

import compressed_sparse_attention_append_b200 as csa
from conftest import ROOT


@pytest.fixture(scope="module")
def L():
    from compressed_sparse_attention_append_b200 import build

    build.build()
    return csa.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "csa2.h")).read()
    return re.findall(r"CSA2_API\s+[\w\s\*]+?\b(csa2_\w+)\s*\(", src)


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert len(names) == 21
    assert set(names) == set(csa.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_header_compiles_as_c():
    import subprocess
    import tempfile

    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        with open(c, "w") as f:
            f.write('#include "csa2.h"\nint main(void){ csa2_shape s; csa2_cache c; csa2_latent_cache l; (void)s; (void)c; (void)l; return 0; }\n')
        subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-c", c,
                               "-o", os.path.join(d, "t.o")])


def test_plain_c_program_links_and_calls_the_host_entry_points(L):
    """A C program built against include/csa2.h and linked to libcsa2.so (no Python, no torch) calls
    the host-only entry points; every call returns before anything touches a GPU."""
    import subprocess
    import tempfile

    prog = r"""
#include <stdio.h>
#include "csa2.h"
int main(void) {
    csa2_shape s = {16, 128, 4, 64, 4, 128, 8, 1};
    size_t ws = 0;
    int st = csa2_workspace_size(&s, 128, 1, 512, 16000, 0, &ws);
    csa2_shape bad = s;
    bad.hq = 64;
    size_t ws2 = 0;
    int st2 = csa2_workspace_size(&bad, 1, 1, 512, 16000, 0, &ws2);
    bad = s;
    bad.ratio = 3;
    int st3 = csa2_workspace_size(&bad, 1, 1, 512, 16000, 0, &ws2);
    printf("%zu %d %d %zu %d %d %d %s\n", csa2_entry_bytes(256), csa2_version(), st, ws, st2, st3,
           st2 == CSA2_ERR_UNSUPPORTED_SHAPE && st3 == CSA2_ERR_UNSUPPORTED_SHAPE,
           csa2_status_string(CSA2_ERR_WORKSPACE));
    return 0;
}
"""
    libdir = os.path.dirname(csa.lib()._name)
    with tempfile.TemporaryDirectory() as d:
        c, exe = os.path.join(d, "p.c"), os.path.join(d, "p")
        with open(c, "w") as f:
            f.write(prog)
        subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), c, "-o",
                               exe, "-L", libdir, "-l:libcsa2.so", f"-Wl,-rpath,{libdir}"])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=60, check=True).stdout.split(maxsplit=7)
    assert out[0] == "144" and out[1] == str(csa.csa2_version()) and out[2] == "0"
    assert int(out[3]) == csa.csa2_workspace_size(csa.make_shape(), 128, 1, 512, 16000, 0)
    assert out[6] == "1"
    assert out[7].strip() == csa.csa2_status_string(csa.CSA2_ERR_WORKSPACE)


def test_plain_c_program_uses_the_latent_declarations(L):
    """The latent cache struct and the entry points of the pages' own shapes, used from plain C:
    MXFP4 entry bytes, the indexer's workspace size, and calls with an empty batch (no launch)."""
    import subprocess
    import tempfile

    prog = r"""
#include <stdio.h>
#include <stdint.h>
#include "csa2.h"
int main(void) {
    static uint8_t planes[5][4096] __attribute__((aligned(256)));
    csa2_latent_cache c = {planes[0], planes[1], planes[2], planes[3], planes[4], 64, 128};
    int64_t qpos[1] = {63};
    uint16_t q[16] __attribute__((aligned(16))) = {0};
    int32_t idx[1] = {-1};
    size_t ws = 0;
    int a = csa2_latent_index_workspace_size(2, 32, 64, &ws);
    int b = csa2_latent_attend(&c, 0, 1, qpos, q, idx, 1, NULL, 128, 1, 0.f, q, NULL, NULL, NULL, 0, NULL);
    int d = csa2_latent_append(&c, 0, 1, qpos, q, NULL, q, NULL, 0, NULL);
    int e = csa2_latent_attend(&c, 1, 1, qpos, q, idx, 1, NULL, 200, 1, 0.f, q, NULL, NULL, NULL, 0, NULL);
    printf("%zu %d %zu %d %d %d\n", csa2_mx_entry_bytes(128), a, ws, b, d, e);
    return 0;
}
"""
    libdir = os.path.dirname(csa.lib()._name)
    with tempfile.TemporaryDirectory() as d:
        c, exe = os.path.join(d, "p.c"), os.path.join(d, "p")
        with open(c, "w") as f:
            f.write(prog)
        subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), c, "-o",
                               exe, "-L", libdir, "-l:libcsa2.so", f"-Wl,-rpath,{libdir}"])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=60, check=True).stdout.split()
    assert out[0] == "68" and out[1] == "0"
    assert int(out[2]) == csa.csa2_latent_index_workspace_size(2, 32, 64)
    assert out[3] == "0" and out[4] == "0"  # empty batches: nothing to do
    assert int(out[5]) == csa.CSA2_ERR_UNSUPPORTED_SHAPE  # a window longer than 128


def test_host_functions(L):
    assert csa.csa2_entry_bytes(256) == 144
    assert csa.csa2_entry_bytes(512) == 288
    assert csa.csa2_entry_bytes(24) == 0 and csa.csa2_entry_bytes(-16) == 0
    assert csa.csa2_version() == 200  # 0.2.0: the entry points of the pages' own shapes
    for s in range(7):
        assert csa.csa2_status_string(s)
    assert csa.csa2_status_string(99) == "unknown status"


def test_workspace_size_is_monotone_and_validates(L):
    sh = csa.make_shape()
    a = csa.csa2_workspace_size(sh, 128, 1, 512, 16000, 0)
    b = csa.csa2_workspace_size(sh, 64, 1, 512, 131072, 2048)
    assert a > 0 and b > a // 4
    assert csa.csa2_workspace_size(sh, 1, 1, 512, 4096) >= 256
    bad = csa.make_shape()
    bad.hq = 8
    with pytest.raises(csa.Csa2Error) as e:
        csa.csa2_workspace_size(bad, 1, 1, 512, 4096)
    assert e.value.status == csa.CSA2_ERR_UNSUPPORTED_SHAPE
    with pytest.raises(csa.Csa2Error) as e:
        csa.csa2_workspace_size(sh, 1, 1, 4096, 4096)
    assert e.value.status == csa.CSA2_ERR_INVALID_ARG
    # compression ratio: 1 or 2 tokens per cache entry
    assert csa.csa2_workspace_size(csa.make_shape(ratio=2), 1, 1, 512, 4096) > 0
    with pytest.raises(csa.Csa2Error) as e:
        csa.csa2_workspace_size(csa.make_shape(ratio=3), 1, 1, 512, 4096)
    assert e.value.status == csa.CSA2_ERR_UNSUPPORTED_SHAPE


def test_decode_workspace_covers_every_region(L):
    """A decode-row workspace must hold, per row: one 8-byte key per scanned position, the score
    histograms (2 x 2048 + 2 x 1024 four-byte bins), two candidate lists of 4096 (key, position)
    pairs, and with a pool the block maxima (rows of an even number of 8-byte entries); plus the
    fixed counter area (status header, 65,536 row counters of 16 bytes, 65,536 attention tickets).
    A multi-row (prefill) plan needs none of the decode regions."""
    sh = csa.make_shape()
    fixed = 256 + 16 * 65536 + 4 * 65536
    for rows, scan, pool in ((1, 4096, 0), (128, 16000, 0), (64, 131072, 2048), (3, 1000, 125)):
        units = (scan + 7) // 8
        bmax = ((units + 1) // 2 * 2) * 8 if pool else 0
        need = fixed + rows * (units * 8 * 8 + (2 * 2048 + 2 * 1024) * 4 + 2 * 4096 * 16 + bmax)
        got = csa.csa2_workspace_size(sh, rows, 1, 512, scan, pool)
        assert got >= need, (rows, scan, pool, got, need)
        assert got < need + 16 * 256 + rows * 16 * 132 * 4 * 64  # alignment and attention partials only
    # the same rows as 4 prefill rows each: no per-position keys, only candidate slots
    assert csa.csa2_workspace_size(sh, 8, 4, 512, 4096) < csa.csa2_workspace_size(sh, 32, 1, 512, 4096)


def _fake_cache(cap=4096, swa_cap=128, align=16):
    base = 1 << 40
    return csa.csa2_cache(base, base + 1 * align * 1024, base + 2 * align * 1024, base + 3 * align * 1024,
                          base + 4 * align * 1024, cap, swa_cap)


def test_validation_before_launch(L):
    """Each call below must return its error without launching (the pointers are not real)."""
    sh = csa.make_shape()
    c = _fake_cache()
    F = 1 << 41
    vp = F
    # unsupported shape
    bad = csa.make_shape()
    bad.di = 32
    assert L.csa2_index_topk_full(ctypes.byref(bad), ctypes.byref(c), 1, 1, vp, vp, 512, vp, 0, None, None, 100, 0,
                                  vp, 1 << 30, None) == csa.CSA2_ERR_UNSUPPORTED_SHAPE
    # k out of range / pool with tq > 1 / max_ctx beyond capacity / unknown flag
    assert L.csa2_index_topk_full(ctypes.byref(sh), ctypes.byref(c), 1, 1, vp, vp, 0, vp, 0, None, None, 100, 0, vp,
                                  1 << 30, None) == csa.CSA2_ERR_INVALID_ARG
    assert L.csa2_index_topk_full(ctypes.byref(sh), ctypes.byref(c), 1, 2, vp, vp, 512, vp, 64, vp, vp, 100, 0, vp,
                                  1 << 30, None) == csa.CSA2_ERR_INVALID_ARG
    assert L.csa2_index_topk_full(ctypes.byref(sh), ctypes.byref(c), 1, 1, vp, vp, 512, vp, 0, None, None, 5000, 0,
                                  vp, 1 << 30, None) == csa.CSA2_ERR_CAPACITY
    assert L.csa2_index_topk_full(ctypes.byref(sh), ctypes.byref(c), 1, 1, vp, vp, 512, vp, 0, None, None, 100, 8,
                                  vp, 1 << 30, None) == csa.CSA2_ERR_INVALID_ARG
    # the composed decode_full and prefill_chunk calls take one entry per token only
    r2 = csa.make_shape(ratio=2)
    assert L.csa2_decode_full(ctypes.byref(r2), ctypes.byref(c), 1, vp, vp, vp, vp, vp, vp, 512, vp, 0, None, None,
                              100, None, 0.0, vp, None, None, 0, vp, 1 << 30, None) == csa.CSA2_ERR_UNSUPPORTED_SHAPE
    assert L.csa2_prefill_chunk(ctypes.byref(r2), ctypes.byref(c), 0, 16, vp, vp, vp, vp, vp, 512, vp, 0, 0.0, vp, None,
                                None, 0, vp, 1 << 30, None) == csa.CSA2_ERR_UNSUPPORTED_SHAPE
    # workspace too small / missing
    assert L.csa2_index_topk_full(ctypes.byref(sh), ctypes.byref(c), 4, 1, vp, vp, 512, vp, 0, None, None, 4096, 0,
                                  vp, 1024, None) == csa.CSA2_ERR_WORKSPACE
    assert L.csa2_sparse_attend(ctypes.byref(sh), ctypes.byref(c), 4, 1, vp, vp, vp, 512, None, 0.0, vp, None, None,
                                None, 0, None) == csa.CSA2_ERR_WORKSPACE
    # misaligned pointer, bad ring capacity, NaN scale
    assert L.csa2_sparse_attend(ctypes.byref(sh), ctypes.byref(c), 4, 1, vp, vp + 2, vp, 512, None, 0.0, vp, None,
                                None, vp, 1 << 30, None) == csa.CSA2_ERR_INVALID_ARG
    c2 = _fake_cache(swa_cap=100)
    assert L.csa2_sparse_attend(ctypes.byref(sh), ctypes.byref(c2), 4, 1, vp, vp, vp, 512, None, 0.0, vp, None, None,
                                vp, 1 << 30, None) == csa.CSA2_ERR_INVALID_ARG
    assert L.csa2_sparse_attend(ctypes.byref(sh), ctypes.byref(c), 4, 1, vp, vp, vp, 512, None, float("nan"), vp, None,
                                None, vp, 1 << 30, None) == csa.CSA2_ERR_INVALID_ARG
    # append beyond capacity (host-visible), null pos
    assert L.csa2_quantize_append(ctypes.byref(sh), ctypes.byref(c), 1, 5000, vp, vp, None, None, None, 0,
                                  None) == csa.CSA2_ERR_CAPACITY
    assert L.csa2_quantize_append(ctypes.byref(sh), ctypes.byref(c), 1, 1, None, vp, None, None, None, 0,
                                  None) == csa.CSA2_ERR_INVALID_ARG
    # prefill: window ring too small for the chunk
    assert L.csa2_prefill_chunk(ctypes.byref(sh), ctypes.byref(c), 0, 256, vp, vp, vp, vp, vp, 512, vp, 0, 0.0, vp,
                                None, None, 0, vp, 1 << 30, None) == csa.CSA2_ERR_CAPACITY
    # device status needs a workspace
    v = ctypes.c_int32(0)
    assert L.csa2_get_device_status(None, None, ctypes.byref(v)) == csa.CSA2_ERR_INVALID_ARG


def test_product_path_has_no_oracle_dependency():
    """The package and the kernels never import, link or read the oracle."""
    pkg = os.path.join(ROOT, "compressed_sparse_attention_append_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.lower(), f


def test_binding_checks_integer_and_float_dtypes(L):
    """The binding refuses an array of the wrong dtype before anything reaches the library (a kernel
    would read an int32 array as int64, or the reverse); the dtype check runs before the device check,
    so CPU tensors show it here."""
    import types

    shape = csa.make_shape()
    cache = types.SimpleNamespace(ref=ctypes.byref(csa.csa2_cache()), cap=64)  # never dereferenced here
    swa = torch.zeros(1, 1, 256, dtype=torch.bfloat16)
    with pytest.raises(AssertionError, match="int64"):
        csa.csa2_quantize_append(shape, cache, 1, 1, torch.zeros(1, dtype=torch.int32), swa_kv=swa)
    with pytest.raises(AssertionError, match="int64"):
        csa.csa2_sparse_attend(shape, cache, 1, 1, torch.zeros(1, dtype=torch.int32), None, None, 512, None)
    with pytest.raises(AssertionError, match="CUDA"):  # right dtype: the device check comes next
        csa.csa2_quantize_append(shape, cache, 1, 1, torch.zeros(1, dtype=torch.int64), swa_kv=swa)
    for fn, good, bad in ((csa._i32, torch.int32, torch.int64), (csa._i64, torch.int64, torch.int32),
                          (csa._f32, torch.float32, torch.bfloat16)):
        with pytest.raises(AssertionError, match=str(good)):
            fn(torch.zeros(2, dtype=bad))
        with pytest.raises(AssertionError, match="CUDA"):
            fn(torch.zeros(2, dtype=good))
        assert fn(None) is None


def test_mx_entry_bytes_and_codec_validation(L):
    """[C] sec. VII: an MXFP4 entry of ch channels is ch/2 + ch/32 bytes (the pages' 128-channel
    indexer key: 68 B); the codec rejects bad arguments before any launch."""
    assert csa.csa2_mx_entry_bytes(128) == 68
    assert csa.csa2_mx_entry_bytes(512) == 272
    assert csa.csa2_mx_entry_bytes(32) == 17
    for bad in (0, 16, 48, -32):
        assert csa.csa2_mx_entry_bytes(bad) == 0
    f = L.csa2_mxfp4_quantize
    buf = ctypes.create_string_buffer(4096 + 16)
    base = (ctypes.addressof(buf) + 15) & ~15
    assert f(None, 1, 32, base, base, None) == csa.CSA2_ERR_INVALID_ARG
    assert f(base, 1, 48, base, base, None) == csa.CSA2_ERR_INVALID_ARG
    assert f(base, -1, 32, base, base, None) == csa.CSA2_ERR_INVALID_ARG
    assert f(base + 2, 1, 32, base, base, None) == csa.CSA2_ERR_INVALID_ARG
    assert f(base, 0, 32, base, base, None) == csa.CSA2_OK  # nothing to do, no launch


def test_latent_entry_points_validate_before_any_launch(L):
    """The pages' own shape (latent cache, 64 x 512 attention): bad pointers, alignment, sizes, window
    and ratio are rejected on the host; an empty batch returns OK without a launch."""
    buf = ctypes.create_string_buffer(1 << 16)
    base = (ctypes.addressof(buf) + 255) & ~255
    c = csa.csa2_latent_cache(base, base + 4096, base + 8192, base + 12288, base + 16384, 1024, 128)
    rc = ctypes.byref(c)
    att, app = L.csa2_latent_attend, L.csa2_latent_append
    q = out = idx = qpos = base + 32768
    # (cache, batch, tq, qpos, q, idx, k, swa_begin, win, ratio, sm_scale, out, out_f32, lse, ws, ws_bytes, stream)
    assert att(rc, 0, 1, qpos, q, idx, 512, None, 128, 1, 0.0, out, None, None, None, 0, None) == csa.CSA2_OK
    assert att(None, 0, 1, qpos, q, idx, 512, None, 128, 1, 0.0, out, None, None, None, 0, None) == csa.CSA2_ERR_INVALID_ARG
    assert att(rc, 0, 1, None, q, idx, 512, None, 128, 1, 0.0, out, None, None, None, 0, None) == csa.CSA2_ERR_INVALID_ARG
    assert att(rc, 0, 1, qpos, q + 2, idx, 512, None, 128, 1, 0.0, out, None, None, None, 0, None) == csa.CSA2_ERR_INVALID_ARG
    assert att(rc, 0, 1, qpos, q, idx, 4096, None, 128, 1, 0.0, out, None, None, None, 0, None) == csa.CSA2_ERR_INVALID_ARG
    assert att(rc, 0, 1, qpos, q, None, 512, None, 128, 1, 0.0, out, None, None, None, 0, None) == csa.CSA2_ERR_INVALID_ARG
    assert att(rc, 0, 1, qpos, q, idx, 512, None, 129, 1, 0.0, out, None, None, None, 0, None) == csa.CSA2_ERR_UNSUPPORTED_SHAPE
    assert att(rc, 0, 1, qpos, q, idx, 512, None, 128, 3, 0.0, out, None, None, None, 0, None) == csa.CSA2_ERR_UNSUPPORTED_SHAPE
    assert att(rc, 0, 1, qpos, q, idx, 512, None, 128, 1, 0.0, out, None, None, base, 16, None) == csa.CSA2_ERR_WORKSPACE
    small = csa.csa2_latent_cache(base, base + 4096, base + 8192, base + 12288, base + 16384, 1024, 64)
    assert att(ctypes.byref(small), 0, 1, qpos, q, idx, 512, None, 128, 1, 0.0, out, None, None, None, 0, None) == \
        csa.CSA2_ERR_CAPACITY  # the window ring is shorter than the window
    odd = csa.csa2_latent_cache(base + 8, base + 4096, base + 8192, base + 12288, base + 16384, 1024, 128)
    assert att(ctypes.byref(odd), 0, 1, qpos, q, idx, 512, None, 128, 1, 0.0, out, None, None, None, 0, None) == \
        csa.CSA2_ERR_INVALID_ARG
    # (cache, batch, t, pos, latent, idx_k, swa, ws, ws_bytes, stream)
    x = base + 40960
    assert app(rc, 0, 1, qpos, x, x, x, None, 0, None) == csa.CSA2_OK
    assert app(rc, 1, 1, None, x, x, x, None, 0, None) == csa.CSA2_ERR_INVALID_ARG
    assert app(rc, -1, 1, qpos, x, x, x, None, 0, None) == csa.CSA2_ERR_INVALID_ARG
    assert app(rc, 1, 1, qpos, x + 2, None, None, None, 0, None) == csa.CSA2_ERR_INVALID_ARG
    assert app(rc, 1, 2048, qpos, x, None, None, None, 0, None) == csa.CSA2_ERR_CAPACITY
    nokey = csa.csa2_latent_cache(base, base + 4096, None, None, base + 16384, 1024, 128)
    assert app(ctypes.byref(nokey), 1, 1, qpos, None, x, None, None, 0, None) == csa.CSA2_ERR_INVALID_ARG


def test_latent_index_entry_points_validate_before_any_launch(L):
    """The indexer of the pages' own shape: workspace sizing and argument checks on the host; an
    empty batch returns OK without a launch."""
    sz = ctypes.c_size_t(0)
    assert L.csa2_latent_index_workspace_size(4, 32, 1000, ctypes.byref(sz)) == csa.CSA2_OK
    # status line, 4 x 32 query codes (64 B) and scales (4 B), 4 x 1000 8-byte keys, 256-byte aligned parts
    assert sz.value == 256 + 8192 + 512 + 32000
    for bad in ((4, 0, 1000), (4, 65, 1000), (-1, 32, 1000), (70000, 32, 1000), (4, 32, 0)):
        assert L.csa2_latent_index_workspace_size(*bad, ctypes.byref(sz)) == csa.CSA2_ERR_INVALID_ARG
    buf = ctypes.create_string_buffer(1 << 16)
    base = (ctypes.addressof(buf) + 255) & ~255
    c = csa.csa2_latent_cache(None, None, base + 8192, base + 12288, None, 1024, 128)
    rc = ctypes.byref(c)
    f = L.csa2_latent_index_topk
    qpos = iq = out = base + 16384
    ws = base + 32768
    # (cache, batch, tq, qpos, idx_q, hi, k, ratio, max_ctx, flags, out_idx, ws, ws_bytes, stream)
    assert f(rc, 0, 1, qpos, iq, 32, 512, 1, 1000, 0, out, ws, 256, None) == csa.CSA2_OK
    assert f(rc, 1, 1, qpos, iq, 32, 512, 1, 1000, 0, out, ws, 256, None) == csa.CSA2_ERR_WORKSPACE
    assert f(rc, 1, 1, qpos, iq, 0, 512, 1, 1000, 0, out, ws, 1 << 20, None) == csa.CSA2_ERR_INVALID_ARG
    assert f(rc, 1, 1, qpos, iq, 32, 4096, 1, 1000, 0, out, ws, 1 << 20, None) == csa.CSA2_ERR_INVALID_ARG
    assert f(rc, 1, 1, qpos, iq, 32, 512, 3, 1000, 0, out, ws, 1 << 20, None) == csa.CSA2_ERR_UNSUPPORTED_SHAPE
    assert f(rc, 1, 1, qpos, iq + 2, 32, 512, 1, 1000, 0, out, ws, 1 << 20, None) == csa.CSA2_ERR_INVALID_ARG
    assert f(rc, 1, 1, qpos, iq, 32, 512, 1, 1000, 0, out, ws + 16, 1 << 20, None) == csa.CSA2_ERR_INVALID_ARG
    assert f(None, 1, 1, qpos, iq, 32, 512, 1, 1000, 0, out, ws, 1 << 20, None) == csa.CSA2_ERR_INVALID_ARG
    nokey = csa.csa2_latent_cache(None, None, None, None, None, 1024, 128)
    assert f(ctypes.byref(nokey), 1, 1, qpos, iq, 32, 512, 1, 1000, 0, out, ws, 1 << 20, None) == \
        csa.CSA2_ERR_INVALID_ARG
