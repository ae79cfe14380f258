"""Planted mistakes in the oracle: the pins must catch each of them.

Each case copies oracle/csa2_oracle.c, plants ONE plausible mistake in the copy (a rounding rule,
a dropped term, a wrong index, sign or operand), builds it with the oracle's own gcc flags, and
runs the oracle's pin tests against that build (oracle.lib() loads the library named by
CSA2_ORACLE_LIB). At least one pin must fail: pytest exits 1 ("tests failed"), not 0 and not with
a collection or usage error. A control build of the unchanged source must pass the same pins, so
a caught mistake means the pins saw it, not that the harness is broken. Everything runs on the
CPU; the CUDA path is not involved.
"""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "csa2_oracle.c")

CODEC = ["tests/test_oracle_codec.py", "tests/test_golden_bytes.py"]
SELECT = ["tests/test_oracle_select.py"]
ATTN = ["tests/test_oracle_attention.py"]
PAGES = ["tests/test_oracle_pages_shapes.py"]

# id, text in csa2_oracle.c (must occur exactly once), the planted mistake, pin files that must catch it
MUTANTS = [
    ("e2m1_ties_away_from_zero", "v = rne_multiple(a, step);", "v = floor(a / step + 0.5) * step;", CODEC),
    ("e4m3_ties_away_from_zero", "r = rne_multiple(a, step);", "r = floor(a / step + 0.5) * step;", CODEC),
    ("e2m1_minus_zero_loses_sign", "int sign = signbit(y) ? 8 : 0;", "int sign = (y < 0) ? 8 : 0;", CODEC),
    ("e2m1_saturates_at_4", "if (a >= 6.0) return sign | 7;", "if (a >= 4.0) return sign | 6;", CODEC),
    ("e4m3_subnormal_step", "if (a < ldexp(1.0, -6)) step = ldexp(1.0, -9);",
     "if (a < ldexp(1.0, -6)) step = ldexp(1.0, -8);", CODEC),
    ("scale_divides_by_4", "int sc = orc_e4m3_encode(amax / 6.0);", "int sc = orc_e4m3_encode(amax / 4.0);", CODEC),
    ("nibbles_swapped", "dr[8 * b + i / 2] = (uint8_t)(c0 | (c1 << 4));",
     "dr[8 * b + i / 2] = (uint8_t)(c1 | (c0 << 4));", CODEC),
    ("dequant_scale_block_32", "orc_e4m3_decode(scale[r * nb + c / 16]);", "orc_e4m3_decode(scale[r * nb + c / 32]);",
     CODEC),
    ("entry_bytes_scale_per_32", "return ch / 2 + ch / 16;", "return ch / 2 + ch / 32;", CODEC),
    ("score_drops_last_head", "for (int h = 0; h < hi; ++h) {\n        int g = h * hk / hi;",
     "for (int h = 0; h < hi - 1; ++h) {\n        int g = h * hk / hi;", SELECT),
    ("key_head_interleaved", "int g = h * hk / hi;", "int g = h % hk;", SELECT),
    ("relu_ignored", "dot += qd[h * 64 + c] * kv[c];\n        total += (relu && dot < 0.0) ? 0.0 : dot;",
     "dot += qd[h * 64 + c] * kv[c];\n        total += dot;", SELECT),
    ("query_not_quantised", "orc_dequant_rows(qdata, qscale, hi, 64, qd);",
     "for (int i = 0; i < hi * 64; ++i) qd[i] = bf16_to_double(idx_q[i]);", SELECT),
    ("topk_ties_to_higher_position", "return (x->p < y->p) ? -1 : (x->p > y->p);",
     "return (x->p > y->p) ? -1 : (x->p < y->p);", SELECT),
    ("topk_keeps_one_less", "int m = (int)(n < k ? n : k);", "int m = (int)(n < k ? n : k - 1);", SELECT),
    ("pool_block_of_seven", "for (int64_t p = b * bs; p < (b + 1) * bs && p < n; ++p)",
     "for (int64_t p = b * bs; p < (b + 1) * bs - 1 && p < n; ++p)", SELECT),
    ("query_token_not_visible", "return qpos < 0 ? 0 : (qpos + 1) / ratio;", "return qpos < 0 ? 0 : qpos / ratio;",
     SELECT + ATTN),
    ("reindex_ignores_causality", "if (q < vis) p[n++] = q;", "p[n++] = q;", SELECT),
    ("window_one_key_short", "must be visible (R12) */\n    int64_t lo = qpos - win + 1;",
     "must be visible (R12) */\n    int64_t lo = qpos - win + 2;", ATTN),
    ("main_v_from_k_half", "memcpy(V + nk * 128, row + 128, 128 * sizeof(double));",
     "memcpy(V + nk * 128, row, 128 * sizeof(double));", ATTN),
    ("window_v_from_k_half", "V[nk * 128 + d] = orc_e4m3_decode(e[128 + d]);",
     "V[nk * 128 + d] = orc_e4m3_decode(e[d]);", ATTN),
    ("lse_without_max", "out[h * 128 + d] / l : 0.0;\n        lse[h] = (nk > 0) ? m + log(l) : -INFINITY;",
     "out[h * 128 + d] / l : 0.0;\n        lse[h] = (nk > 0) ? log(l) : -INFINITY;", ATTN),
    ("attention_skips_last_selected", "for (int j = 0; j < k; ++j) {\n        if (idx[j] < 0) continue;\n"
     "        if (idx[j] >= vis || idx[j] >= c->cap)", "for (int j = 0; j < k - 1; ++j) {\n        if (idx[j] < 0) "
     "continue;\n        if (idx[j] >= vis || idx[j] >= c->cap)", ATTN),
    # the pages' own shapes: MXFP4 indexer key, 32 x 128 MQA indexer, 512-channel latent attention
    ("mx_scale_exponent_off_by_one", "sbyte = (e2 - 1) - 2 + 127;", "sbyte = (e2 - 1) - 1 + 127;", PAGES),
    ("mx_zero_block_scale_one", "int sbyte = 0;\n            if (amax > 0.0) {",
     "int sbyte = 127;\n            if (amax > 0.0) {", PAGES),
    ("mx_nibbles_swapped", "data[r * (ch / 2) + 16 * b + i / 2] = (uint8_t)(c0 | (c1 << 4));",
     "data[r * (ch / 2) + 16 * b + i / 2] = (uint8_t)(c1 | (c0 << 4));", PAGES),
    ("mx_scale_read_as_e4m3", "orc_e2m1_decode(code) * orc_e8m0_decode(scale[r * nb + c / 32]);",
     "orc_e2m1_decode(code) * orc_e4m3_decode(scale[r * nb + c / 32]);", PAGES),
    ("mx_entry_bytes_scale_per_16", "return ch / 2 + ch / 32;", "return ch / 2 + ch / 16;", PAGES),
    ("mx_query_not_quantised", "orc_mx_dequant_rows(qdata, qscale, hi, 128, qd);",
     "for (int i = 0; i < hi * 128; ++i) qd[i] = bf16_to_double(idx_q[i]);", PAGES),
    ("mx_relu_ignored", "dot += qd[h * 128 + c] * kd[c];\n            total += (relu && dot < 0.0) ? 0.0 : dot;",
     "dot += qd[h * 128 + c] * kd[c];\n            total += dot;", PAGES),
    ("latent_window_one_key_short", "const int64_t vis = orc_visible(qpos, ratio);\n    int64_t lo = qpos - win + 1;",
     "const int64_t vis = orc_visible(qpos, ratio);\n    int64_t lo = qpos - win + 2;", PAGES),
    ("latent_skips_last_selected", "for (int j = 0; j < k; ++j) {\n        if (idx[j] < 0) continue;\n"
     "        if (idx[j] >= vis || idx[j] >= cap)", "for (int j = 0; j < k - 1; ++j) {\n        if (idx[j] < 0) "
     "continue;\n        if (idx[j] >= vis || idx[j] >= cap)", PAGES),
    ("latent_window_channels_swapped", "L[nk * 512 + d] = orc_e4m3_decode(e[d]);",
     "L[nk * 512 + d] = orc_e4m3_decode(e[d ^ 1]);", PAGES),
    ("latent_lse_without_max", "out[h * 512 + d] / l : 0.0;\n        lse[h] = (nk > 0) ? m + log(l) : -INFINITY;",
     "out[h * 512 + d] / l : 0.0;\n        lse[h] = (nk > 0) ? log(l) : -INFINITY;", PAGES),
]


def _gcc_flags():
    sys.path.insert(0, ROOT)
    import oracle

    return oracle.GCC_FLAGS


def _build(text, path):
    c = path + ".c"
    with open(c, "w") as f:
        f.write(text)
    subprocess.check_call(["gcc", *_gcc_flags(), "-o", path + ".so", c, "-lm"])
    return path + ".so"


def _pins(lib, files):
    env = dict(os.environ, CSA2_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", *files, "-x", "-q", "-p", "no:cacheprovider", "-m",
                        "not gpu"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-1500:]


@pytest.fixture(scope="module")
def outcomes():
    """Builds the control and every mutant, and runs their pins, several at a time."""
    with open(SRC) as f:
        src = f.read()
    res = {}
    with tempfile.TemporaryDirectory() as d:
        jobs = {"control": (src, CODEC + SELECT + ATTN + PAGES)}
        for mid, old, new, files in MUTANTS:
            n = src.count(old)
            if n != 1:
                res[mid] = ("snippet", f"the text to mutate occurs {n} times in csa2_oracle.c")
                continue
            jobs[mid] = (src.replace(old, new), files)

        def run(item):
            mid, (text, files) = item
            return mid, _pins(_build(text, os.path.join(d, mid)), files)

        with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            for mid, out in ex.map(run, jobs.items()):
                res[mid] = out
    return res


def test_control_build_passes_the_pins(outcomes):
    rc, out = outcomes["control"]
    assert rc == 0, out


@pytest.mark.parametrize("mid", [m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(outcomes, mid):
    rc, out = outcomes[mid]
    assert rc == 1, f"{mid}: pins exited {rc}\n{out}"
