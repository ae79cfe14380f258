/*
 * csa2_oracle.c -- plain, slow CPU oracle for one CSA2 layer step over an FP4 KV cache.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference leg load this library. It shares no code, header, table or helper with the
 * CUDA path under compressed_sparse_attention_append_b200/, and it never reads anything the
 * CUDA path produced.
 *
 * Sources (cited below by tag and section):
 *   [A] "DeepSeek-V4.1-Flash: Shrinking KV Cache at 552B Scale" (visualisation captions page)
 *   [B] "DeepSeek Cuts KV Cache Footprint Fourfold" (paper summary page), "Technical Approach"
 *   [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token"
 *       (engineering article), sections VI, VII, IX, XI, XII
 *
 * Arithmetic: fp64 throughout. Codec decisions are taken on fp64 quotients; the quotients
 * x/s and amax/6 can never sit within fp64 rounding distance of an E2M1/E4M3 rounding
 * boundary without sitting exactly on it (x has 8 significant bits, s has 4), so the
 * decisions equal those of exact rational arithmetic. Index scores are sums of products
 * that are multiples of 2^-20 with magnitude below 2^31, so fp64 sums are exact in any order.
 *
 * Readings of the pages where the sources leave a step open; "(Rn)" marks where each applies:
 *   R1  scale s = E4M3_RNE_satfinite(amax / 6); s == 0 gives all-zero codes; element code =
 *       E2M1_RNE_satfinite(x / s), sign kept (a negative value rounding to 0 gives code 0x8).
 *   R2  index score = sum over the 4 indexer heads of q_h . k_h on dequantised values; with the
 *       ReLU flag, sum over heads of max(0, q_h . k_h).
 *   R3  4 indexer key heads of 64 channels; query head h uses key head h * hk / hi.
 *   R4  the indexer query is quantised with the R1 codec before scoring.
 *   R5  ranking by score descending, ties to the lower position (lower block id for the pool).
 *   R6  selected positions are emitted ascending; fewer than k visible -> all, padded with -1.
 *   R7  one softmax over the selected FP4 rows and the FP8 window rows, no de-duplication,
 *       scale 1/sqrt(128), no sink.
 *   R8  window entries are E4M3 without a scale (RNE, satfinite); K = channels 0..127, V =
 *       128..255; a query at i sees window positions max(s, i - 127) .. i.
 *   R9  cache planes per sequence: packed codes (channel 2j in the low nibble of byte j) and
 *       one scale byte per 16 channels; an entry is ch/2 + ch/16 bytes.
 *   R10 pool = the top min(2048, ceil(N / 8)) blocks by their maximum visible score; block b
 *       covers positions 8b .. 8b+7.
 *   R11 a decode query sits at N - 1 and is appended before scoring (so it is visible);
 *       prefill row i sees positions <= i.
 *   R12 compression ratio r in {1, 2}: cache entry e summarises tokens r*e .. r*e + r - 1 and is
 *       visible to a query at token i once all of them are <= i, i.e. the first floor((i + 1) / r)
 *       entries; the window stays per token.
 *   R13 (the pages' own shapes) MXFP4 indexer key: per 32-channel block the shared E8M0 scale is
 *       X = 2^(floor(log2 amax) - 2), the microscaling rule for E2M1 elements (whose largest value
 *       is 1.5 * 2^2); elements E2M1_RNE_satfinite(x / X); amax == 0 gives scale byte 0 and +0 codes.
 *   R14 (the pages' own shapes) indexer of 32 query heads x 128 channels over ONE shared 128-channel
 *       key per entry (MQA); score = sum_h q_h . k (ReLU variant: sum_h max(0, q_h . k)); the query
 *       goes through the same MXFP4 codec as the keys.
 *   R15 (the pages' own shapes) attention over the 512-channel latent, which is both K and V, for
 *       64 query heads of 512 channels; the latent in the R1 codec (288 B per entry), window rows
 *       FP8 at 512 channels; one softmax over selected and window entries; scale 1/sqrt(512).
 *
 * Parity pins: every function here is checked by tests/test_oracle_*.py against exact
 * rational arithmetic, library routines (torch float8 conversion, Python sorted(), torch
 * fp64 softmax attention), closed forms and the byte figures printed in [C] sec. VII.
 * The R2/R3/R7 semantics (score formula, key heads, one softmax over selected + window)
 * are definitions stated here: no page figure can confirm them ("parity unpinned" as to
 * the pages; pinned as to the definitions stated here).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <fenv.h>

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------------------ */
/* Element formats. [A] last-but-one caption; [C] sec. XI "FP4 Main KV Cache": E2M1 elements, */
/* one E4M3 scale per 16 channels, no tensor-wide scale on top; SWA KV kept at FP8.        */
/* ------------------------------------------------------------------------------------ */

/* E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0. No inf/NaN. */
ORC_API double orc_e2m1_decode(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E4M3 (OFP8 "fn" variant): sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.
 * Exponent 15 with mantissa 7 is NaN; there is no infinity; max finite 448. */
ORC_API double orc_e4m3_decode(int byte)
{
    int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);             /* subnormal: m/8 * 2^-6 */
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round |a| to a multiple of `step` with ties to the even multiple (the current FP
 * rounding mode is round-to-nearest-even, which nearbyint uses). */
static double rne_multiple(double a, double step)
{
    return nearbyint(a / step) * step;
}

/* E2M1 encode, round-to-nearest-even with saturation to +-6 (R1). The sign is kept, so a
 * negative value (or -0) that rounds to zero gives code 0x8. Input must be finite. */
ORC_API int orc_e2m1_encode(double y)
{
    int sign = signbit(y) ? 8 : 0;
    double a = fabs(y), v, step;
    if (a >= 6.0) return sign | 7;
    /* binades: [0,2) step 0.5 (subnormal 0, 0.5 and normal 1, 1.5), [2,4) step 1, [4,8) step 2 */
    if (a < 2.0) step = 0.5;
    else if (a < 4.0) step = 1.0;
    else step = 2.0;
    v = rne_multiple(a, step);
    if (v > 6.0) v = 6.0;
    for (int c = 0; c < 8; ++c)
        if (orc_e2m1_decode(c) == v) return sign | c;
    return -1; /* unreachable */
}

/* E4M3 encode, round-to-nearest-even, saturating to +-448 ("satfinite"). Input finite. */
ORC_API int orc_e4m3_encode(double y)
{
    int sign = signbit(y) ? 0x80 : 0;
    double a = fabs(y), r, step;
    int e2, code;
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) step = ldexp(1.0, -9);       /* subnormal spacing */
    else { frexp(a, &e2); step = ldexp(1.0, (e2 - 1) - 3); } /* binade [2^(e2-1), 2^e2), 3 mantissa bits */
    r = rne_multiple(a, step);
    if (r > 448.0) r = 448.0;
    if (r < ldexp(1.0, -6)) {
        code = (int)(r / ldexp(1.0, -9));                 /* 0..7; 8 would be the min normal */
    } else {
        frexp(r, &e2);
        int E = e2 - 1;
        int m = (int)(r / ldexp(1.0, E) * 8.0) - 8;
        code = ((E + 7) << 3) | m;
    }
    return sign | code;
}

/* bf16 bit pattern -> exact double. */
static double bf16_to_double(uint16_t h)
{
    union { uint32_t u; float f; } v;
    v.u = (uint32_t)h << 16;
    return (double)v.f;
}

ORC_API double orc_bf16_to_double(uint16_t h) { return bf16_to_double(h); }

/* [C] sec. VII: bytes per cached entry of `ch` channels stored as E2M1 plus one 1-byte
 * E4M3 scale per 16 channels = ch/2 + ch/16. Returns 0 when ch is not a multiple of 16. */
ORC_API int64_t orc_entry_bytes(int ch)
{
    if (ch <= 0 || ch % 16) return 0;
    return ch / 2 + ch / 16;
}

/* ------------------------------------------------------------------------------------ */
/* Quantiser (R1): per row, per 16-channel block: amax = max|x|, s = E4M3_RNE(amax / 6),   */
/* code_i = E2M1_RNE(x_i / s); s == 0 gives all-zero codes. Packing (R9): channel 2j in the */
/* low nibble of byte j, channel 2j+1 in the high nibble; scale byte b for block b.        */
/* ------------------------------------------------------------------------------------ */
ORC_API void orc_quantize_rows(const uint16_t* x, int64_t rows, int ch, uint8_t* data, uint8_t* scale)
{
    int nb = ch / 16;
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* xr = x + r * ch;
        uint8_t* dr = data + r * (ch / 2);
        uint8_t* sr = scale + r * nb;
        for (int b = 0; b < nb; ++b) {
            double amax = 0.0;
            for (int i = 0; i < 16; ++i) {
                double v = fabs(bf16_to_double(xr[16 * b + i]));
                if (v > amax) amax = v;
            }
            int sc = orc_e4m3_encode(amax / 6.0);
            double s = orc_e4m3_decode(sc);
            sr[b] = (uint8_t)sc;
            for (int i = 0; i < 16; i += 2) {
                int c0 = 0, c1 = 0;
                if (s != 0.0) {
                    c0 = orc_e2m1_encode(bf16_to_double(xr[16 * b + i]) / s);
                    c1 = orc_e2m1_encode(bf16_to_double(xr[16 * b + i + 1]) / s);
                }
                dr[8 * b + i / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    }
}

/* SWA entries (R8): each bf16 value rounded to E4M3 (RNE, satfinite), no scale. */
ORC_API void orc_fp8_rows(const uint16_t* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)orc_e4m3_encode(bf16_to_double(x[i]));
}

/* Dequantise packed rows: v = E2M1(code) * E4M3(scale). [C] sec. XI: cached values are
 * dequantised before attention. */
ORC_API void orc_dequant_rows(const uint8_t* data, const uint8_t* scale, int64_t rows, int ch, double* out)
{
    int nb = ch / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int c = 0; c < ch; ++c) {
            uint8_t byte = data[r * (ch / 2) + c / 2];
            int code = (c & 1) ? (byte >> 4) : (byte & 15);
            out[r * ch + c] = orc_e2m1_decode(code) * orc_e4m3_decode(scale[r * nb + c / 16]);
        }
}

/* ------------------------------------------------------------------------------------ */
/* Cache of one sequence (R9 layout; planes owned by the caller).                          */
/* ------------------------------------------------------------------------------------ */
typedef struct {
    uint8_t* kv_data;   /* [cap][128]   main K||V, 256 channels FP4            */
    uint8_t* kv_scale;  /* [cap][16]    E4M3 scale per 16 channels            */
    uint8_t* ik_data;   /* [cap][hk*32] indexer keys, hk heads x 64 channels  */
    uint8_t* ik_scale;  /* [cap][hk*4]                                        */
    uint8_t* swa;       /* [swa_cap][256] FP8 E4M3 K||V ring, slot = pos & (swa_cap-1) */
    int64_t cap;
    int64_t swa_cap;
    int hk;
} orc_seq_cache;

/* Quantise-append of t new tokens at positions pos..pos+t-1 (R11). [C] sec. XI: keys are
 * quantised after RoPE, i.e. the inputs here are post-RoPE values. [B] "Technical
 * Approach": Full mode writes main KV and indexer keys; Reindex and Minimal write only
 * their own sliding-window KV (NULL planes are skipped). */
ORC_API int orc_quantize_append(const orc_seq_cache* c, int64_t pos, int t, const uint16_t* kv,
                                const uint16_t* idx_k, const uint16_t* swa_kv)
{
    if (pos < 0 || pos + t > c->cap) return -1;
    if (kv) orc_quantize_rows(kv, t, 256, c->kv_data + pos * 128, c->kv_scale + pos * 16);
    if (idx_k) orc_quantize_rows(idx_k, t, c->hk * 64, c->ik_data + pos * c->hk * 32, c->ik_scale + pos * c->hk * 4);
    if (swa_kv)
        for (int i = 0; i < t; ++i) {
            int64_t slot = (pos + i) & (c->swa_cap - 1);
            orc_fp8_rows(swa_kv + (int64_t)i * 256, 256, c->swa + slot * 256);
        }
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* Index score (R2, R3, R4). The indexer query (4 heads x 64) is quantised with the same   */
/* codec ([C] sec. XI: FP4 indexer queries and keys). score(p) = sum_h q_h . k_{p, g(h)}    */
/* on dequantised values, g(h) = h * hk / hi; relu != 0 gives sum_h max(0, q_h . k).       */
/* ------------------------------------------------------------------------------------ */
static double score_one(const double* qd /*[hi*64]*/, int hi, const uint8_t* kd, const uint8_t* ks,
                        int hk, int relu)
{
    double total = 0.0, kv[64];
    for (int h = 0; h < hi; ++h) {
        int g = h * hk / hi;
        orc_dequant_rows(kd + g * 32, ks + g * 4, 1, 64, kv);
        double dot = 0.0;
        for (int c = 0; c < 64; ++c) dot += qd[h * 64 + c] * kv[c];
        total += (relu && dot < 0.0) ? 0.0 : dot;
    }
    return total;
}

ORC_API void orc_quantize_index_query(const uint16_t* idx_q, int hi, uint8_t* qdata, uint8_t* qscale)
{
    orc_quantize_rows(idx_q, hi, 64, qdata, qscale);
}

/* Exact scores of positions p[0..n) for one quantised query. */
ORC_API void orc_scores(const orc_seq_cache* c, const uint16_t* idx_q, int hi, const int64_t* p, int64_t n,
                        int relu, double* out)
{
    uint8_t qdata[32 * 16], qscale[4 * 16];
    double qd[64 * 16];
    orc_quantize_rows(idx_q, hi, 64, qdata, qscale);
    orc_dequant_rows(qdata, qscale, hi, 64, qd);
    for (int64_t i = 0; i < n; ++i)
        out[i] = score_one(qd, hi, c->ik_data + p[i] * c->hk * 32, c->ik_scale + p[i] * c->hk * 4, c->hk, relu);
}

/* ------------------------------------------------------------------------------------ */
/* Top-K (R5, R6): rank by score descending, ties to the lower position; keep min(k, n);   */
/* emit ascending positions, padded with -1. [B] "Technical Approach": Top-512 indices.     */
/* ------------------------------------------------------------------------------------ */
typedef struct { double s; int64_t p; } orc_pair;

static int cmp_rank(const void* a, const void* b)
{
    const orc_pair* x = (const orc_pair*)a; const orc_pair* y = (const orc_pair*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->p < y->p) ? -1 : (x->p > y->p);
}

static int cmp_i64(const void* a, const void* b)
{
    int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
    return (x < y) ? -1 : (x > y);
}

ORC_API int orc_topk(const double* scores, const int64_t* pos, int64_t n, int k, int32_t* out)
{
    orc_pair* v = (orc_pair*)malloc(sizeof(orc_pair) * (n > 0 ? n : 1));
    int64_t* sel = (int64_t*)malloc(sizeof(int64_t) * (k > 0 ? k : 1));
    for (int64_t i = 0; i < n; ++i) { v[i].s = scores[i]; v[i].p = pos[i]; }
    qsort(v, n, sizeof(orc_pair), cmp_rank);
    int m = (int)(n < k ? n : k);
    for (int i = 0; i < m; ++i) sel[i] = v[i].p;
    qsort(sel, m, sizeof(int64_t), cmp_i64);
    for (int i = 0; i < k; ++i) out[i] = (i < m) ? (int32_t)sel[i] : -1;
    free(v); free(sel);
    return m;
}

/* Block pool (R10). [C] sec. VI "Shortlist-of-a-shortlist" and sec. IX Figure 4: a block's
 * score is the largest score of its visible positions (`bs` positions per block), and the
 * best blocks, at most `pool_blocks` (2,048) of them, make up the candidate pool. Blocks rank by block score descending, ties to the lower block id; the pool is
 * emitted as ascending block ids. scores[p] for p in [0, n). */
ORC_API int orc_pool(const double* scores, int64_t n, int bs, int pool_blocks, int32_t* out)
{
    int64_t nblk = (n + bs - 1) / bs;
    double* bsc = (double*)malloc(sizeof(double) * (nblk > 0 ? nblk : 1));
    int64_t* ids = (int64_t*)malloc(sizeof(int64_t) * (nblk > 0 ? nblk : 1));
    for (int64_t b = 0; b < nblk; ++b) {
        double m = -INFINITY;
        for (int64_t p = b * bs; p < (b + 1) * bs && p < n; ++p) if (scores[p] > m) m = scores[p];
        bsc[b] = m; ids[b] = b;
    }
    int32_t* tmp = (int32_t*)malloc(sizeof(int32_t) * (pool_blocks > 0 ? pool_blocks : 1));
    int m = orc_topk(bsc, ids, nblk, pool_blocks, tmp);
    memcpy(out, tmp, sizeof(int32_t) * pool_blocks);
    free(bsc); free(ids); free(tmp);
    return m;
}

/* Entries visible to a query at token qpos (R11, R12): entry e covers tokens ratio*e ..
 * ratio*e + ratio - 1, all of which must be <= qpos. */
static int64_t orc_visible(int64_t qpos, int ratio) { return qpos < 0 ? 0 : (qpos + 1) / ratio; }

/* Full mode index step for one query at token qpos (R11, R12: the visible entries are 0 ..
 * orc_visible - 1). [B] "Technical Approach"; [C] sec. VI "Shortlist-of-a-shortlist": scores
 * every causally visible entry, keeps Top-k, and (pool_blocks > 0) builds the block pool. */
ORC_API int orc_index_topk_full(const orc_seq_cache* c, int64_t qpos, const uint16_t* idx_q, int hi, int k,
                                int relu, int32_t* out_idx, int pool_blocks, int bs, int32_t* out_pool,
                                int32_t* out_pool_n, int ratio)
{
    int64_t n = orc_visible(qpos, ratio);
    int64_t* p = (int64_t*)malloc(sizeof(int64_t) * n);
    double* s = (double*)malloc(sizeof(double) * n);
    for (int64_t i = 0; i < n; ++i) p[i] = i;
    orc_scores(c, idx_q, hi, p, n, relu, s);
    int m = orc_topk(s, p, n, k, out_idx);
    if (pool_blocks > 0) *out_pool_n = orc_pool(s, n, bs, pool_blocks, out_pool);
    free(p); free(s);
    return m;
}

/* Reindex mode: [B] "Technical Approach" and [C] sec. VI: a fresh indexer query picks its
 * Top-k only among the pool's positions {bs*b .. bs*b+bs-1 : b in pool}, limited to the
 * entries visible at token qpos (R12). */
ORC_API int orc_index_topk_reindex(const orc_seq_cache* c, int64_t qpos, const uint16_t* idx_q, int hi,
                                   const int32_t* pool, int pool_n, int bs, int k, int relu, int32_t* out_idx,
                                   int ratio)
{
    const int64_t vis = orc_visible(qpos, ratio);
    int64_t* p = (int64_t*)malloc(sizeof(int64_t) * ((int64_t)pool_n * bs + 1));
    int64_t n = 0;
    for (int i = 0; i < pool_n; ++i)
        for (int j = 0; j < bs; ++j) {
            int64_t q = (int64_t)pool[i] * bs + j;
            if (q < vis) p[n++] = q;
        }
    double* s = (double*)malloc(sizeof(double) * (n + 1));
    orc_scores(c, idx_q, hi, p, n, relu, s);
    int m = orc_topk(s, p, n, k, out_idx);
    free(p); free(s);
    return m;
}

/* ------------------------------------------------------------------------------------ */
/* Sparse attention (R7, R8). [C] sec. VI "What one layer looks like": the layer's own     */
/* query attends to the selected entries of the shared main KV plus its own recent window. */
/* [C] sec. XII: with a replay start s, a query at i sees window keys [max(s, i-win+1), i].*/
/* One softmax over both key sets, 16 query heads sharing one KV head, channels 0..127 are */
/* K and 128..255 are V in both the FP4 main entry and the FP8 window entry.               */
/* ------------------------------------------------------------------------------------ */
ORC_API int orc_sparse_attend(const orc_seq_cache* c, int64_t qpos, const uint16_t* q /*[hq][128]*/, int hq,
                              const int32_t* idx, int k, int64_t swa_begin, int win, double sm_scale,
                              double* out /*[hq][128]*/, double* lse /*[hq]*/, int ratio)
{
    const int64_t vis = orc_visible(qpos, ratio);  /* selected entries must be visible (R12) */
    int64_t lo = qpos - win + 1;
    if (lo < swa_begin) lo = swa_begin;
    if (lo < 0) lo = 0;
    int nw = (int)(qpos - lo + 1);
    if (nw < 0) nw = 0;
    int nk = 0;
    double* K = (double*)malloc(sizeof(double) * 128 * (k + nw + 1));
    double* V = (double*)malloc(sizeof(double) * 128 * (k + nw + 1));
    double row[256];
    for (int j = 0; j < k; ++j) {
        if (idx[j] < 0) continue;
        if (idx[j] >= vis || idx[j] >= c->cap) { free(K); free(V); return -1; }
        orc_dequant_rows(c->kv_data + (int64_t)idx[j] * 128, c->kv_scale + (int64_t)idx[j] * 16, 1, 256, row);
        memcpy(K + nk * 128, row, 128 * sizeof(double));
        memcpy(V + nk * 128, row + 128, 128 * sizeof(double));
        ++nk;
    }
    for (int64_t p = lo; p <= qpos; ++p) {
        const uint8_t* e = c->swa + (p & (c->swa_cap - 1)) * 256;
        for (int d = 0; d < 128; ++d) { K[nk * 128 + d] = orc_e4m3_decode(e[d]); V[nk * 128 + d] = orc_e4m3_decode(e[128 + d]); }
        ++nk;
    }
    double* lg = (double*)malloc(sizeof(double) * (nk + 1));
    for (int h = 0; h < hq; ++h) {
        double qh[128], m = -INFINITY, l = 0.0;
        for (int d = 0; d < 128; ++d) qh[d] = bf16_to_double(q[h * 128 + d]);
        for (int j = 0; j < nk; ++j) {
            double dot = 0.0;
            for (int d = 0; d < 128; ++d) dot += qh[d] * K[j * 128 + d];
            lg[j] = dot * sm_scale;
            if (lg[j] > m) m = lg[j];
        }
        for (int d = 0; d < 128; ++d) out[h * 128 + d] = 0.0;
        for (int j = 0; j < nk; ++j) {
            double pj = exp(lg[j] - m);
            l += pj;
            for (int d = 0; d < 128; ++d) out[h * 128 + d] += pj * V[j * 128 + d];
        }
        for (int d = 0; d < 128; ++d) out[h * 128 + d] = (nk > 0) ? out[h * 128 + d] / l : 0.0;
        lse[h] = (nk > 0) ? m + log(l) : -INFINITY;
    }
    free(K); free(V); free(lg);
    return nk;
}

/* ==================================================================================== */
/* The pages' own shapes ([C] sec. VII and the configuration list in its closing         */
/* section): a 512-channel main KV latent that serves as both K and V for 64 query heads  */
/* of dimension 512, and an indexer of 32 query heads of dimension 128 over ONE shared    */
/* 128-channel key stored in MXFP4 (E2M1 elements, one E8M0 scale per 32 channels).       */
/* ==================================================================================== */

/* E8M0 (the microscaling shared scale): 2^(byte - 127); 0xFF is NaN. */
ORC_API double orc_e8m0_decode(int byte)
{
    if ((byte & 0xFF) == 0xFF) return NAN;
    return ldexp(1.0, (byte & 0xFF) - 127);
}

/* [C] sec. VII: bytes of an MXFP4 entry of `ch` channels = ch/2 (E2M1) + ch/32 (one E8M0 byte
 * per 32 channels). Returns 0 when ch is not a multiple of 32. */
ORC_API int64_t orc_mx_entry_bytes(int ch)
{
    if (ch <= 0 || ch % 32) return 0;
    return ch / 2 + ch / 32;
}

/* MXFP4 quantiser (R13). Per 32-channel block: amax = max|x|; the shared scale is the power of
 * two X = 2^(floor(log2 amax) - 2) (2 = the exponent of E2M1's largest value 6 = 1.5 * 2^2), its
 * byte log2(X) + 127 clamped to 0..254; code_i = E2M1_RNE_satfinite(x_i / X) (x / X is exact).
 * amax == 0 gives scale byte 0 and all codes +0. Packing as R9 (channel 2j low nibble). */
ORC_API void orc_mx_quantize_rows(const uint16_t* x, int64_t rows, int ch, uint8_t* data, uint8_t* scale)
{
    int nb = ch / 32;
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* xr = x + r * ch;
        for (int b = 0; b < nb; ++b) {
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double v = fabs(bf16_to_double(xr[32 * b + i]));
                if (v > amax) amax = v;
            }
            int sbyte = 0;
            if (amax > 0.0) {
                int e2;
                frexp(amax, &e2);                 /* amax in [2^(e2-1), 2^e2): floor(log2) = e2-1 */
                sbyte = (e2 - 1) - 2 + 127;
                if (sbyte < 0) sbyte = 0;
                if (sbyte > 254) sbyte = 254;
            }
            scale[r * nb + b] = (uint8_t)sbyte;
            double X = orc_e8m0_decode(sbyte);
            for (int i = 0; i < 32; i += 2) {
                int c0 = 0, c1 = 0;
                if (amax > 0.0) {
                    c0 = orc_e2m1_encode(bf16_to_double(xr[32 * b + i]) / X);
                    c1 = orc_e2m1_encode(bf16_to_double(xr[32 * b + i + 1]) / X);
                }
                data[r * (ch / 2) + 16 * b + i / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    }
}

/* Dequantise MXFP4 rows: v = E2M1(code) * E8M0(scale of the code's 32-channel block). */
ORC_API void orc_mx_dequant_rows(const uint8_t* data, const uint8_t* scale, int64_t rows, int ch, double* out)
{
    int nb = ch / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int c = 0; c < ch; ++c) {
            uint8_t byte = data[r * (ch / 2) + c / 2];
            int code = (c & 1) ? (byte >> 4) : (byte & 15);
            out[r * ch + c] = orc_e2m1_decode(code) * orc_e8m0_decode(scale[r * nb + c / 32]);
        }
}

/* Indexer of the pages' shape (R14): the query (hi heads x 128 channels) goes through the same
 * MXFP4 codec as the keys; score(p) = sum_h q_h . k_p over the ONE shared key of entry p (MQA);
 * relu != 0 gives sum_h max(0, q_h . k_p). Keys: kdata [cap][64], kscale [cap][4]. Scores the
 * entries visible at token qpos (R11, R12) and keeps the Top-k as orc_topk does (R5, R6). */
ORC_API int orc_mx_index_topk_full(const uint8_t* kdata, const uint8_t* kscale, int64_t cap, int64_t qpos,
                                   const uint16_t* idx_q, int hi, int k, int relu, int32_t* out_idx, double* out_scores,
                                   int ratio)
{
    int64_t n = orc_visible(qpos, ratio);
    if (n > cap || hi <= 0 || hi > 64) return -1;
    uint8_t qdata[64 * 64], qscale[64 * 4];
    double qd[64 * 128], kd[128];
    orc_mx_quantize_rows(idx_q, hi, 128, qdata, qscale);
    orc_mx_dequant_rows(qdata, qscale, hi, 128, qd);
    int64_t* p = (int64_t*)malloc(sizeof(int64_t) * (n > 0 ? n : 1));
    double* s = (double*)malloc(sizeof(double) * (n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) {
        p[i] = i;
        orc_mx_dequant_rows(kdata + i * 64, kscale + i * 4, 1, 128, kd);
        double total = 0.0;
        for (int h = 0; h < hi; ++h) {
            double dot = 0.0;
            for (int c = 0; c < 128; ++c) dot += qd[h * 128 + c] * kd[c];
            total += (relu && dot < 0.0) ? 0.0 : dot;
        }
        s[i] = total;
        if (out_scores) out_scores[i] = total;
    }
    int m = orc_topk(s, p, n, k, out_idx);
    free(p); free(s);
    return m;
}

/* Attention of the pages' shape (R15): the 512-channel latent is both K and V. Main entries:
 * ldata [cap][256] E2M1 codes + lscale [cap][32] E4M3 scales (the R1 codec at 512 channels,
 * 288 B per entry); window entries: swa [swa_cap][512] E4M3 without scale, slot = pos &
 * (swa_cap - 1). A query at token qpos with hq heads of 512 channels attends, in ONE softmax,
 * to the selected entries (idx, -1 skipped; each must be visible, R12) and the window tokens
 * [max(swa_begin, qpos - win + 1), qpos]; logits (q_h . l_j) * sm_scale; out_h = sum_j p_j l_j. */
ORC_API int orc_latent_attend(const uint8_t* ldata, const uint8_t* lscale, int64_t cap, const uint8_t* swa,
                              int64_t swa_cap, int64_t qpos, const uint16_t* q /*[hq][512]*/, int hq,
                              const int32_t* idx, int k, int64_t swa_begin, int win, double sm_scale,
                              double* out /*[hq][512]*/, double* lse /*[hq]*/, int ratio)
{
    const int64_t vis = orc_visible(qpos, ratio);
    int64_t lo = qpos - win + 1;
    if (lo < swa_begin) lo = swa_begin;
    if (lo < 0) lo = 0;
    int nw = (int)(qpos - lo + 1);
    if (nw < 0) nw = 0;
    double* L = (double*)malloc(sizeof(double) * 512 * (k + nw + 1));
    int nk = 0;
    for (int j = 0; j < k; ++j) {
        if (idx[j] < 0) continue;
        if (idx[j] >= vis || idx[j] >= cap) { free(L); return -1; }
        orc_dequant_rows(ldata + (int64_t)idx[j] * 256, lscale + (int64_t)idx[j] * 32, 1, 512, L + nk * 512);
        ++nk;
    }
    for (int64_t p = lo; p <= qpos; ++p) {
        const uint8_t* e = swa + (p & (swa_cap - 1)) * 512;
        for (int d = 0; d < 512; ++d) L[nk * 512 + d] = orc_e4m3_decode(e[d]);
        ++nk;
    }
    double* lg = (double*)malloc(sizeof(double) * (nk + 1));
    for (int h = 0; h < hq; ++h) {
        double m = -INFINITY, l = 0.0;
        for (int j = 0; j < nk; ++j) {
            double dot = 0.0;
            for (int d = 0; d < 512; ++d) dot += bf16_to_double(q[h * 512 + d]) * L[j * 512 + d];
            lg[j] = dot * sm_scale;
            if (lg[j] > m) m = lg[j];
        }
        for (int d = 0; d < 512; ++d) out[h * 512 + d] = 0.0;
        for (int j = 0; j < nk; ++j) {
            double pj = exp(lg[j] - m);
            l += pj;
            for (int d = 0; d < 512; ++d) out[h * 512 + d] += pj * L[j * 512 + d];
        }
        for (int d = 0; d < 512; ++d) out[h * 512 + d] = (nk > 0) ? out[h * 512 + d] / l : 0.0;
        lse[h] = (nk > 0) ? m + log(l) : -INFINITY;
    }
    free(L); free(lg);
    return nk;
}
