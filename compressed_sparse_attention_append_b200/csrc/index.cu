// index.cu -- indexer scoring and exact Top-k selection for several query rows per sequence (the
// prefill chunk, where row i of a chunk sees positions <= i, and multi-token decode, where the
// draft tokens of a sequence are verified together). Rows of one query per sequence (decode: Full
// with its block pool, and Reindex) run in index_decode.cu.
//
// [B] "DeepSeek Cuts KV Cache Footprint Fourfold", "Technical Approach": Full mode computes the
// Top-K indices. [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token",
// sec. IX (the indexer scores every visible position), sec. XI: indexer queries and keys are FP4.
//
// Score (the reading taken here; the pages give no formula): score(p) = sum_h q_h . k_{p,h} over 4
// heads x 64 channels of dequantised FP4 values, computed EXACTLY as the integer S = score * 2^20:
//   * an E2M1 code c decodes to the integer 2*value(c) in {0, +-1, +-2, +-3, +-4, +-6, +-8, +-12}
//     through a byte permute (prmt) of the table {0,1,2,3,4,6,8,12}: the permute's sign-replicate
//     mode turns the codes of one sign into 0, so one prmt of the codes gives the magnitudes of
//     the positive channels and one prmt of the sign-flipped codes those of the negative ones;
//   * a 16-channel block's dot product D = sum (2q)(2k) comes from dp4a (|D| <= 2304);
//   * an E4M3 scale s = M * 2^(E-10) (M <= 15, E >= 1) enters as the integer f(s) = M * 2^(E-1)
//     (<= 448 * 2^9 = 229376); D * f(s_k) fits in int32 and (D * f(s_k)) * f(s_q) is added to an int64
//     with one wide multiply-add (each term < 2^47, the sum of 16 terms < 2^51).
// No floating-point conversion runs in the scoring loop. Ranking is by S descending, ties to the
// lower position; S is the same integer the exact rational score gives, so the selected set is
// unique and reproducible.
//
// Structure (one kernel, persistent CTAs taking work items from an atomic counter):
//   item = (chunk of 8-position units, query row), chunk-major so that later chunks of a row start
//   with the admission threshold left by its earlier chunks. Each warp scores four units per step
//   (32 positions, 4 KB of keys + 512 B of scales) from a private 2-stage cp.async ring; a running
//   local Top-k sits in shared memory (admission threshold + radix select over orderable keys,
//   skipping the bits all keys share and histogramming with match_any). A CTA emits its local
//   Top-k to the row's candidate list; the CTA that finishes a row's last chunk merges the
//   candidates into the final ascending outputs and clears the row's counters.
#include "csa2_internal.cuh"

namespace csa2 {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 2;
constexpr int kUnitsPerStep = 4;                      // units scored by one warp step (32 positions)
constexpr int kStepBytes = kUnitsPerStep * (1024 + 128);  // codes + scales of 4 units
constexpr int kStagingBytes = kWarps * kStages * kStepBytes;
constexpr int kStepsPerFlush = 4;                     // warp steps between two selection flushes
constexpr int kSubUnits = kWarps * kUnitsPerStep * kStepsPerFlush;  // 128 units
constexpr int kNewCap = kSubUnits * kBS;              // admissions per sub-chunk, worst case

struct SelBuf {
    unsigned long long* keep_key[2];
    int* keep_pos[2];
    unsigned long long* new_key;
    int* new_pos;
};

struct __align__(16) Scal {
    int cur, nkeep, nnew, digit, above, cnt, last, misc;
    unsigned long long thr, prefix, red_and[kWarps], red_or[kWarps];
    int qf[16];
    __align__(16) uint8_t qcode[128];
    __align__(16) uint32_t qv[128];   // [chunk s][word i][pa, pb, na, nb]
};

// ---- integer decode of E2M1 codes -------------------------------------------------------------
// prmt with the table bytes {0,1,2,3,4,6,8,12}: selector nibble = code; a set sign bit selects the
// sign-replicate mode, whose result is 0 because every table byte is positive.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
constexpr uint32_t kTab0 = 0x03020100u, kTab1 = 0x0C080604u;

// sum over the 8 channels of word w of (2q)(2k); qa/qb = 2q of channels 0..3 / 4..7 as int8x4
__device__ __forceinline__ int dot8(uint32_t w, uint32_t qa, uint32_t qb, uint32_t nqa, uint32_t nqb, int acc) {
    const uint32_t wx = w ^ 0x88888888u;
    acc = __dp4a((int)prmt(kTab0, kTab1, w), (int)qa, acc);
    acc = __dp4a((int)prmt(kTab0, kTab1, wx), (int)nqa, acc);
    acc = __dp4a((int)prmt(kTab0, kTab1, w >> 16), (int)qb, acc);
    acc = __dp4a((int)prmt(kTab0, kTab1, wx >> 16), (int)nqb, acc);
    return acc;
}

// f(s) = M * 2^(E-1) for an E4M3 byte (value M * 2^(E-10)); sign applied; NaN codes give 0.
__device__ __forceinline__ int e4m3_fixed(int byte) {
    const int e = (byte >> 3) & 15, m = byte & 7;
    if (e == 15 && m == 7) return 0;
    const int M = e ? (8 | m) : m;
    const int v = M << (e ? e - 1 : 0);
    return (byte & 0x80) ? -v : v;
}

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m) {
    return __shfl_xor_sync(0xffffffffu, v, m);
}
__device__ __forceinline__ long long shfl_xor_s64(long long v, int m) { return __shfl_xor_sync(0xffffffffu, v, m); }

// ---- query quantisation (same codec as the cache), 8 threads per 16-channel block ---------------
__device__ __forceinline__ uint32_t q_f32x2_to_e2m1x2(float lo, float hi) {
    uint16_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\tmov.b16 %0, {t, 0};\n\t}"
        : "=h"(r) : "f"(lo), "f"(hi));
    return r & 0xFF;
}
__device__ __forceinline__ uint32_t q_f32_to_e4m3(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(r) : "f"(v), "f"(0.f));
    return r & 0xFF;
}

__device__ void quantize_query(const uint16_t* q, Scal& S, const int* kf_lut) {
    const int t = threadIdx.x;
    if (t < 128) {
        const int blk = t >> 3, sub = t & 7;  // 2 channels per thread
        const uint32_t w = *reinterpret_cast<const uint32_t*>(q + blk * 16 + 2 * sub);
        const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xFFFF0000u);
        float amax = fmaxf(fabsf(x0), fabsf(x1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        const uint32_t sc = q_f32_to_e4m3(__fdiv_rn(amax, 6.0f));
        const float s = __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)sc, __NV_E4M3)));
        S.qcode[blk * 8 + sub] = (s == 0.f) ? 0 : (uint8_t)q_f32x2_to_e2m1x2(__fdiv_rn(x0, s), __fdiv_rn(x1, s));
        if (sub == 0) S.qf[blk] = kf_lut[sc];
    }
}

// 2 * value of an E2M1 code as a signed byte
__device__ __forceinline__ uint32_t e2m1_int2(uint32_t c) {
    const uint32_t mag = (prmt(kTab0, kTab1, c & 7) & 0xFF);
    return (c & 8) ? ((0u - mag) & 0xFF) : mag;
}

// ---- CTA radix select ----------------------------------------------------------------------------
// Elements i < na: (ka, pa); the rest: (kb, pb). Writes the top K (key desc, pos asc) into (ko, po);
// S.thr becomes a lower bound of the kept keys.
__device__ void cta_select(const unsigned long long* ka, const int* pa, int na, const unsigned long long* kb,
                           const int* pb, int nb, int K, unsigned long long* ko, int* po, unsigned int* hist,
                           Scal& S) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = na + nb;
    auto key_at = [&](int i) { return i < na ? ka[i] : kb[i - na]; };
    auto pos_at = [&](int i) { return i < na ? pa[i] : pb[i - na]; };
    // bits shared by every key are skipped
    unsigned long long va = ~0ull, vo = 0ull;
    for (int i = tid; i < n; i += kThreads) { const unsigned long long k = key_at(i); va &= k; vo |= k; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) { va &= shfl_xor_u64(va, o); vo |= shfl_xor_u64(vo, o); }
    if (lane == 0) { S.red_and[warp] = va; S.red_or[warp] = vo; }
    __syncthreads();
    va = ~0ull; vo = 0ull;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) { va &= S.red_and[w]; vo |= S.red_or[w]; }
    const unsigned long long diff = va ^ vo;
    int top = diff ? 63 - __clzll((long long)diff) : -1;
    unsigned long long mask = (top >= 63) ? 0ull : ~((2ull << top) - 1ull);
    unsigned long long prefix = va & mask;
    if (top < 0) { mask = ~0ull; prefix = va; }
    int kr = K;
    bool exact = false;
    while (top >= 0) {
        const int shift = top >= 7 ? top - 7 : 0;
        const int nbits = top - shift + 1;
        const unsigned int dmask = (1u << nbits) - 1u;
        hist[tid] = 0;
        __syncthreads();
        for (int base = 0; base < n; base += kThreads) {
            const int i = base + tid;
            int d = -1;
            if (i < n) {
                const unsigned long long key = key_at(i);
                if ((key & mask) == prefix) d = (int)((key >> shift) & dmask);
            }
            const unsigned int peers = __match_any_sync(0xffffffffu, d);
            if (d >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (unsigned)__popc(peers));
        }
        __syncthreads();
        if (warp == 0) {
            // lane L owns bins 255-8L ... 248-8L (descending)
            unsigned int c[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { c[j] = hist[255 - 8 * lane - j]; sum += c[j]; }
            unsigned int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const unsigned int excl = incl - sum;
            if (excl < (unsigned)kr && incl >= (unsigned)kr) {
                unsigned int run = excl;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (run + c[j] >= (unsigned)kr) {
                        S.digit = 255 - 8 * lane - j;
                        S.above = (int)run;
                        S.cnt = (int)c[j];
                        break;
                    }
                    run += c[j];
                }
            }
        }
        __syncthreads();
        kr -= S.above;
        prefix |= (unsigned long long)S.digit << shift;
        mask |= (unsigned long long)dmask << shift;
        exact = (S.cnt == kr);
        top = shift - 1;
        __syncthreads();
        if (exact) break;
    }
    // all keys equal down to the last bit: the kr lowest positions among key == prefix
    unsigned int pthr = 0xFFFFFFFFu;
    if (!exact) {
        unsigned int pp = 0, pm = 0;
        int r = kr;
        for (int shift = 24; shift >= 0; shift -= 8) {
            hist[tid] = 0;
            __syncthreads();
            for (int base = 0; base < n; base += kThreads) {
                const int i = base + tid;
                int d = -1;
                if (i < n && key_at(i) == prefix) {
                    const unsigned int p = (unsigned int)pos_at(i);
                    if ((p & pm) == pp) d = (int)((p >> shift) & 255u);
                }
                const unsigned int peers = __match_any_sync(0xffffffffu, d);
                if (d >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (unsigned)__popc(peers));
            }
            __syncthreads();
            if (warp == 0) {
                unsigned int c[8], sum = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) { c[j] = hist[8 * lane + j]; sum += c[j]; }
                unsigned int incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned int v = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += v;
                }
                const unsigned int excl = incl - sum;
                if (excl < (unsigned)r && incl >= (unsigned)r) {
                    unsigned int run = excl;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (run + c[j] >= (unsigned)r) { S.digit = 8 * lane + j; S.above = (int)run; S.cnt = (int)c[j]; break; }
                        run += c[j];
                    }
                }
            }
            __syncthreads();
            r -= S.above;
            pp |= (unsigned int)S.digit << shift;
            pm |= 0xFFu << shift;
            const bool done = (S.cnt == r);
            __syncthreads();
            if (done) break;
        }
        pthr = pp | ~pm;
    }
    if (tid == 0) S.misc = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kThreads) {
        const int i = base + tid;
        bool sel = false;
        unsigned long long key = 0;
        int p = 0;
        if (i < n) {
            key = key_at(i);
            p = pos_at(i);
            sel = exact ? (key & mask) >= prefix : (key > prefix || (key == prefix && (unsigned int)p <= pthr));
        }
        const unsigned int bal = __ballot_sync(0xffffffffu, sel);
        int wbase = 0;
        if (lane == 0 && bal) wbase = atomicAdd(&S.misc, __popc(bal));
        wbase = __shfl_sync(0xffffffffu, wbase, 0);
        if (sel) {
            const int o = wbase + __popc(bal & ((1u << lane) - 1));
            ko[o] = key;
            po[o] = p;
        }
    }
    __syncthreads();
    if (tid == 0 && prefix > S.thr) S.thr = prefix;
    __syncthreads();
}

__device__ void flush(SelBuf& B, unsigned int* hist, Scal& S, int K) {
    const int nk = S.nkeep, nn = S.nnew, cur = S.cur;
    if (nn == 0) return;
    if (nk + nn <= K) {
        for (int i = threadIdx.x; i < nn; i += kThreads) {
            B.keep_key[cur][nk + i] = B.new_key[i];
            B.keep_pos[cur][nk + i] = B.new_pos[i];
        }
        __syncthreads();
        if (threadIdx.x == 0) { S.nkeep = nk + nn; S.nnew = 0; }
        __syncthreads();
        return;
    }
    cta_select(B.keep_key[cur], B.keep_pos[cur], nk, B.new_key, B.new_pos, nn, K, B.keep_key[cur ^ 1],
               B.keep_pos[cur ^ 1], hist, S);
    if (threadIdx.x == 0) { S.cur = cur ^ 1; S.nkeep = K; S.nnew = 0; }
    __syncthreads();
}

__device__ __forceinline__ void admit(SelBuf& B, Scal& S, bool valid, unsigned long long key, int pos) {
    const int lane = threadIdx.x & 31;
    const unsigned int bal = __ballot_sync(0xffffffffu, valid);
    if (!bal) return;
    int base = 0;
    if (lane == 0) base = atomicAdd(&S.nnew, __popc(bal));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (valid) {
        const int o = base + __popc(bal & ((1u << lane) - 1));
        B.new_key[o] = key;
        B.new_pos[o] = pos;
    }
}

// Ascending bitonic sort of n int32 values in `a` (room for the next power of two of n).
__device__ void sort_ascending(int* a, int n) {
    int P = 1;
    while (P < n) P <<= 1;
    for (int i = n + threadIdx.x; i < P; i += kThreads) a[i] = 0x7FFFFFFF;
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < P; i += kThreads) {
                const int l = i ^ j;
                if (l > i) {
                    const int x = a[i], y = a[l];
                    const bool up = (i & k) == 0;
                    if ((x > y) == up) { a[i] = y; a[l] = x; }
                }
            }
            __syncthreads();
        }
    }
}

struct RowInfo {
    int64_t qpos;
    int b;
    int n_units;
    bool ok;
};

__device__ RowInfo row_info(const IndexArgs& a, int row) {
    RowInfo r;
    r.b = row / a.tq;
    r.qpos = index_row_last(a, row);  // the last visible entry
    r.ok = r.qpos >= -1;
    if (!r.ok) {
        r.n_units = 0;
        return r;
    }
    r.n_units = (int)((r.qpos + kBS) / kBS);
    return r;
}

// Block id of unit u of row R (the unit itself) and its number of scoreable positions (0..8);
// -1 / 0 when the unit is past the chunk.
__device__ __forceinline__ void unit_info(const IndexArgs& a, const RowInfo& R, int u, int u_end, int& blk, int& nv) {
    blk = -1;
    nv = 0;
    if (u >= u_end) return;
    const int id = u;
    const int64_t p0 = (int64_t)id * kBS;
    int64_t n = R.qpos - p0 + 1;
    if (a.c.cap - p0 < n) n = a.c.cap - p0;
    if (n <= 0) return;
    blk = id;
    nv = n > kBS ? kBS : (int)n;
}

// One warp step: units u .. u+3. Lane u (< 4) resolves unit u; the result is broadcast.
// Staging: codes of unit j at 1024*j, scales at 4096 + 128*j.
__device__ __forceinline__ int stage_step(const IndexArgs& a, const RowInfo& R, int ustep, int u_end,
                                          unsigned char* st) {
    const int lane = threadIdx.x & 31;
    int blk = -1, nv = 0;
    if (lane < kUnitsPerStep) unit_info(a, R, ustep + lane, u_end, blk, nv);
    const int packed = (blk << 4) | nv;  // blk < 2^26 (cap <= 2^30 positions); -1 packs to -16
    const uint8_t* base = a.c.ik_data + (size_t)R.b * a.c.cap * kIKBytes;
    const uint8_t* sbase = a.c.ik_scale + (size_t)R.b * a.c.cap * kIKScales;
#pragma unroll
    for (int u = 0; u < kUnitsPerStep; ++u) {
        const int pk = __shfl_sync(0xffffffffu, packed, u);
        const int b = pk >> 4, n = pk & 15;
        if (b < 0) continue;
        const size_t row0 = (size_t)b * kBS;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int off = 512 * h + 16 * lane;  // position 4h + lane/8 of the unit
            if (4 * h + (lane >> 3) < n) cp_async16(st + 1024 * u + off, base + row0 * kIKBytes + off);
        }
        if ((lane >> 3) == u && (lane & 7) < n)
            cp_async16(st + 4096 + 128 * u + 16 * (lane & 7), sbase + (row0 + (lane & 7)) * kIKScales);
    }
    return packed;
}

// Scores the staged step (lane (m, s), load j: position (j&1)*4+m of unit j>>1, channels 32s..32s+31),
// reduce-scatters over the octet so that lane (m, s) holds the score of position (s&1)*4+m of unit s>>1.
template <bool RELU>
__device__ __forceinline__ void score_step(const unsigned char* st, int packed, int ustep, const uint32_t (&qv)[16],
                                           int qf0, int qf1, const int* kf_lut, SelBuf& B, Scal& S,
                                           unsigned long long thr) {
    const int lane = threadIdx.x & 31;
    const int m = lane >> 3, s = lane & 7;
    long long v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(st + 1024 * (j >> 1) + 512 * (j & 1) + 16 * lane);
        const uint32_t sc = *reinterpret_cast<const uint16_t*>(st + 4096 + 128 * (j >> 1) + 16 * ((j & 1) * 4 + m) + 2 * s);
        int d0 = dot8(w.x, qv[0], qv[1], qv[2], qv[3], 0);
        d0 = dot8(w.y, qv[4], qv[5], qv[6], qv[7], d0);
        int d1 = dot8(w.z, qv[8], qv[9], qv[10], qv[11], 0);
        d1 = dot8(w.w, qv[12], qv[13], qv[14], qv[15], d1);
        v[j] = (long long)(d0 * kf_lut[sc & 0xFF]) * qf0 + (long long)(d1 * kf_lut[sc >> 8]) * qf1;
    }
    if (RELU) {  // head s>>1 lives on lanes s and s^1
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            v[j] += shfl_xor_s64(v[j], 1);
            v[j] = (v[j] > 0 && (s & 1) == 0) ? v[j] : 0;
        }
    }
    // reduce-scatter over the octet: lane s ends with position j = s
    const bool b2 = s & 4, b1 = s & 2, b0 = s & 1;
    long long w4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const long long keep = b2 ? v[4 + i] : v[i], send = b2 ? v[i] : v[4 + i];
        w4[i] = keep + shfl_xor_s64(send, 4);
    }
    long long w2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const long long keep = b1 ? w4[2 + i] : w4[i], send = b1 ? w4[i] : w4[2 + i];
        w2[i] = keep + shfl_xor_s64(send, 2);
    }
    const long long keep = b0 ? w2[1] : w2[0], send = b0 ? w2[0] : w2[1];
    const long long x = keep + shfl_xor_s64(send, 1);
    // position of this lane
    const int u = s >> 1, idx = (s & 1) * 4 + m;
    const int pk = __shfl_sync(0xffffffffu, packed, u);
    const int blk = pk >> 4, nv = pk & 15;
    const bool valid = blk >= 0 && idx < nv;
    const unsigned long long key = valid ? ((unsigned long long)x ^ 0x8000000000000000ull) : 0ull;
    admit(B, S, valid && key >= thr, key, blk * kBS + idx);
}

__device__ void stream_select_global(const unsigned long long* gk, const int* gp, int n, unsigned long long tau,
                                     int K, SelBuf& B, unsigned int* hist, Scal& S, bool pos_is_index) {
    if (threadIdx.x == 0) { S.nkeep = 0; S.nnew = 0; S.cur = 0; S.thr = tau; }
    __syncthreads();
    for (int base = 0; base < n; base += kNewCap) {
        const unsigned long long thr = S.thr;
        const int cnt = min(kNewCap, n - base);
        for (int i0 = 0; i0 < cnt; i0 += kThreads) {
            const int i = i0 + threadIdx.x;
            bool v = false;
            unsigned long long key = 0;
            int p = 0;
            if (i < cnt) {
                key = gk[base + i];
                p = pos_is_index ? base + i : gp[base + i];
                v = key >= thr && key != 0ull;
            }
            admit(B, S, v, key, p);
        }
        __syncthreads();
        flush(B, hist, S, K);
    }
}

template <bool RELU>
__global__ void __launch_bounds__(kThreads, 2) index_kernel(IndexArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ Scal S;
    __shared__ unsigned int hist[256];
    __shared__ int kf_lut[256];
    const int K = a.plan.k;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // shared memory: staging ring | keep[2] | new
    unsigned char* staging = smem;
    SelBuf B;
    {
        unsigned char* p = smem + kStagingBytes;
        B.keep_key[0] = reinterpret_cast<unsigned long long*>(p); p += 8 * K;
        B.keep_key[1] = reinterpret_cast<unsigned long long*>(p); p += 8 * K;
        B.new_key = reinterpret_cast<unsigned long long*>(p); p += 8 * kNewCap;
        B.keep_pos[0] = reinterpret_cast<int*>(p); p += 4 * K;
        B.keep_pos[1] = reinterpret_cast<int*>(p); p += 4 * K;
        B.new_pos = reinterpret_cast<int*>(p);
    }
    kf_lut[tid] = e4m3_fixed(tid);
    __syncthreads();

    unsigned char* ws = a.ws;
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + kHdrStatus);
    unsigned int* next = reinterpret_cast<unsigned int*>(ws + kHdrIndexNext);
    unsigned int* done = reinterpret_cast<unsigned int*>(ws + kHdrIndexDone);
    RowCtr* rctr = reinterpret_cast<RowCtr*>(ws + a.L.row_ctr);
    unsigned long long* cand_key = reinterpret_cast<unsigned long long*>(ws + a.L.cand_key);
    int* cand_pos = reinterpret_cast<int*>(ws + a.L.cand_pos);
    // rows handed over by the tensor-core filter, or every row
    const int rows = a.row_list ? (int)*(volatile const uint32_t*)a.row_n : a.plan.rows;
    const int total = rows * a.plan.chunks;
    unsigned char* wst = staging + warp * kStages * kStepBytes;

    for (;;) {
        if (tid == 0) S.misc = (int)atomicAdd(next, 1u);
        __syncthreads();
        const int item = S.misc;
        __syncthreads();
        if (item >= total) break;
        const int chunk = item / rows;
        const int row = a.row_list ? a.row_list[item % rows] : item % rows;
        const RowInfo R = row_info(a, row);
        RowCtr* rc = rctr + row;
        if (!R.ok && chunk == 0 && tid == 0) set_status(status, CSA2_DEV_BAD_POS);
        const int u0 = chunk * a.plan.chunk_units;
        const int u1 = min(u0 + a.plan.chunk_units, R.n_units);
        if (tid == 0) {
            S.nkeep = 0; S.nnew = 0; S.cur = 0;
            S.thr = *(volatile unsigned long long*)&rc->tau;  // lower bound left by earlier chunks
        }
        if (u0 < u1) {
            quantize_query(a.idx_q + (size_t)row * (kHI * kDI), S, kf_lut);
            __syncthreads();
            // query words per channel chunk s and word i: 2q of channels 8i..8i+3, 8i+4..8i+7, negated
            if (tid < 128) {
                const int cs = tid >> 4, wi = (tid >> 2) & 3, kind = tid & 3;
                const uint32_t cw = *reinterpret_cast<const uint32_t*>(&S.qcode[16 * cs + 4 * wi]);
                uint32_t r = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t vq = e2m1_int2((cw >> (4 * j + ((kind & 1) ? 16 : 0))) & 15);
                    if (kind & 2) vq = (0u - vq) & 0xFF;
                    r |= vq << (8 * j);
                }
                S.qv[tid] = r;
            }
            __syncthreads();
            const int s = lane & 7;
            uint32_t qv[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 q4 = *reinterpret_cast<const uint4*>(&S.qv[16 * s + 4 * i]);
                qv[4 * i + 0] = q4.x; qv[4 * i + 1] = q4.y; qv[4 * i + 2] = q4.z; qv[4 * i + 3] = q4.w;
            }
            const int qf0 = S.qf[2 * s], qf1 = S.qf[2 * s + 1];
            // every warp runs the same number of steps; step i of warp w covers units
            // u0 + 32 i + 4 w .. +3; a selection flush follows every kStepsPerFlush steps
            const int nsteps = (u1 - u0 + kWarps * kUnitsPerStep - 1) / (kWarps * kUnitsPerStep);
            static_assert(kStages == 2, "two staging slots");
            int pk0 = stage_step(a, R, u0 + kUnitsPerStep * warp, u1, wst), pk1 = -16;
            cp_async_commit();
            unsigned long long thr = S.thr;
            for (int i = 0; i < nsteps; ++i) {
                const int nx = i + 1;
                if (nx < nsteps) {
                    const int p = stage_step(a, R, u0 + kWarps * kUnitsPerStep * nx + kUnitsPerStep * warp, u1,
                                             wst + (nx & 1) * kStepBytes);
                    if (nx & 1) pk1 = p; else pk0 = p;
                }
                cp_async_commit();
                cp_async_wait<kStages - 1>();
                __syncwarp();
                score_step<RELU>(wst + (i & 1) * kStepBytes, (i & 1) ? pk1 : pk0,
                                 u0 + kWarps * kUnitsPerStep * i + kUnitsPerStep * warp, qv, qf0, qf1, kf_lut, B, S,
                                 thr);
                __syncwarp();
                if ((i + 1) % kStepsPerFlush == 0 || i + 1 == nsteps) {
                    __syncthreads();
                    flush(B, hist, S, K);
                    thr = S.thr;
                }
            }
            cp_async_wait<0>();
        }
        __syncthreads();
        // publish the local Top-k: raise the row's threshold, then emit entries >= it
        if (tid == 0) {
            if (S.nkeep >= K && S.thr) atomicMax(&rc->tau, S.thr);
            S.prefix = atomicAdd(&rc->tau, 0ull);
        }
        __syncthreads();
        const unsigned long long tau = S.prefix;
        const int cur = S.cur, nk = S.nkeep;
        int cnt_local = 0;
        for (int i = tid; i < nk; i += kThreads) cnt_local += (B.keep_key[cur][i] >= tau);
        for (int o = 16; o > 0; o >>= 1) cnt_local += __shfl_xor_sync(0xffffffffu, cnt_local, o);
        if (lane == 0) hist[warp] = cnt_local;
        __syncthreads();
        if (tid == 0) {
            int tot = 0;
            for (int w2 = 0; w2 < kWarps; ++w2) tot += hist[w2];
            S.misc = tot ? (int)atomicAdd(&rc->ncand, (unsigned)tot) : 0;
            S.above = 0;
        }
        __syncthreads();
        {
            const size_t cbase = (size_t)row * a.plan.cand_cap + S.misc;
            for (int base = 0; base < nk; base += kThreads) {
                const int i = base + tid;
                const bool v = i < nk && B.keep_key[cur][i] >= tau;
                const unsigned int bal = __ballot_sync(0xffffffffu, v);
                int wb = 0;
                if (lane == 0 && bal) wb = atomicAdd(&S.above, __popc(bal));
                wb = __shfl_sync(0xffffffffu, wb, 0);
                if (v) {
                    const size_t o = cbase + wb + __popc(bal & ((1u << lane) - 1));
                    cand_key[o] = B.keep_key[cur][i];
                    cand_pos[o] = B.keep_pos[cur][i];
                }
            }
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) S.last = (atomicAdd(&rc->ticket, 1u) == (unsigned)a.plan.chunks - 1);
        __syncthreads();
        if (!S.last) continue;
        // ---- this CTA merges the row ----
        __threadfence();
        const unsigned int ncand = *(volatile unsigned int*)&rc->ncand;
        const unsigned long long tau_f = *(volatile unsigned long long*)&rc->tau;
        stream_select_global(cand_key + (size_t)row * a.plan.cand_cap, cand_pos + (size_t)row * a.plan.cand_cap,
                             (int)ncand, tau_f, K, B, hist, S, false);
        {
            const int n = S.nkeep, c = S.cur;
            int* buf = reinterpret_cast<int*>(B.keep_key[c ^ 1]);  // 2K ints >= next power of two of n
            for (int i = tid; i < n; i += kThreads) buf[i] = B.keep_pos[c][i];
            __syncthreads();
            sort_ascending(buf, n);
            int32_t* out = a.out_idx + (size_t)row * K;
            for (int i = tid; i < K; i += kThreads) out[i] = i < n ? buf[i] : -1;
            __syncthreads();
        }
        if (tid == 0) { rc->ticket = 0; rc->ncand = 0; rc->tau = 0; }
        __syncthreads();
    }
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(done, 1u) == gridDim.x - 1) {
            *next = 0;
            *done = 0;
            __threadfence();
        }
    }
}

// ---- final selection of the tensor-core filter (index_mma.cu): one CTA per row ----------------------
// A lower bound of the k-th largest of n orderable values in shared memory (n >= k >= 1): that value
// with its low 8 bits cleared (three 8-bit radix passes), so at least k values are >= the result.
__device__ uint32_t kth_lower_bound(const uint32_t* v, int n, int k, unsigned int* hist, Scal& S) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t prefix = 0, mask = 0;
    int kr = k;
    for (int shift = 24; shift >= 8; shift -= 8) {
        hist[tid] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += kThreads)
            if ((v[i] & mask) == prefix) atomicAdd(&hist[(v[i] >> shift) & 255u], 1u);
        __syncthreads();
        if (warp == 0) {
            // lane L owns bins 255-8L ... 248-8L (descending)
            unsigned int c[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { c[j] = hist[255 - 8 * lane - j]; sum += c[j]; }
            unsigned int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const unsigned int excl = incl - sum;
            if (excl < (unsigned)kr && incl >= (unsigned)kr) {
                unsigned int run = excl;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (run + c[j] >= (unsigned)kr) {
                        S.digit = 255 - 8 * lane - j;
                        S.above = (int)run;
                        break;
                    }
                    run += c[j];
                }
            }
        }
        __syncthreads();
        kr -= S.above;
        prefix |= (uint32_t)S.digit << shift;
        mask |= 255u << shift;
        __syncthreads();
    }
    return prefix;
}

// Shared memory (64 KB, three CTAs per SM): A0 = u32[kMmaCap], A1 = i32[kMmaCap], B = u64[kMmaCap].
// Filtered rows: candidate images in A0 and positions in A1, then the rescored set's positions in A0
// and keys in B, the Top-k (u64[k] keys, i32[k] positions) in A1. Rows rescored whole: positions in
// A1, keys in B, the Top-k in A0.
size_t final_smem_bytes(int) { return (size_t)16 * kMmaCap; }

// Per row: gathers the candidates of the filter's work items, checks the conditions under which
// they contain the exact Top-k, rescores {S^ >= A - 2 eps} exactly (A: a lower bound of the k-th
// largest S^ among the candidates, so at least k of them are >= A) and ranks it (a row seeing at
// most kMmaCap positions rescores all of them); a row failing a condition is listed for the exact
// scan instead.
__global__ void __launch_bounds__(kThreads, 3) mma_final_kernel(IndexArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ Scal S;
    __shared__ unsigned int hist[256];
    __shared__ int kf_lut[256];
    __shared__ unsigned int nabove, nsel, bad, ntot;
    __shared__ unsigned int coff[256], ccnt[256];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = blockIdx.x, K = a.plan.k;
    const MmaPlan& P = a.plan.mma;
    static_assert(kMmaCap % kThreads == 0 && kMmaCap / kThreads <= 16, "two-phase compaction registers");
    unsigned char* A0 = smem;
    unsigned char* A1 = smem + 4 * kMmaCap;
    uint32_t* ckey = reinterpret_cast<uint32_t*>(A0);
    int* cposs = reinterpret_cast<int*>(A1);
    unsigned long long* rkey = reinterpret_cast<unsigned long long*>(smem + 8 * kMmaCap);
    uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + kHdrStatus);
    int32_t* out = a.out_idx + (size_t)row * K;

    const int64_t ql = index_row_last(a, row);
    if (ql < -1 && tid == 0) set_status(status, CSA2_DEV_BAD_POS);
    const int64_t n = ql + 1;
    if (n <= K) {  // every visible position (none for an invalid row)
        for (int i = tid; i < K; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    kf_lut[tid] = e4m3_fixed(tid);
    const float4 rp = reinterpret_cast<const float4*>(a.ws + a.L.mma_row)[row];
    const float tau = rp.x, eps = rp.y;
    const bool whole = n <= kMmaCap;
    int* rpos = reinterpret_cast<int*>(whole ? A1 : A0);
    unsigned long long* okey = reinterpret_cast<unsigned long long*>(whole ? A0 : A1);
    int* opos = reinterpret_cast<int*>(okey + K);
    if (tid == 0) { bad = 0; nsel = 0; nabove = 0; ntot = 0; }
    __syncthreads();
    bool ok = true;
    if (whole) {
        for (int i = tid; i < (int)n; i += kThreads) rpos[i] = i;
        if (tid == 0) nsel = (unsigned)n;
    } else {
        // the row's lists, one per filter item over its visible key tiles
        const int b = row / a.tq, j = (row % a.tq) / P.nq;
        const int te = (int)reinterpret_cast<const uint32_t*>(a.ws + a.L.mma_tend)[b * P.nqt + j];
        const int nch = (te + P.kc - 1) / P.kc;
        const uint32_t* cc = reinterpret_cast<const uint32_t*>(a.ws + a.L.mma_cnt) + (size_t)row * P.nchunks;
        // every list's count into shared memory in one pass, then their offsets
        for (int c = tid; c < nch && c < 256; c += kThreads) ccnt[c] = cc[c];
        __syncthreads();
        if (warp == 0) {
            unsigned int run = 0;
            for (int c0 = 0; c0 < nch; c0 += 32) {
                const int c = c0 + lane;
                const unsigned int v = (c < nch && c < 256) ? ccnt[c] : 0u;
                if (v > (unsigned)P.subcap) atomicOr(&bad, 1u);
                unsigned int incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                if (c < nch && c < 256) coff[c] = run + incl - v;
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) { ntot = run; if (nch > 256) bad = 1; }
        }
        __syncthreads();
        ok = bad == 0 && ntot <= (unsigned)kMmaCap;
        if (ok) {
            const float* cv = reinterpret_cast<const float*>(a.ws + a.L.mma_cval) + (size_t)row * P.nchunks * P.subcap;
            const int* cp = reinterpret_cast<const int*>(a.ws + a.L.mma_cpos) + (size_t)row * P.nchunks * P.subcap;
            const uint32_t otau = f32_order(tau);
            unsigned int above = 0;
            // candidate o of the row: list c = the last one starting at or before o (binary search
            // over the offsets); every thread's loads are independent of one another
            const int tot = (int)ntot;
#pragma unroll 4
            for (int o = tid; o < tot; o += kThreads) {
                int lo = 0, hi = nch - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if ((int)coff[mid] <= o) lo = mid; else hi = mid - 1;
                }
                const size_t src = (size_t)lo * P.subcap + (o - (int)coff[lo]);
                const uint32_t k2 = f32_order(cv[src]);
                ckey[o] = k2;
                cposs[o] = cp[src];
                above += k2 >= otau;
            }
            above = __reduce_add_sync(0xffffffffu, above);
            if (lane == 0 && above) atomicAdd(&nabove, above);
            __syncthreads();
            ok = nabove >= (unsigned)K;  // at least k positions above the estimate
        }
        if (ok) {
            const int cnt = (int)ntot;
            const float A = f32_unorder(kth_lower_bound(ckey, cnt, K, hist, S));
            const uint32_t olo = f32_order(__double2float_rd((double)A - 2.0 * (double)eps));
            // two-phase compaction of {S^ >= A - 2 eps} (the positions then overwrite A0): every
            // element is read into registers before any is written, output in candidate order
            constexpr int kPer = kMmaCap / kThreads;
            uint32_t kr[kPer];
            int pr[kPer];
            unsigned int sel = 0, mine = 0;
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int i = j * kThreads + tid;
                kr[j] = 0;
                pr[j] = 0;
                if (i < cnt) {
                    kr[j] = ckey[i];
                    pr[j] = cposs[i];
                    if (kr[j] >= olo) { sel |= 1u << j; ++mine; }
                }
            }
            unsigned int incl = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            if (lane == 31) coff[warp] = incl;
            __syncthreads();
            unsigned int base = incl - mine;
            for (int w = 0; w < warp; ++w) base += coff[w];
            if (tid == kThreads - 1) nsel = base + mine;
#pragma unroll
            for (int j = 0; j < kPer; ++j)
                if (sel & (1u << j)) {
                    rkey[base] = kr[j];
                    rpos[base] = pr[j];
                    ++base;
                }
        }
    }
    __syncthreads();
    if (ok) {
        // the query exactly as the tensor cores saw it, as the integer words of score_step
        const uint8_t* qc = a.ws + a.L.mma_qc + (size_t)row * kIKBytes;
        if (tid < 128) S.qcode[tid] = qc[tid];
        if (tid < 16) S.qf[tid] = kf_lut[a.ws[a.L.mma_qs + (size_t)row * kIKScales + tid]];
        __syncthreads();
        if (tid < 128) {
            const int cs = tid >> 4, wi = (tid >> 2) & 3, kind = tid & 3;
            const uint32_t cw = *reinterpret_cast<const uint32_t*>(&S.qcode[16 * cs + 4 * wi]);
            uint32_t r = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t vq = e2m1_int2((cw >> (4 * j + ((kind & 1) ? 16 : 0))) & 15);
                if (kind & 2) vq = (0u - vq) & 0xFF;
                r |= vq << (8 * j);
            }
            S.qv[tid] = r;
        }
        __syncthreads();
        // exact scores: 8 threads per position, each 32 channels (two scale blocks)
        const int sub = lane & 7, grp = tid >> 3;
        uint32_t qv[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 q4 = *reinterpret_cast<const uint4*>(&S.qv[16 * sub + 4 * i]);
            qv[4 * i + 0] = q4.x; qv[4 * i + 1] = q4.y; qv[4 * i + 2] = q4.z; qv[4 * i + 3] = q4.w;
        }
        const int qf0 = S.qf[2 * sub], qf1 = S.qf[2 * sub + 1];
        const int nr = (int)nsel;
        const int b = row / a.tq;
        const uint8_t* kbase = a.c.ik_data + (size_t)b * a.c.cap * kIKBytes;
        const uint8_t* sbase = a.c.ik_scale + (size_t)b * a.c.cap * kIKScales;
        constexpr int kG = kThreads / 8;  // positions per round and unrolled group
        for (int base = 0; base < nr; base += 4 * kG) {
            uint4 w[4];
            uint32_t sc[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const int i = base + h * kG + grp;
                w[h] = make_uint4(0, 0, 0, 0);
                sc[h] = 0;
                if (i < nr) {
                    const size_t p = (size_t)rpos[i];
                    w[h] = __ldg(reinterpret_cast<const uint4*>(kbase + p * kIKBytes + 16 * sub));
                    sc[h] = __ldg(reinterpret_cast<const uint16_t*>(sbase + p * kIKScales + 2 * sub));
                }
            }
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const int i = base + h * kG + grp;
                int d0 = dot8(w[h].x, qv[0], qv[1], qv[2], qv[3], 0);
                d0 = dot8(w[h].y, qv[4], qv[5], qv[6], qv[7], d0);
                int d1 = dot8(w[h].z, qv[8], qv[9], qv[10], qv[11], 0);
                d1 = dot8(w[h].w, qv[12], qv[13], qv[14], qv[15], d1);
                long long v = (long long)(d0 * kf_lut[sc[h] & 0xFF]) * qf0 + (long long)(d1 * kf_lut[sc[h] >> 8]) * qf1;
                v += shfl_xor_s64(v, 1);
                v += shfl_xor_s64(v, 2);
                v += shfl_xor_s64(v, 4);
                if (sub == 0 && i < nr) {
                    if (!whole) {  // the error bound held for this position
                        const double shat = (double)f32_unorder((uint32_t)rkey[i]);
                        if (fabs(shat - (double)v * 0x1p-20) > (double)eps) atomicOr(&bad, 1u);
                    }
                    rkey[i] = (unsigned long long)v ^ 0x8000000000000000ull;
                }
            }
        }
        __syncthreads();
        ok = bad == 0;
    }
    if (!ok) {  // the exact scan takes this row
        if (tid == 0) {
            const unsigned int f = atomicAdd(reinterpret_cast<uint32_t*>(a.ws + a.L.mma_fail_n), 1u);
            reinterpret_cast<int32_t*>(a.ws + a.L.mma_fail)[f] = row;
        }
        return;
    }
    if (tid == 0) S.thr = 0;
    __syncthreads();
    cta_select(rkey, rpos, (int)nsel, nullptr, nullptr, 0, K, okey, opos, hist, S);
    int* buf = reinterpret_cast<int*>(rkey);  // kMmaCap ints >= the next power of two of K
    for (int i = tid; i < K; i += kThreads) buf[i] = opos[i];
    __syncthreads();
    sort_ascending(buf, K);
    for (int i = tid; i < K; i += kThreads) out[i] = buf[i];
}

size_t smem_bytes(const IndexPlan& p) {
    return (size_t)kStagingBytes + (size_t)12 * (2 * p.k + kNewCap);
}

}  // namespace

cudaError_t launch_index(const IndexArgs& a0, cudaStream_t s) {
    // rows of one query per sequence (Full with a pool, Reindex) take index_decode.cu
    if (a0.reindex || a0.plan.pool_blocks > 0) return cudaErrorInvalidValue;
    const bool relu = (a0.flags & CSA2_SCORE_RELU) != 0;
    IndexArgs a = a0;
    if (a.plan.mma.on && !relu && a.ratio == 1) {
        // tensor-core filter and exact final selection; the rows it hands back take the exact scan
        cudaError_t e = launch_index_mma(a, s);
        if (e != cudaSuccess) return e;
        const size_t fs = final_smem_bytes(a.plan.k);
        e = cudaFuncSetAttribute(mma_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fs);
        if (e != cudaSuccess) return e;
        mma_final_kernel<<<(unsigned)a.plan.rows, kThreads, fs, s>>>(a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        a.row_list = reinterpret_cast<const int32_t*>(a.ws + a.L.mma_fail);
        a.row_n = reinterpret_cast<const uint32_t*>(a.ws + a.L.mma_fail_n);
    }
    const size_t smem = smem_bytes(a.plan);
    const void* fn = relu ? (const void*)index_kernel<true> : (const void*)index_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const long long items = (long long)a.plan.rows * a.plan.chunks;  // at most (row list: fewer)
    long long grid = (long long)sms * per_sm;
    if (grid > items) grid = items;
    if (grid < 1) grid = 1;
    if (relu) index_kernel<true><<<(unsigned)grid, kThreads, smem, s>>>(a);
    else index_kernel<false><<<(unsigned)grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace csa2
