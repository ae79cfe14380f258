// index.cu -- indexer scoring, exact Top-k selection and the block candidate pool.
//
// [B] "DeepSeek Cuts KV Cache Footprint Fourfold", "Technical Approach": Full mode computes the
// Top-K indices; Reindex recomputes the selection inside the shared candidate pool built by the
// decoder's first Full layer. [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890
// Bytes per Token", sec. VI "Shortlist-of-a-shortlist" and sec. IX Figure 4: each block of 8
// positions is scored by the maximum index score among its positions and the winning blocks (up
// to 2,048) form the pool. sec. XI: indexer queries and keys are FP4.
//
// Score (this build's reading; the pages give no formula): score(p) = sum_h q_h . k_{p,h} over 4
// heads x 64 channels of dequantised FP4 values. The score is EXACT: per 16-channel block, the
// sum of 16 products of E2M1 values is accumulated in fp16 in two halves of 8 products (each a
// multiple of 1/4 below 288, exact in fp16), the two halves are added in fp32 (exact, < 576),
// multiplied by the fp32 product of the two E4M3 scales (exact, <= 8 significant bits; the
// product has <= 20 bits), and the 16 block partials are summed in fp64 (all terms are multiples
// of 2^-20 below 2^31). Ranking is by score descending, ties to the lower position (to the lower
// block id for the pool), so the selected set is unique.
//
// Structure (one kernel, persistent CTAs taking work items from an atomic counter):
//   item = (query row, chunk of 8-position units). A CTA scores the chunk two units per warp
//   step (16 positions, 2 KB of indexer keys, loaded as coalesced 16-byte vectors), keeps a
//   running local Top-k in shared memory (admission threshold + radix select), and emits its
//   local Top-k to the row's candidate list in the workspace. The CTA that finishes a row's
//   last chunk merges the candidates (and, for the pool, the per-unit block maxima) into the
//   final ascending outputs and clears the row's counters.
#include "csa2_internal.cuh"

namespace csa2 {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSubUnits = 256;            // units scored between two selection flushes
constexpr int kNewCap = kSubUnits * kBS;  // admissions per sub-chunk, worst case

struct Smem {
    unsigned long long* keep_key[2];
    int* keep_pos[2];
    unsigned long long* new_key;
    int* new_pos;
    unsigned int* hist;      // 256
    int kcap;
};

struct __align__(16) SmemScalars {
    int cur, nkeep, nnew, digit, above, cnt, last, misc;
    unsigned long long thr, prefix;
    float qscale[16];
    __align__(16) uint8_t qcode[128];  // read back as 16-byte vectors
};

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m) {
    return __shfl_xor_sync(0xffffffffu, v, m);
}

// ---- query quantisation (same codec as the cache) ------------------------------------------
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

__device__ void quantize_query(const uint16_t* q, SmemScalars& S) {
    const int t = threadIdx.x;
    if (t < 16) {
        float x[16];
        const uint4 a = *reinterpret_cast<const uint4*>(q + t * 16);
        const uint4 b = *reinterpret_cast<const uint4*>(q + t * 16 + 8);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            amax = fmaxf(amax, fmaxf(fabsf(x[2 * i]), fabsf(x[2 * i + 1])));
        }
        const uint32_t sc = q_f32_to_e4m3(__fdiv_rn(amax, 6.0f));
        const float s = e4m3_to_f32((uint8_t)sc);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            S.qcode[t * 8 + j] = (s == 0.f) ? 0 : (uint8_t)q_f32x2_to_e2m1x2(__fdiv_rn(x[2 * j], s), __fdiv_rn(x[2 * j + 1], s));
        S.qscale[t] = s;
    }
}

// ---- CTA radix select ----------------------------------------------------------------------------
// Elements i < na come from (ka, pa), the rest from (kb, pb). Writes the top `K` (key desc,
// pos asc) into (ko, po) in arbitrary order; returns through S.thr a lower bound of the kept keys.
__device__ void cta_select(const unsigned long long* ka, const int* pa, int na, const unsigned long long* kb,
                           const int* pb, int nb, int K, unsigned long long* ko, int* po, Smem& M, SmemScalars& S) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = na + nb;
    auto key_at = [&](int i) { return i < na ? ka[i] : kb[i - na]; };
    auto pos_at = [&](int i) { return i < na ? pa[i] : pb[i - na]; };

    unsigned long long prefix = 0, mask = 0;
    int kr = K;
    bool exact = false;
    for (int shift = 56; shift >= 0; shift -= 8) {
        M.hist[tid] = 0;  // kThreads == 256 bins
        __syncthreads();
        for (int i = tid; i < n; i += kThreads) {
            const unsigned long long key = key_at(i);
            if ((key & mask) == prefix) atomicAdd(&M.hist[(key >> shift) & 255], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            // lane L owns bins 255-8L ... 248-8L (descending)
            unsigned int c[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { c[j] = M.hist[255 - 8 * lane - j]; sum += c[j]; }
            unsigned int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                unsigned int v = __shfl_up_sync(0xffffffffu, incl, o);
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
        mask |= 0xFFull << shift;
        if (S.cnt == kr) { exact = true; }
        __syncthreads();
        if (exact) break;
    }
    // tie on the full key: the kr lowest positions among key == prefix
    unsigned int pthr = 0xFFFFFFFFu;
    if (!exact) {
        unsigned int pp = 0, pm = 0;
        int r = kr;
        for (int shift = 24; shift >= 0; shift -= 8) {
            M.hist[tid] = 0;
            __syncthreads();
            for (int i = tid; i < n; i += kThreads) {
                if (key_at(i) != prefix) continue;
                const unsigned int p = (unsigned int)pos_at(i);
                if ((p & pm) == pp) atomicAdd(&M.hist[(p >> shift) & 255], 1u);
            }
            __syncthreads();
            if (warp == 0) {
                unsigned int c[8], sum = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) { c[j] = M.hist[8 * lane + j]; sum += c[j]; }
                unsigned int incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    unsigned int v = __shfl_up_sync(0xffffffffu, incl, o);
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
        pthr = pp | ~pm;  // every position with the chosen prefix qualifies
    }
    // compaction
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
            if (exact) sel = (key & mask) >= prefix;
            else sel = key > prefix || (key == prefix && (unsigned int)p <= pthr);
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
    if (tid == 0) S.thr = prefix;
    __syncthreads();
}

// Merge the pending admissions into the running Top-K.
__device__ void flush(Smem& M, SmemScalars& S, int K) {
    const int nk = S.nkeep, nn = S.nnew, cur = S.cur;
    if (nn == 0) return;
    if (nk + nn <= K) {
        for (int i = threadIdx.x; i < nn; i += kThreads) {
            M.keep_key[cur][nk + i] = M.new_key[i];
            M.keep_pos[cur][nk + i] = M.new_pos[i];
        }
        __syncthreads();
        if (threadIdx.x == 0) { S.nkeep = nk + nn; S.nnew = 0; }
        __syncthreads();
        return;
    }
    cta_select(M.keep_key[cur], M.keep_pos[cur], nk, M.new_key, M.new_pos, nn, K, M.keep_key[cur ^ 1],
               M.keep_pos[cur ^ 1], M, S);
    if (threadIdx.x == 0) { S.cur = cur ^ 1; S.nkeep = K; S.nnew = 0; }
    __syncthreads();
}

// Admit (key, pos) from lanes with `valid`, warp-aggregated.
__device__ __forceinline__ void admit(Smem& M, SmemScalars& S, bool valid, unsigned long long key, int pos) {
    const int lane = threadIdx.x & 31;
    const unsigned int bal = __ballot_sync(0xffffffffu, valid);
    if (!bal) return;
    int base = 0;
    if (lane == 0) base = atomicAdd(&S.nnew, __popc(bal));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (valid) {
        const int o = base + __popc(bal & ((1u << lane) - 1));
        M.new_key[o] = key;
        M.new_pos[o] = pos;
    }
}

// Ascending bitonic sort of n <= kNewCap int32 values in `a` (padded with INT_MAX to a power of 2).
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
    r.qpos = a.qpos ? a.qpos[row] : a.qpos_base + row % a.tq;
    r.ok = true;
    if (r.qpos < 0 || r.qpos >= a.c.cap || (!a.reindex && r.qpos >= a.max_ctx)) {
        r.ok = false;
        r.n_units = 0;
        return r;
    }
    if (a.reindex) {
        int n = a.pool_n[r.b];
        if (n < 0 || n > a.pool_stride) n = n < 0 ? 0 : a.pool_stride;
        r.n_units = n;
    } else {
        r.n_units = (int)((r.qpos + kBS) / kBS);
    }
    return r;
}

// ---- scoring of two 8-position units by one warp --------------------------------------------------
template <bool RELU>
__device__ __forceinline__ void score_pair(const IndexArgs& a, const RowInfo& R, int unitA, int u_end,
                                           const uint32_t (&qh)[16], float qs0, float qs1, Smem& M,
                                           SmemScalars& S, unsigned long long thr, unsigned long long* bmax_row,
                                           uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int m = lane >> 3, s = lane & 7;
    int blk[2];
    bool uvalid[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int unit = unitA + u;
        uvalid[u] = unit < u_end;
        blk[u] = unit;
        if (uvalid[u] && a.reindex) {
            const int id = a.pool[(size_t)R.b * a.pool_stride + unit];
            if (id < 0 || (int64_t)id * kBS >= a.c.cap) {
                if (lane == 0) set_status(status, CSA2_DEV_BAD_POOL);
                uvalid[u] = false;
            }
            blk[u] = id;
        }
    }
    // loads: j -> unit j>>1, unit position (j&1)*4 + m, channel chunk s (32 channels)
    uint4 w[4];
    uint32_t sc[4];
    bool pv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int u = j >> 1;
        const int64_t p = (int64_t)blk[u] * kBS + (j & 1) * 4 + m;
        pv[j] = uvalid[u] && p <= R.qpos && p < a.c.cap;
        w[j] = make_uint4(0, 0, 0, 0);
        sc[j] = 0;
        if (pv[j]) {
            const size_t row = (size_t)R.b * a.c.cap + (size_t)p;
            w[j] = __ldg(reinterpret_cast<const uint4*>(a.c.ik_data + row * kIKBytes) + s);
            sc[j] = __ldg(reinterpret_cast<const uint16_t*>(a.c.ik_scale + row * kIKScales) + s);
        }
    }
    double v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t k0[4], k1[4], k2[4], k3[4];
        e2m1x8_to_h2x4(w[j].x, k0);
        e2m1x8_to_h2x4(w[j].y, k1);
        e2m1x8_to_h2x4(w[j].z, k2);
        e2m1x8_to_h2x4(w[j].w, k3);
        uint32_t acc0 = 0, acc1 = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) acc0 = hfma2(qh[i], k0[i], acc0);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc0 = hfma2(qh[4 + i], k1[i], acc0);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc1 = hfma2(qh[8 + i], k2[i], acc1);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc1 = hfma2(qh[12 + i], k3[i], acc1);
        const float2 ks = h2_to_f2(e4m3x2_to_h2((uint16_t)sc[j]));
        const float2 f0 = h2_to_f2(acc0), f1 = h2_to_f2(acc1);
        const float p0 = (f0.x + f0.y) * (qs0 * ks.x);
        const float p1 = (f1.x + f1.y) * (qs1 * ks.y);
        v[j] = (double)p0 + (double)p1;
    }
    if (RELU) {
        // head h = s >> 1 lives on lanes s and s^1: complete each head's dot first
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[j] += __shfl_xor_sync(0xffffffffu, v[j], 1);
            v[j] = v[j] > 0.0 ? v[j] : 0.0;
            if (s & 1) v[j] = 0.0;  // count each head once
        }
    }
    // reduce-scatter over the 8 lanes of an octet: lane ends with position j = s >> 1
    const bool h2 = s & 4, h1 = s & 2;
    const double s0 = h2 ? v[0] : v[2], s1 = h2 ? v[1] : v[3];
    const double k0 = h2 ? v[2] : v[0], k1 = h2 ? v[3] : v[1];
    const double w0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 4);
    const double w1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 4);
    const double snd = h1 ? w0 : w1, kp = h1 ? w1 : w0;
    double x = kp + __shfl_xor_sync(0xffffffffu, snd, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    const int j = s >> 1;
    const int u = j >> 1;
    const int64_t pos = (int64_t)blk[u] * kBS + (j & 1) * 4 + m;
    const bool valid = pv[j];
    const unsigned long long key = valid ? score_key(x) : 0ull;
    admit(M, S, valid && (s & 1) == 0 && key >= thr, key, (int)pos);
    if (bmax_row) {
        // block maxima: unit u on lanes with (s >> 2) == u; reduce over m (xor 8, 16) and bit 1 (xor 2)
        unsigned long long bm = key;
        unsigned long long o = shfl_xor_u64(bm, 2); bm = o > bm ? o : bm;
        o = shfl_xor_u64(bm, 8); bm = o > bm ? o : bm;
        o = shfl_xor_u64(bm, 16); bm = o > bm ? o : bm;
        if (m == 0 && (s & 3) == 0 && uvalid[u]) bmax_row[unitA + u] = bm;
    }
}

// ---- final merge of one row --------------------------------------------------------------------
__device__ void stream_select_global(const unsigned long long* gk, const int* gp, int n, unsigned long long tau,
                                     int K, Smem& M, SmemScalars& S, bool pos_is_index) {
    if (threadIdx.x == 0) { S.nkeep = 0; S.nnew = 0; S.cur = 0; S.thr = 0; }
    __syncthreads();
    for (int base = 0; base < n; base += kNewCap) {
        const unsigned long long thr = S.thr > tau ? S.thr : tau;
        const int cnt = min(kNewCap, n - base);
        for (int i0 = 0; i0 < cnt; i0 += kThreads) {
            const int i = i0 + threadIdx.x;
            bool v = false;
            unsigned long long key = 0;
            int p = 0;
            if (i < cnt) {
                key = gk[base + i];
                p = pos_is_index ? base + i : gp[base + i];
                v = key >= thr;
            }
            admit(M, S, v, key, p);
        }
        __syncthreads();
        flush(M, S, K);
    }
}

template <bool RELU>
__global__ void __launch_bounds__(kThreads) index_kernel(IndexArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ __align__(16) SmemScalars S;
    Smem M;
    {
        const int kcap = max(a.plan.k, a.plan.pool_blocks);
        unsigned char* p = smem_raw;
        M.kcap = kcap;
        M.keep_key[0] = reinterpret_cast<unsigned long long*>(p); p += 8 * kcap;
        M.keep_key[1] = reinterpret_cast<unsigned long long*>(p); p += 8 * kcap;
        M.new_key = reinterpret_cast<unsigned long long*>(p); p += 8 * kNewCap;
        M.keep_pos[0] = reinterpret_cast<int*>(p); p += 4 * kcap;
        M.keep_pos[1] = reinterpret_cast<int*>(p); p += 4 * kcap;
        M.new_pos = reinterpret_cast<int*>(p); p += 4 * kNewCap;
        M.hist = reinterpret_cast<unsigned int*>(p);
    }
    unsigned char* ws = a.ws;
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + kHdrStatus);
    unsigned int* next = reinterpret_cast<unsigned int*>(ws + kHdrIndexNext);
    unsigned int* done = reinterpret_cast<unsigned int*>(ws + kHdrIndexDone);
    RowCtr* rctr = reinterpret_cast<RowCtr*>(ws + a.L.row_ctr);
    unsigned long long* cand_key = reinterpret_cast<unsigned long long*>(ws + a.L.cand_key);
    int* cand_pos = reinterpret_cast<int*>(ws + a.L.cand_pos);
    unsigned long long* bmax = reinterpret_cast<unsigned long long*>(ws + a.L.bmax);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = a.plan.k;
    const int total = a.plan.rows * a.plan.chunks;
    const bool pool = a.plan.pool_blocks > 0;

    for (;;) {
        if (tid == 0) S.misc = (int)atomicAdd(next, 1u);
        __syncthreads();
        const int item = S.misc;
        __syncthreads();
        if (item >= total) break;
        const int row = item / a.plan.chunks;
        const int chunk = item % a.plan.chunks;
        const RowInfo R = row_info(a, row);
        if (!R.ok && chunk == 0 && tid == 0) set_status(status, CSA2_DEV_BAD_POS);
        const int u0 = chunk * a.plan.chunk_units;
        const int u1 = min(u0 + a.plan.chunk_units, R.n_units);
        if (tid == 0) { S.nkeep = 0; S.nnew = 0; S.cur = 0; S.thr = 0; }
        if (u0 < u1) {
            quantize_query(a.idx_q + (size_t)row * (kHI * kDI), S);
            __syncthreads();
            // this lane's 32 query channels: bytes 16 s .. 16 s + 15 of the code array
            const int s = lane & 7;
            uint32_t qh[16];
            {
                const uint4 c = *reinterpret_cast<const uint4*>(&S.qcode[16 * s]);
                uint32_t t4[4];
                e2m1x8_to_h2x4(c.x, t4); qh[0] = t4[0]; qh[1] = t4[1]; qh[2] = t4[2]; qh[3] = t4[3];
                e2m1x8_to_h2x4(c.y, t4); qh[4] = t4[0]; qh[5] = t4[1]; qh[6] = t4[2]; qh[7] = t4[3];
                e2m1x8_to_h2x4(c.z, t4); qh[8] = t4[0]; qh[9] = t4[1]; qh[10] = t4[2]; qh[11] = t4[3];
                e2m1x8_to_h2x4(c.w, t4); qh[12] = t4[0]; qh[13] = t4[1]; qh[14] = t4[2]; qh[15] = t4[3];
            }
            const float qs0 = S.qscale[2 * s], qs1 = S.qscale[2 * s + 1];
            unsigned long long* bmax_row = (pool && !a.reindex) ? bmax + (size_t)row * a.plan.units_max : nullptr;
            for (int sub = u0; sub < u1; sub += kSubUnits) {
                const int se = min(sub + kSubUnits, u1);
                const unsigned long long thr = S.thr;
                for (int ua = sub + 2 * warp; ua < se; ua += 2 * kWarps)
                    score_pair<RELU>(a, R, ua, se, qh, qs0, qs1, M, S, thr, bmax_row, status);
                __syncthreads();
                flush(M, S, K);
            }
        }
        __syncthreads();
        // publish the local Top-k: raise the row's threshold, then emit entries >= it
        RowCtr* rc = rctr + row;
        if (tid == 0) {
            unsigned long long mine = (S.nkeep >= K) ? S.thr : 0ull;
            if (mine) atomicMax(&rc->tau, mine);
            S.prefix = atomicAdd(&rc->tau, 0ull);
        }
        __syncthreads();
        const unsigned long long tau = S.prefix;
        const int cur = S.cur, nk = S.nkeep;
        int cnt_local = 0;
        for (int i = tid; i < nk; i += kThreads) cnt_local += (M.keep_key[cur][i] >= tau);
        // block-wide sum
        for (int o = 16; o > 0; o >>= 1) cnt_local += __shfl_xor_sync(0xffffffffu, cnt_local, o);
        if (lane == 0) M.hist[warp] = cnt_local;
        __syncthreads();
        if (tid == 0) {
            int tot = 0;
            for (int w2 = 0; w2 < kWarps; ++w2) tot += M.hist[w2];
            S.misc = tot ? (int)atomicAdd(&rc->ncand, (unsigned)tot) : 0;
            S.last = 0;
        }
        __syncthreads();
        {
            const size_t cbase = (size_t)row * a.plan.cand_cap + S.misc;
            if (tid == 0) S.above = 0;
            __syncthreads();
            for (int base = 0; base < nk; base += kThreads) {
                const int i = base + tid;
                const bool v = i < nk && M.keep_key[cur][i] >= tau;
                const unsigned int bal = __ballot_sync(0xffffffffu, v);
                int wb = 0;
                if (lane == 0 && bal) wb = atomicAdd(&S.above, __popc(bal));
                wb = __shfl_sync(0xffffffffu, wb, 0);
                if (v) {
                    const size_t o = cbase + wb + __popc(bal & ((1u << lane) - 1));
                    cand_key[o] = M.keep_key[cur][i];
                    cand_pos[o] = M.keep_pos[cur][i];
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
                             (int)ncand, tau_f, K, M, S, false);
        {
            const int n = S.nkeep, c = S.cur;
            int* buf = M.new_pos;
            for (int i = tid; i < n; i += kThreads) buf[i] = M.keep_pos[c][i];
            __syncthreads();
            sort_ascending(buf, n);
            int32_t* out = a.out_idx + (size_t)row * K;
            for (int i = tid; i < K; i += kThreads) out[i] = i < n ? buf[i] : -1;
            __syncthreads();
        }
        if (pool && !a.reindex) {
            const int P = a.plan.pool_blocks;
            stream_select_global(bmax + (size_t)row * a.plan.units_max, nullptr, R.n_units, 0ull, P, M, S, true);
            const int n = S.nkeep, c = S.cur;
            int* buf = M.new_pos;
            for (int i = tid; i < n; i += kThreads) buf[i] = M.keep_pos[c][i];
            __syncthreads();
            sort_ascending(buf, n);
            int32_t* outp = a.out_pool + (size_t)R.b * P;
            for (int i = tid; i < P; i += kThreads) outp[i] = i < n ? buf[i] : -1;
            if (tid == 0) a.out_pool_n[R.b] = n;
            __syncthreads();
        }
        if (tid == 0) { rc->ticket = 0; rc->ncand = 0; rc->tau = 0; }
        __syncthreads();
    }
    // last CTA out clears the work counters
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(done, 1u) == gridDim.x - 1) {
            *next = 0;
            *done = 0;
            __threadfence();
        }
    }
}

size_t smem_bytes(const IndexPlan& p) {
    const int kcap = p.k > p.pool_blocks ? p.k : p.pool_blocks;
    return (size_t)12 * (2 * kcap + kNewCap) + 4 * 256;
}

}  // namespace

cudaError_t launch_index(const IndexArgs& a, cudaStream_t s) {
    const size_t smem = smem_bytes(a.plan);
    const bool relu = (a.flags & CSA2_SCORE_RELU) != 0;
    const void* fn = relu ? (const void*)index_kernel<true> : (const void*)index_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const long long items = (long long)a.plan.rows * a.plan.chunks;
    long long grid = (long long)sms * per_sm;
    if (grid > items) grid = items;
    if (grid < 1) grid = 1;
    if (relu) index_kernel<true><<<(unsigned)grid, kThreads, smem, s>>>(a);
    else index_kernel<false><<<(unsigned)grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace csa2
