// index_tc.cu -- the index step of decode rows on the tensor cores: one CTA per query row scores
// the row's candidate positions with tcgen05 block-scaled FP4 MMAs and selects the exact Top-k (and,
// in Full mode, the block pool) in shared memory, with no intermediate written to global memory.
//
// Method: [B] "DeepSeek Cuts KV Cache Footprint Fourfold", "Technical Approach" (Full / Reindex
// selection); [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token",
// sec. VI "Shortlist-of-a-shortlist" and sec. IX Figure 4 (block pool), sec. XI (FP4 indexer
// queries and keys). Score (the reading taken here): score(p) = sum over the 4 heads of q_h . k_{p,h}
// on dequantised values, exact; ranking by score descending, ties to the lower position.
//
// Exact scores on the tensor cores. A score is sum_b s_q[b] s_k[p,b] D[p,b] over the 16 blocks b of
// 16 channels, D[p,b] = sum_{c in b} q_c k_{p,c} on the E2M1 values. The MMA computes D for a tile of
// 128 positions at once: A = the positions' packed E2M1 codes (128 x 256, K-major, as stored in the
// cache), B = a block-diagonal query (16 x 256: row b holds the query's codes of block b and zeros
// elsewhere), every block scale set to 1.0, so column b of the fp32 accumulator is D[p,b] itself.
// Each D is a multiple of 1/4 below 2^10 in magnitude and has only 16 non-zero products, so the
// fp32 accumulation is exact in any order. The epilogue then forms, per block, D * s_k (exact in
// fp32: at most 12 + 4 significant bits) times s_q * 2^20 (at most 20 bits), an integer below 2^47,
// and sums the 16 of them in int64: S = score * 2^20 exactly, the same integer the CUDA-core path
// computes.
//
// Roles (12 warps): warps 0, 2 and 3 take the 128-position tiles in turn and stream their code rows
// into an 8-stage ring with TMA (bulk tensor copies, which the SM tracks apart from ordinary loads,
// so that many tiles can be in flight): a Full row's tile is one box of 128 consecutive rows, a
// Reindex tile one box of 8 rows per pool block, each landing in the 128-byte swizzle pattern the
// MMA reads; warp 1 holds the tensor memory and issues 4 MMAs (K = 64 each) per tile into one of 4
// accumulators; warp 2 first quantises the query and builds the block-diagonal operand; warps 4-11,
// two per TMEM lane quadrant taking alternate tiles, load the positions' scale bytes themselves
// (ahead of use), read the accumulators (warp w reads TMEM lanes 32 (w % 4) ..), form the exact
// keys, count them
// into a 2048-bin histogram in shared memory and keep them in tensor memory (two columns per tile).
// Every wait is bounded; a wait that runs out sets CSA2_DEV_TIMEOUT and the CTA winds down without
// selecting.
//
// Histogram bins: a monotone, integer-only function of the key (sign, position of the leading one,
// the next 4 bits; the following 10 bits give the second level), so that a larger key never has a
// smaller bin.
//
// Selection (warps 0-7): the histogram's cut bin (fewer than k keys above it); one pass over the
// keys marks every key above the cut bin in a bitmap and lists the keys inside it; a 1024-bin
// second level over that list, and the few keys left in its final bin ranked pairwise (ties to the
// lower position); each selected element's output slot is its rank among the selected elements,
// read from the bitmap (or a sort when a Reindex pool lists its blocks out of order). A cut bin of
// more than 4096 keys, or a final bin of more than 256, falls back to an exact radix select.
#include <mutex>

#include "csa2_internal.cuh"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int kT = 256;                              // the selection team (warps 0-7)
constexpr int kTAll = 384;                           // all warps during the scan
constexpr int kTileUnits = 16;                       // 8-position units per tile
constexpr int kTileP = kTileUnits * kBS;             // 128 positions = the MMA's M
constexpr int kStages = 8;
constexpr int kStageBytes = kTileP * kIKBytes;       // 16384 code bytes per tile
constexpr int kScaleAhead = 4;                       // tiles whose scale bytes an epilogue thread holds
constexpr int kAcc = 8;                              // accumulators of 16 columns
constexpr int kTmemCols = 512;
constexpr int kSfaCol = 128, kSfbCol = 132;          // unit scale factors (columns 128..143 hold 1.0)
constexpr int kKeyCol = 144;                         // keys of tile i: columns 144 + 2i (low), 145 + 2i (high)
constexpr int kFusedUnits = 2048;                    // longest row: 16,384 positions (128 tiles)
constexpr int kFusedMax = kFusedUnits * kBS;
constexpr int kCutCap = 4096;
constexpr int kTieCap = 256;
constexpr uint64_t kWaitNs = 2000000000ull;          // 2 s: far beyond any legitimate wait here
static_assert(kKeyCol + 2 * (kFusedMax / kTileP) + 32 <= kTmemCols, "keys fit in tensor memory");

// shared memory plan (offsets from a 1024-byte aligned base)
constexpr int kOffStages = 0;
constexpr int kOffQB = kStages * kStageBytes;                 // 2048 bytes, 1024-aligned
constexpr int kOffBKeys = kOffQB + 2048;                      // u64[kFusedUnits] (pool)
constexpr int kOffBlk = kOffBKeys + 8 * kFusedUnits;          // i32[kFusedUnits] block id of each unit, -1 if invalid
constexpr int kOffUInfo = kOffBlk + 4 * kFusedUnits;          // i32[kFusedUnits] (block << 4) | visible positions, or -16
constexpr int kOffHist = kOffUInfo + 4 * kFusedUnits;         // u32[kKeyBins]
constexpr int kOffPHist = kOffHist + 4 * kKeyBins;            // u32[kKeyBins] (pool)
constexpr int kCandCap = 3072;                       // candidate keys kept during the scan
constexpr int kOffCandK = kOffPHist + 4 * kKeyBins;           // u64[kCandCap]
constexpr int kOffCandE = kOffCandK + 8 * kCandCap;           // i32[kCandCap]
constexpr int kOffMisc = kOffCandE + 4 * kCandCap;
constexpr int kSmemBytes = kOffMisc + 1024 + 1024;            // + alignment slack
// selection scratch, reusing the stage ring after the scan
constexpr int kOffBitmap = 0;                                 // u32[kFusedMax / 32]
constexpr int kOffWpre = kOffBitmap + 4 * (kFusedMax / 32);   // i32[kFusedMax / 32]
constexpr int kOffSub = kOffWpre + 4 * (kFusedMax / 32);      // u32[kSubBins]
constexpr int kOffCutK = kOffSub + 4 * kSubBins;              // u64[kCutCap]
constexpr int kOffCutE = kOffCutK + 8 * kCutCap;              // i32[kCutCap]
constexpr int kOffTieK = kOffCutE + 4 * kCutCap;              // u64[kTieCap]
constexpr int kOffTieI = kOffTieK + 8 * kTieCap;              // i32[kTieCap]
constexpr int kOffList = kOffTieI + 4 * kTieCap;              // i32[kMaxK]
constexpr int kOffRHist = kOffList + 4 * kMaxK;               // u32[256]
static_assert(kOffRHist + 1024 <= kStages * kStageBytes, "selection scratch fits in the stage ring");
static_assert(kOffQB % 1024 == 0 && kStageBytes % 1024 == 0, "swizzled tiles are 1024-byte aligned");

// Scale bytes of position pt of tile i (zeros when the position is not in the plane).
__device__ __forceinline__ uint4 load_scales(const IndexArgs& a, const int* blkid, int n_units, int64_t row0, int i,
                                             int pt) {
    const int u = i * kTileUnits + (pt >> 3);
    if (u >= n_units) return make_uint4(0u, 0u, 0u, 0u);
    const int blk = a.reindex ? blkid[u] : u;
    const int64_t p = (int64_t)blk * kBS + (pt & 7);
    if (blk < 0 || p >= a.c.cap) return make_uint4(0u, 0u, 0u, 0u);
    return __ldg(reinterpret_cast<const uint4*>(a.c.ik_scale + (size_t)(row0 + p) * kIKScales));
}

struct Misc {
    uint64_t full[kStages], empty[kStages], accf[kAcc], acce[kAcc];
    uint32_t tmem;
    int abort;
    float qf[16];                        // query scale of block b times 2^20
    int ncut, ntie, unsorted;
    int ncand, lbin;                     // candidates kept so far; bins below lbin cannot be selected
    int rdigit, rabove, rcnt;
    int wsum[kT / 32];
};
static_assert(sizeof(Misc) <= 1024, "misc area");

struct RowDesc {
    int64_t qlast;   // last visible entry
    int b;           // sequence
    int n_units;     // units of the row (0: nothing to score)
};

__device__ __forceinline__ RowDesc row_desc(const IndexArgs& a, int row, bool& ok) {
    RowDesc r;
    r.b = row;
    const int64_t tok = a.qpos ? a.qpos[row] : a.qpos_base;
    r.qlast = tok < 0 ? -1 : (tok + 1) / a.ratio - 1;
    ok = !(tok < 0 || r.qlast >= a.c.cap || (!a.reindex && r.qlast >= a.max_ctx));
    if (!ok) {
        r.n_units = 0;
    } else if (a.reindex) {
        const int n = a.pool_n[r.b];
        r.n_units = n < 0 ? 0 : (n > a.pool_stride ? a.pool_stride : n);
    } else {
        r.n_units = (int)((r.qlast + kBS) / kBS);
    }
    if (r.n_units > kFusedUnits) r.n_units = kFusedUnits;  // the plan never launches longer rows here
    return r;
}

// ---- histogram bins of a key (0 = no key) -------------------------------------------------------------
// bin: 1024 for a zero score; 1025 + f for a positive one and 1022 - f for a negative one, with
// f = 16 * (position of the leading one of |S|) + (the next 4 bits) in 0..815 (|S| < 2^51); sub: the
// next 10 bits (mirrored for negative scores). Larger keys never get smaller (bin, sub).
__device__ __forceinline__ void key_bins(unsigned long long k, int& bin, int& sub) {
    const long long S = (long long)(k ^ 0x8000000000000000ull);
    const unsigned long long mag = S < 0 ? (unsigned long long)(-S) : (unsigned long long)S;
    if (mag == 0) {
        bin = 1024;
        sub = 0;
        return;
    }
    const int lz = __clzll((long long)mag);
    const unsigned long long m = (mag << lz) << 1;  // the bits after the leading one, left-aligned
    const int f = (63 - lz) * 16 + (int)(m >> 60);
    const int s10 = (int)((m >> 50) & 1023u);
    bin = S > 0 ? 1025 + f : 1022 - f;
    sub = S > 0 ? s10 : 1023 - s10;
}
__device__ __forceinline__ int kbin(unsigned long long k) {
    int b, s;
    key_bins(k, b, s);
    return b;
}
__device__ __forceinline__ int ksub(unsigned long long k) {
    int b, s;
    key_bins(k, b, s);
    return s;
}

// ---- selection-team helpers (warps 0-7; the other warps have left) -----------------------------------
__device__ __forceinline__ void sel_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ int block_excl_scan(int v, Misc& M, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) M.wsum[warp] = incl;
    sel_sync();
    int before = 0;
    total = 0;
#pragma unroll
    for (int w = 0; w < kT / 32; ++w) {
        const int c = M.wsum[w];
        before += w < warp ? c : 0;
        total += c;
    }
    sel_sync();
    return before + incl - v;
}

// The cut bin of h[0..nbins): fewer than K counted keys lie above it, at least K at or above it.
// Returns -1 when at most K keys are counted; *above = the count above the cut bin.
template <int NB>
__device__ int cut_bin(const unsigned int* h, int K, Misc& M, int* above) {
    constexpr int per = NB / kT;  // 8 or 4
    const int tid = threadIdx.x;
    unsigned int hb[per];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) {
        hb[j] = h[NB - per * (tid + 1) + j];
        sum += (int)hb[j];
    }
    if (tid == 0) { M.rdigit = -1; M.rabove = 0; }
    int total;
    const int excl = block_excl_scan(sum, M, total);  // its barriers order the reset above
    if (total > K && excl < K && excl + sum >= K) {
        int run = excl;
        for (int j = per - 1; j >= 0; --j) {
            if (run + (int)hb[j] >= K) {
                M.rdigit = NB - per * (tid + 1) + j;
                M.rabove = run;
                break;
            }
            run += (int)hb[j];
        }
    }
    sel_sync();
    *above = M.rabove;
    const int d = M.rdigit;
    sel_sync();
    return d;
}

// 256-bin digit histogram scan from the top (desc) or the bottom: the bin where the running count
// reaches kr; sets M.rdigit, M.rabove (count before it), M.rcnt (its count). Warp 0.
__device__ void scan256(const unsigned int* hist, int kr, bool desc, Misc& M) {
    const int lane = threadIdx.x & 31;
    unsigned int c[8], sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        c[j] = hist[desc ? 255 - 8 * lane - j : 8 * lane + j];
        sum += c[j];
    }
    unsigned int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const unsigned int excl = incl - sum;
    if (excl < (unsigned)kr && incl >= (unsigned)kr) {
        unsigned int run = excl;
        for (int j = 0; j < 8; ++j) {
            if (run + c[j] >= (unsigned)kr) {
                M.rdigit = desc ? 255 - 8 * lane - j : 8 * lane + j;
                M.rabove = (int)run;
                M.rcnt = (int)c[j];
                break;
            }
            run += c[j];
        }
    }
}

// Positions of a row's elements: element i is position 8 * blk[i / 8] + i % 8.
struct Pos {
    const int* blk;  // shared memory, or nullptr (element i is position / block i itself)
    __device__ __forceinline__ int operator()(int i) const { return blk ? blk[i >> 3] * kBS + (i & 7) : i; }
};

// Keys held in tensor memory: element e = 128 i + L of tile i, lane L, at columns kKeyCol + 2i (low
// 32 bits) and kKeyCol + 2i + 1 (high). Warp w reads the lanes of quadrant w % 4 and the tiles of
// parity w / 4, so bitmap word 4i + (w % 4) (elements 128 i + 32 (w % 4) ..) is owned by one warp.
struct TmemKeys {
    uint32_t tbase;
    int ntiles;
    template <class F>
    __device__ __forceinline__ void for_words(F f) const {
        const int warp = threadIdx.x >> 5, q = warp & 3, h = warp >> 2;
        for (int i0 = 0; i0 < ntiles; i0 += 16) {
            uint32_t r[32];
            tc::tmem_ld32(tbase + ((uint32_t)(32 * q) << 16) + kKeyCol + 2 * i0, r);
            tc::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int i = i0 + j;
                if ((j & 1) == h && i < ntiles) f(4 * i + q, ((unsigned long long)r[2 * j + 1] << 32) | r[2 * j]);
            }
        }
    }
};

// Keys in shared memory, element e at k[e]; warp w owns bitmap words w, w + 8, ...
struct SmemKeys {
    const unsigned long long* k;
    int n;
    template <class F>
    __device__ __forceinline__ void for_words(F f) const {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        for (int w = warp; w < (n + 31) / 32; w += kT / 32) {
            const int e = 32 * w + lane;
            f(w, e < n ? k[e] : 0ull);
        }
    }
};

// Exact selection of the K largest keys among the n elements of `src` (key 0 = no key), ties to
// the lower position; writes the selected positions ascending to out[0..K), padded with -1, and
// returns the count. `hist` is the 2048-bin histogram of the valid keys; `scr` the selection scratch.
// When `lk` is given, the lk / le list (nl keys and their elements) holds every key whose bin is not
// below the cut bin, and only it is read in the first pass; `src` is read only by the radix fallback.
template <class Src>
__device__ int select_keys(const Src& src, int n, int K, const unsigned int* hist, Pos pos, bool sorted, int32_t* out,
                           unsigned char* scr, Misc& M, const unsigned long long* lk = nullptr,
                           const int* le = nullptr, int nl = 0) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned int* bitmap = reinterpret_cast<unsigned int*>(scr + kOffBitmap);
    int* wpre = reinterpret_cast<int*>(scr + kOffWpre);
    unsigned int* sub = reinterpret_cast<unsigned int*>(scr + kOffSub);
    unsigned long long* ck = reinterpret_cast<unsigned long long*>(scr + kOffCutK);
    int* ce = reinterpret_cast<int*>(scr + kOffCutE);
    unsigned long long* tk = reinterpret_cast<unsigned long long*>(scr + kOffTieK);
    int* ti = reinterpret_cast<int*>(scr + kOffTieI);
    int* list = reinterpret_cast<int*>(scr + kOffList);
    unsigned int* rh = reinterpret_cast<unsigned int*>(scr + kOffRHist);
    const int words = (n + 31) >> 5;
    for (int j = tid; j < kSubBins; j += kT) sub[j] = 0u;
    if (tid == 0) { M.ncut = 0; M.ntie = 0; }
    int above = 0;
    const int bstar = cut_bin<kKeyBins>(hist, K, M, &above);  // its barriers order the resets above
    // ---- one pass: keys above the cut bin into the bitmap, keys inside it into the cut list ----
    if (lk) {
        for (int w = tid; w < words; w += kT) bitmap[w] = 0u;
        sel_sync();
        for (int c = tid; c < nl; c += kT) {
            const unsigned long long k = lk[c];
            const int e = le[c], bb = kbin(k);
            if (bstar < 0 || bb > bstar) {
                atomicOr(&bitmap[e >> 5], 1u << (e & 31));
            } else if (bb == bstar) {
                const int o = atomicAdd(&M.ncut, 1);
                if (o < kCutCap) { ck[o] = k; ce[o] = e; }
            }
        }
    } else src.for_words([&](int w, unsigned long long k) {
        const int bb = k ? kbin(k) : -1;
        const bool sel = k && (bstar < 0 || bb > bstar);
        const bool cut = k && bstar >= 0 && bb == bstar;
        const unsigned int bal = __ballot_sync(0xffffffffu, sel);
        if (lane == 0 && w < words) bitmap[w] = bal;
        const unsigned int cb = __ballot_sync(0xffffffffu, cut);
        if (cb) {
            int base = 0;
            if (lane == 0) base = atomicAdd(&M.ncut, __popc(cb));
            base = __shfl_sync(0xffffffffu, base, 0) + __popc(cb & ((1u << lane) - 1u));
            if (cut && base < kCutCap) { ck[base] = k; ce[base] = 32 * w + lane; }
        }
    });
    sel_sync();
    bool radix = false;
    if (bstar >= 0) {
        const int nc = M.ncut;
        if (nc > kCutCap) {
            radix = true;
        } else {
            for (int c = tid; c < nc; c += kT) atomicAdd(&sub[ksub(ck[c])], 1u);
            sel_sync();
            // sstar < 0: the cut bin holds exactly the K - above keys still needed; all of it is taken
            int above2 = 0;
            const int sstar = cut_bin<kSubBins>(sub, K - above, M, &above2);
            for (int c = tid; c < nc; c += kT) {
                const int sb = ksub(ck[c]);
                if (sstar < 0 || sb > sstar) {
                    atomicOr(&bitmap[ce[c] >> 5], 1u << (ce[c] & 31));
                } else if (sb == sstar) {
                    const int o = atomicAdd(&M.ntie, 1);
                    if (o < kTieCap) { tk[o] = ck[c]; ti[o] = ce[c]; }
                }
            }
            sel_sync();
            const int m = M.ntie;
            if (m > kTieCap) {
                radix = true;
            } else {
                const int need = K - above - above2;
                for (int t = tid; t < m; t += kT) {
                    const unsigned long long kt = tk[t];
                    const int pt = pos(ti[t]);
                    int rank = 0;
                    for (int f = 0; f < m; ++f) {
                        const unsigned long long kf = tk[f];
                        rank += (kf > kt) || (kf == kt && pos(ti[f]) < pt);
                    }
                    if (rank < need) atomicOr(&bitmap[ti[t] >> 5], 1u << (ti[t] & 31));
                }
            }
            sel_sync();
        }
    }
    if (radix) {
        // exact K-th largest key by 8-bit digits, then the lowest positions among the keys equal to it
        unsigned long long prefix = 0, mask = 0;
        int kr = K;
        for (int shift = 56; shift >= 0; shift -= 8) {
            for (int j = tid; j < 256; j += kT) rh[j] = 0u;
            sel_sync();
            src.for_words([&](int, unsigned long long k) {
                if (k && (k & mask) == prefix) atomicAdd(&rh[(k >> shift) & 255u], 1u);
            });
            sel_sync();
            if (warp == 0) scan256(rh, kr, true, M);
            sel_sync();
            kr -= M.rabove;
            prefix |= (unsigned long long)M.rdigit << shift;
            mask |= 255ull << shift;
            sel_sync();
        }
        const unsigned long long thr = prefix;
        unsigned int pp = 0, pm = 0;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int j = tid; j < 256; j += kT) rh[j] = 0u;
            sel_sync();
            src.for_words([&](int w, unsigned long long k) {
                if (k == thr) {
                    const unsigned int p = (unsigned int)pos(32 * w + lane);
                    if ((p & pm) == pp) atomicAdd(&rh[(p >> shift) & 255u], 1u);
                }
            });
            sel_sync();
            if (warp == 0) scan256(rh, kr, false, M);
            sel_sync();
            kr -= M.rabove;
            pp |= (unsigned int)M.rdigit << shift;
            pm |= 255u << shift;
            sel_sync();
        }
        src.for_words([&](int w, unsigned long long k) {
            const bool sel = k && (k > thr || (k == thr && (unsigned int)pos(32 * w + lane) <= pp));
            const unsigned int bal = __ballot_sync(0xffffffffu, sel);
            if (lane == 0 && w < words) bitmap[w] = bal;
        });
        sel_sync();
    }
    // ---- output: slot of element i = selected elements in earlier words + those below i in its word ----
    const int per = (words + kT - 1) / kT;
    const int w0 = min(tid * per, words), w1 = min(w0 + per, words);
    int wc = 0;
    for (int w = w0; w < w1; ++w) wc += __popc(bitmap[w]);
    int total;
    int run = block_excl_scan(wc, M, total);
    for (int w = w0; w < w1; ++w) {
        wpre[w] = run;
        run += __popc(bitmap[w]);
    }
    sel_sync();
    const int cnt = total < K ? total : K;
    for (int w = w0; w < w1; ++w) {
        unsigned int bw = bitmap[w];
        int slot = wpre[w];
        while (bw) {
            const int bit = __ffs(bw) - 1;
            bw &= bw - 1u;
            if (slot < K) {
                if (sorted) out[slot] = pos(32 * w + bit);
                else list[slot] = pos(32 * w + bit);
            }
            ++slot;
        }
    }
    if (!sorted) {
        sel_sync();
        // ascending bitonic sort of list[0..cnt) (room for the next power of two, <= kMaxK)
        int P = 1;
        while (P < cnt) P <<= 1;
        for (int i = cnt + tid; i < P; i += kT) list[i] = 0x7FFFFFFF;
        sel_sync();
        for (int k2 = 2; k2 <= P; k2 <<= 1) {
            for (int j = k2 >> 1; j > 0; j >>= 1) {
                for (int i = tid; i < P; i += kT) {
                    const int l = i ^ j;
                    if (l > i) {
                        const int x = list[i], y = list[l];
                        if ((x > y) == ((i & k2) == 0)) { list[i] = y; list[l] = x; }
                    }
                }
                sel_sync();
            }
        }
        for (int i = tid; i < cnt; i += kT) out[i] = list[i];
    }
    for (int i = cnt + tid; i < K; i += kT) out[i] = -1;
    sel_sync();
    return cnt;
}

template <bool RELU, bool POOL>
__global__ void __launch_bounds__(kTAll, 1) index_tc_kernel(const IndexArgs a, const __grid_constant__ CUtensorMap tmap) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Misc& M = *reinterpret_cast<Misc*>(sm + kOffMisc);
    unsigned long long* bkeys = reinterpret_cast<unsigned long long*>(sm + kOffBKeys);
    int* blkid = reinterpret_cast<int*>(sm + kOffBlk);
    unsigned int* hist = reinterpret_cast<unsigned int*>(sm + kOffHist);
    unsigned int* phist = reinterpret_cast<unsigned int*>(sm + kOffPHist);
    uint8_t* qb = sm + kOffQB;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = blockIdx.x;
    uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + kHdrStatus);

    if (warp == 1) tc::tmem_alloc(&M.tmem, kTmemCols);
    if (tid == 32) tc::prefetch_tmap(&tmap);
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) { tc::mbar_init(&M.full[s], 1); tc::mbar_init(&M.empty[s], 1); }
        for (int c = 0; c < kAcc; ++c) { tc::mbar_init(&M.accf[c], 1); tc::mbar_init(&M.acce[c], 4); }
        tc::mbar_fence_init();
        M.abort = 0;
        M.unsorted = 0;
        M.ncand = 0;
        M.lbin = -1;
    }
    for (int i = tid; i < kKeyBins; i += kTAll) {
        hist[i] = 0u;
        if (POOL) phist[i] = 0u;
    }
    wait_prior_grid();  // the cache, the query and the pool come from earlier work on the stream
    bool ok;
    const RowDesc R = row_desc(a, row, ok);
    if (!ok && tid == 0) set_status(status, CSA2_DEV_BAD_POS);
    const int n_units = R.n_units;
    const int ntiles = (n_units + kTileUnits - 1) / kTileUnits;
    // block id of every unit (-1: invalid pool id, nothing to score) and its record
    // (block << 4) | visible positions (-16: nothing visible)
    int* uinfo = reinterpret_cast<int*>(sm + kOffUInfo);
    for (int u = tid; u < n_units; u += kTAll) {
        int blk = u;
        if (a.reindex) {
            blk = __ldg(a.pool + (size_t)row * a.pool_stride + u);
            if (blk < 0 || (int64_t)blk * kBS >= a.c.cap) {
                set_status(status, CSA2_DEV_BAD_POOL);
                blk = -1;
            }
        }
        blkid[u] = blk;
        int info = -16;
        if (blk >= 0) {
            int64_t nv = R.qlast - (int64_t)blk * kBS + 1;
            if (a.c.cap - (int64_t)blk * kBS < nv) nv = a.c.cap - (int64_t)blk * kBS;
            if (nv > 0) info = (blk << 4) | (nv > kBS ? kBS : (int)nv);
        }
        uinfo[u] = info;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tbase = M.tmem;

    // ---- set-up: the block-diagonal query operand and the unit scale factors ----
    if (warp == 2) {
        // zero the 16 x 128-byte operand, then lanes 0..15 quantise block b = lane into row b
        for (int i = lane; i < 2048 / 16; i += 32) *reinterpret_cast<uint4*>(qb + 16 * i) = make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
        if (lane < 16 && n_units > 0) {
            const int bq = lane;
            float x[16];
            load16_bf16(a.idx_q + (size_t)row * (kHI * kDI) + 16 * bq, x);
            uint2 codes;
            uint8_t sc;
            quantize_block(x, codes, sc);
            // row bq, bytes 8 bq .. 8 bq + 7: chunk bq / 2 of the row, swizzled by the row within its group of 8
            const int off = (bq >> 3) * 1024 + (bq & 7) * 128 + ((((bq >> 1) ^ (bq & 7))) << 4) + 8 * (bq & 1);
            *reinterpret_cast<uint2*>(qb + off) = codes;
            M.qf[bq] = e4m3_to_f32(sc) * 1048576.0f;
        }
        tc::fence_async_smem();
    } else if (warp >= 4 && warp < 8) {
        uint32_t one[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) one[i] = 0x38383838u;  // UE4M3 1.0 in every byte
        tc::tmem_st16(tbase + ((uint32_t)(32 * (warp & 3)) << 16) + kSfaCol, one);
        tc::tmem_st_wait();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    if (warp == 0 || warp == 2 || warp == 3) {
        // ---- producers: warps 0, 2, 3 take tiles 0, 1, 2, 3, ... in turn; a tile's TMA boxes are
        // issued by one warp (lane j: pool block j of a Reindex tile; lane 0: the 128-row box of a
        // Full tile), so one warp's bookkeeping overlaps another's copies ----
        const int p = warp == 0 ? 0 : warp - 1;
        for (int i = p; i < ntiles; i += 3) {
            const int s = i % kStages;
            const uint32_t ph = (uint32_t)(i / kStages) & 1u;
            if (!tc::mbar_wait(&M.empty[s], ph ^ 1u, kWaitNs)) { M.abort = 1; set_status(status, CSA2_DEV_TIMEOUT); }
            if (__any_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&M.abort) != 0)) break;
            uint8_t* st = sm + kOffStages + s * kStageBytes;
            const int u = i * kTileUnits + lane;
            const int info = (lane < kTileUnits && u < n_units) ? uinfo[u] : -16;
            const uint32_t bytes = a.reindex ? (uint32_t)__popc(__ballot_sync(0xffffffffu, info >= 0)) * (kBS * kIKBytes)
                                             : (uint32_t)kStageBytes;  // one box; rows past the plane read as zeros
            if (lane == 0) tc::mbar_expect_tx(&M.full[s], bytes);
            __syncwarp();
            if (a.reindex) {
                if (info >= 0) tc::tma_3d_g2s(st + lane * 1024, &tmap, 0, (info >> 4) * kBS, R.b, &M.full[s]);
            } else if (lane == 0) {
                tc::tma_3d_g2s(st, &tmap, 0, i * kTileP, R.b, &M.full[s]);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer ----
        const uint32_t idesc = tc::mxf4_idesc(kTileP, 16);
        const uint32_t qaddr = tc::smem_u32(qb);
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % kStages, c = i % kAcc;
            const uint32_t ph = (uint32_t)(i / kStages) & 1u, aph = (uint32_t)(i / kAcc) & 1u;
            bool okw = tc::mbar_wait(&M.full[s], ph, kWaitNs);
            okw = okw && tc::mbar_wait(&M.acce[c], aph ^ 1u, kWaitNs);
            if (!okw) { M.abort = 1; set_status(status, CSA2_DEV_TIMEOUT); }
            if (__any_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&M.abort) != 0)) break;
            tc::tc_fence_after();
            if (lane == 0) {
                const uint32_t aaddr = tc::smem_u32(sm + kOffStages + s * kStageBytes);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    tc::mma_mxf4(tbase + 16 * c, tc::sw128_desc(aaddr + 32 * j), tc::sw128_desc(qaddr + 32 * j), idesc,
                                 tbase + kSfaCol, tbase + kSfbCol, j > 0);
                tc::mma_commit(&M.accf[c]);
                tc::mma_commit(&M.empty[s]);
            }
            __syncwarp();
        }
    } else if (warp >= 4) {
        // ---- epilogue: exact keys into tensor memory, histogram, block maxima; warps 4-7 take the
        // even tiles, warps 8-11 the odd ones ----
        const int q = warp & 3, grp = (warp - 4) >> 2;
        const int pt = 32 * q + lane;  // position within the tile
        const int64_t row0 = (int64_t)R.b * a.c.cap;
        float qf[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) qf[j] = M.qf[j];
        uint4 scr[kScaleAhead];
#pragma unroll
        for (int j = 0; j < kScaleAhead; ++j) scr[j] = load_scales(a, blkid, n_units, row0, grp + 2 * j, pt);
        unsigned long long* cand_k = reinterpret_cast<unsigned long long*>(sm + kOffCandK);
        int* cand_e = reinterpret_cast<int*>(sm + kOffCandE);
        // the accumulator of this warp's next tile is requested as soon as it is complete, so that its
        // load overlaps the current tile's arithmetic
        uint32_t dn[16];
        bool pending = false;  // a load of this tile's accumulator is already in flight
        for (int i = grp; i < ntiles; i += 2) {
            const int c = i % kAcc;
            if (!pending) {
                if (!tc::mbar_wait(&M.accf[c], (uint32_t)(i / kAcc) & 1u, kWaitNs)) {
                    M.abort = 1;
                    set_status(status, CSA2_DEV_TIMEOUT);
                }
                if (__any_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&M.abort) != 0)) break;
                tc::tc_fence_after();
                tc::tmem_ld16(tbase + ((uint32_t)(32 * q) << 16) + 16 * c, dn);
            }
            tc::tmem_ld_wait();
            pending = false;
            uint32_t d[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) d[j] = dn[j];
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&M.acce[c]);
            if (i + 2 < ntiles) {
                const int cn = (i + 2) % kAcc;
                if (__all_sync(0xffffffffu, tc::mbar_try_wait(&M.accf[cn], (uint32_t)((i + 2) / kAcc) & 1u, 0u))) {
                    tc::tc_fence_after();
                    tc::tmem_ld16(tbase + ((uint32_t)(32 * q) << 16) + 16 * cn, dn);
                    pending = true;
                }
            }
            const int u = i * kTileUnits + (pt >> 3);
            const int info = u < n_units ? uinfo[u] : -16;
            const uint4 sc4 = scr[0];
#pragma unroll
            for (int j = 0; j < kScaleAhead - 1; ++j) scr[j] = scr[j + 1];
            scr[kScaleAhead - 1] = load_scales(a, blkid, n_units, row0, i + 2 * kScaleAhead, pt);
            const bool valid = info >= 0 && (pt & 7) < (info & 15);
            const uint32_t scw[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
            long long acc = 0;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                long long hs = 0;
                const uint32_t w = scw[h];
                const float2 s01 = h2_to_f2(e4m3x2_to_h2((uint16_t)(w & 0xFFFF)));
                const float2 s23 = h2_to_f2(e4m3x2_to_h2((uint16_t)(w >> 16)));
                const float sk[4] = {s01.x, s01.y, s23.x, s23.y};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int bb = 4 * h + j;
                    const float v = (__uint_as_float(d[bb]) * sk[j]) * qf[bb];
                    hs += __float2ll_rn(v);
                }
                acc += RELU ? (hs > 0 ? hs : 0) : hs;
            }
            const unsigned long long key = valid ? ((unsigned long long)acc ^ 0x8000000000000000ull) : 0ull;
            tc::tmem_st2(tbase + ((uint32_t)(32 * q) << 16) + kKeyCol + 2 * i, (uint32_t)key, (uint32_t)(key >> 32));
            const int kb = valid ? kbin(key) : -1;
            if (valid) atomicAdd(&hist[kb], 1u);
            // candidates: every key whose bin is not below the provisional cut (a lower bound of the
            // final cut bin, since counts only grow)
            const bool take = valid && kb >= *reinterpret_cast<volatile int*>(&M.lbin);
            const unsigned int tb = __ballot_sync(0xffffffffu, take);
            if (tb) {
                int base = 0;
                if (lane == 0) base = atomicAdd(&M.ncand, __popc(tb));
                base = __shfl_sync(0xffffffffu, base, 0) + __popc(tb & ((1u << lane) - 1u));
                if (take && base < kCandCap) { cand_k[base] = key; cand_e[base] = i * kTileP + pt; }
            }
            if (POOL) {
                unsigned long long bm = key, o;
                o = __shfl_xor_sync(0xffffffffu, bm, 1); bm = o > bm ? o : bm;
                o = __shfl_xor_sync(0xffffffffu, bm, 2); bm = o > bm ? o : bm;
                o = __shfl_xor_sync(0xffffffffu, bm, 4); bm = o > bm ? o : bm;
                const int uu = (i * kTileP + pt) >> 3;
                if ((pt & 7) == 0 && uu < n_units) {
                    bkeys[uu] = bm;
                    if (bm) atomicAdd(&phist[kbin(bm)], 1u);
                }
            }
            // warp 4 raises the provisional cut every 8 of its tiles: the bin where the counts so far,
            // read from the top, reach k (lane l covers bins 2047 - 64 l .. 2047 - 64 l - 63)
            if (warp == 4 && (i & 15) == 14) {
                const int K = a.plan.k;
                const volatile unsigned int* vh = hist;
                unsigned int sum = 0;
                for (int j = 0; j < 64; ++j) sum += vh[kKeyBins - 1 - (64 * lane + j)];
                unsigned int incl = sum;
#pragma unroll
                for (int o2 = 1; o2 < 32; o2 <<= 1) {
                    const unsigned int t2 = __shfl_up_sync(0xffffffffu, incl, o2);
                    if (lane >= o2) incl += t2;
                }
                const unsigned int excl = incl - sum;
                int cut = -1;
                if (excl < (unsigned)K && incl >= (unsigned)K) {
                    // the counts were read above; re-reading can only find larger ones, so the bin
                    // found this way is still a lower bound of the final cut
                    unsigned int run = excl;
                    for (int j = 0; j < 64; ++j) {
                        run += vh[kKeyBins - 1 - (64 * lane + j)];
                        if (run >= (unsigned)K) {
                            cut = kKeyBins - 1 - (64 * lane + j);
                            break;
                        }
                    }
                }
#pragma unroll
                for (int o2 = 16; o2 > 0; o2 >>= 1) cut = max(cut, __shfl_xor_sync(0xffffffffu, cut, o2));
                if (lane == 0 && cut > M.lbin) M.lbin = cut;
            }
        }
        tc::tmem_ld_wait();
        tc::tmem_st_wait();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (M.abort) {
        if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);
        return;
    }
    if (warp >= 8) return;  // the selection runs on warps 0-7 (named barrier 1)

    // ---- selection ----
    const int K = a.plan.k;
    int32_t* out = a.out_idx + (size_t)row * K;
    if (a.reindex) {
        for (int u = tid; u + 1 < n_units; u += kT)
            if (blkid[u] >= blkid[u + 1]) M.unsorted = 1;
        sel_sync();
    }
    const bool sorted = !a.reindex || M.unsorted == 0;
    // invalid pool entries have no keys: their block id only has to stay a valid position for pos()
    if (a.reindex) {
        for (int u = tid; u < n_units; u += kT)
            if (blkid[u] < 0) blkid[u] = 0;
        sel_sync();
    }
    // the candidates kept during the scan hold every key at or above the cut bin unless they overflowed
    const int nc = M.ncand;
    const bool list = nc <= kCandCap;
    select_keys(TmemKeys{tbase, ntiles}, ntiles * kTileP, K, hist, Pos{a.reindex ? blkid : nullptr}, sorted, out,
                sm + kOffStages, M, list ? reinterpret_cast<const unsigned long long*>(sm + kOffCandK) : nullptr,
                reinterpret_cast<const int*>(sm + kOffCandE), nc);
    tc::tc_fence_before();
    sel_sync();
    tc::tc_fence_after();
    if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);
    if (POOL) {
        const int P = a.plan.pool_blocks;
        const int cnt = select_keys(SmemKeys{bkeys, n_units}, n_units, P, phist, Pos{nullptr}, true,
                                    a.out_pool + (size_t)row * P, sm + kOffStages, M);
        if (tid == 0) a.out_pool_n[row] = cnt;
    }
}

}  // namespace

bool index_tc_fits(const IndexPlan& p) {
    return p.decode && p.units_max <= kFusedUnits && p.k <= kMaxK && p.pool_blocks <= kFusedUnits;
}

// cuTensorMapEncodeTiled from the driver, looked up once
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

cudaError_t launch_index_tc(const IndexArgs& a, cudaStream_t s) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    // the indexer code plane as [sequence][position][128 bytes]; a box is one pool block of 8
    // positions (Reindex) or a tile of 128 (Full); positions past the capacity read as zeros
    CUtensorMap map;
    const cuuint64_t gdim[3] = {(cuuint64_t)kIKBytes, (cuuint64_t)a.c.cap, (cuuint64_t)a.plan.rows};
    const cuuint64_t gstr[2] = {(cuuint64_t)kIKBytes, (cuuint64_t)a.c.cap * kIKBytes};
    const cuuint32_t box[3] = {(cuuint32_t)kIKBytes, (cuuint32_t)(a.reindex ? kBS : kTileP), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.c.ik_data, gdim, gstr, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const bool relu = (a.flags & CSA2_SCORE_RELU) != 0;
    const bool pool = a.plan.pool_blocks > 0 && !a.reindex;
    void (*k)(const IndexArgs, const CUtensorMap) =
        relu ? (pool ? index_tc_kernel<true, true> : index_tc_kernel<true, false>)
             : (pool ? index_tc_kernel<false, true> : index_tc_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    if (a.plan.rows == 0) return cudaSuccess;
    return launch_after_prior(k, dim3((unsigned)a.plan.rows), dim3(kTAll), (size_t)kSmemBytes, s, a, map);
}

}  // namespace csa2
