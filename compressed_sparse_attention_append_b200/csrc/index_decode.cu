// index_decode.cu -- the index step for decode rows (one query row per sequence): zero_kernel,
// score_kernel, select_kernel.
//
// Same method and the same exact integer scores as index.cu (see its header): [B] "DeepSeek Cuts
// KV Cache Footprint Fourfold", "Technical Approach" (Full / Reindex selection); [C] "DeepSeek-V4.1-
// Flash: Pushing KV Cache Compression to 890 Bytes per Token", sec. VI "Shortlist-of-a-shortlist"
// and sec. IX Figure 4 (block pool), sec. XI (FP4 indexer queries and keys).
//
// zero_kernel: clears the rows' score histograms.
// Every kernel here launches with programmatic stream serialisation and waits for the kernel
// before it (griddepcontrol.wait) before touching memory that kernel may use.
// score_kernel: CTAs of 8 independent warps, two per SM. The rows' steps of 4 units (32 positions)
//   are laid end to end and split evenly over all resident warps; each warp streams its steps
//   through a private 3-stage cp.async ring. Lane l scores step position l on its own (all 256
//   channels: 32 code words against the row's query words, broadcast from the warp's shared slot),
//   so no cross-lane sum is needed. It writes one orderable 64-bit key per position (0 for a
//   position that is not visible), counts each key into the row's histogram by key_bin, and for a
//   Full pool writes (and counts) the maximum key of each unit. No block-wide synchronisation.
// select_kernel: rows x slices of CTAs, one resident wave. The row's histogram gives the bin that
//   holds its k-th largest key; every CTA appends its keys in that bin or above to the row's
//   candidate list (and counts the cut-bin keys into a second-level histogram); the last CTA of
//   the row takes the keys above the cut, ranks the few keys left at the second-level cut exactly
//   (ties to the lower position), and writes the positions in ascending order. Then the pool (top
//   blocks by maximum key, ties to the lower block id) the same way. Rows the histograms cannot
//   settle fall back to an exact radix select over all of the row's keys.
#include "csa2_internal.cuh"

namespace csa2 {

namespace {

constexpr int kSThreads = 256;                 // score kernel: 8 warps, 2 CTAs per SM
constexpr int kSWarps = kSThreads / 32;
constexpr int kSStages = 3;
constexpr int kUnitsPerStep = 4;               // 32 positions per warp step
constexpr int kStepBytes = kUnitsPerStep * (1024 + 128);
constexpr int kWarpBytes = kSStages * kStepBytes + 512;  // staging ring + query words
constexpr int kQThreads = 128;                 // select kernel: 4 warps, up to 8 CTAs per SM
constexpr int kQWarps = kQThreads / 32;
constexpr int kPerT = 8;                       // keys per select thread and batch
constexpr int kBatch = kPerT * kQThreads;      // keys per batch (kBatch / 8 units: one per thread)
constexpr int kTie = 256;                      // keys of the second-level cut bin ranked pairwise
constexpr int kCtaCand = 512;                  // candidates a select CTA gathers before one flush
constexpr int kMapBits = 131072;               // longest row whose selection is read out in order

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
constexpr uint32_t kTab0 = 0x03020100u, kTab1 = 0x0C080604u;  // 2 * E2M1 magnitudes

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
__device__ __forceinline__ uint32_t e2m1_int2(uint32_t c) {
    const uint32_t mag = (prmt(kTab0, kTab1, c & 7) & 0xFF);
    return (c & 8) ? ((0u - mag) & 0xFF) : mag;
}

struct DRow {
    int64_t qpos;  // the last visible entry: floor((query token + 1) / ratio) - 1
    int b;
    int n_units;
};

__device__ __forceinline__ DRow drow(const IndexArgs& a, int row, bool& ok) {
    DRow r;
    r.b = row;  // decode: tq == 1
    const int64_t tok = a.qpos ? a.qpos[row] : a.qpos_base;
    r.qpos = tok < 0 ? -1 : (tok + 1) / a.ratio - 1;
    ok = !(tok < 0 || r.qpos >= a.c.cap || (!a.reindex && r.qpos >= a.max_ctx));
    if (!ok) {
        r.n_units = 0;
    } else if (a.reindex) {
        int n = a.pool_n[r.b];
        r.n_units = n < 0 ? 0 : (n > a.pool_stride ? a.pool_stride : n);
    } else {
        r.n_units = (int)((r.qpos + kBS) / kBS);
    }
    return r;
}

// Unit u of row R with block id `id` (u itself in Full mode) -> packed (blk << 4) | positions to
// score (0..8); -16 when the unit is past the row or its id is invalid.
__device__ __forceinline__ int unit_pack(const IndexArgs& a, const DRow& R, int u, int id, uint32_t* status) {
    if (u >= R.n_units) return -16;
    if (a.reindex && (id < 0 || (int64_t)id * kBS >= a.c.cap)) {
        set_status(status, CSA2_DEV_BAD_POOL);
        return -16;
    }
    const int64_t p0 = (int64_t)id * kBS;
    int64_t n = R.qpos - p0 + 1;
    if (a.c.cap - p0 < n) n = a.c.cap - p0;
    if (n <= 0) return -16;
    return (id << 4) | (int)(n > kBS ? kBS : n);
}

__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, int src_bytes) {
    uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(src_bytes));
}

// Step layout in shared memory (32 positions, lane l owns step position P = l = 8 * unit + index):
//   [0, 4096)      codes: position P at 128 P; its 16-byte chunk c at ((c ^ (P & 7)) << 4), so
//                  that the 8 lanes of a quarter-warp reading chunk c hit 8 different bank groups
//   [4096, 4608)   scales: position P at 4096 + 16 P
// Chunk q = 32 h + l of a unit's 1024 code bytes is position 4 h + (l >> 3), chunk l & 7: lane l
// copies it to 1024 u + 512 h + 128 (l >> 3) + ((((l & 7) ^ (l >> 3)) << 4) ^ 64 h).
// Copies of positions that are not scored read nothing and fill zeros.
struct StageLane {
    int dst0, dst1;  // code destinations of this lane within a unit (h = 0, 1)
    int m, idx;      // lane >> 3, lane & 7
};

__device__ __forceinline__ void stage_step(const IndexArgs& a, int b, int packed, unsigned char* st,
                                           const StageLane& L) {
    const int lane = threadIdx.x & 31;
    const uint8_t* base = a.c.ik_data + (size_t)b * a.c.cap * kIKBytes;
    const uint8_t* sbase = a.c.ik_scale + (size_t)b * a.c.cap * kIKScales;
#pragma unroll
    for (int u = 0; u < kUnitsPerStep; ++u) {
        const int pk = __shfl_sync(0xffffffffu, packed, u);
        const int blk = pk >> 4, n = pk & 15;
        const uint8_t* cb = base + (size_t)(blk < 0 ? 0 : blk) * (kBS * kIKBytes) + 16 * lane;
        cp_async16_zfill(st + 1024 * u + L.dst0, cb, (blk >= 0 && L.m < n) ? 16 : 0);
        cp_async16_zfill(st + 1024 * u + L.dst1, cb + 512, (blk >= 0 && 4 + L.m < n) ? 16 : 0);
    }
    const int pk = __shfl_sync(0xffffffffu, packed, L.m);
    const int blk = pk >> 4, n = pk & 15;
    cp_async16_zfill(st + 4096 + 16 * lane,
                     sbase + ((size_t)(blk < 0 ? 0 : blk) * kBS + L.idx) * kIKScales, (blk >= 0 && L.idx < n) ? 16 : 0);
}

// Indexer query of one row into the warp's slot: q4[w] = {2q of channels 8w..8w+3, of 8w+4..8w+7,
// and both negated} as signed bytes; returns in every lane the fixed-point scale of block (lane & 15).
// Lane l quantises word l (block l >> 1).
__device__ __forceinline__ int quantize_query_warp(const uint16_t* q, uint4* q4, const int* kf_lut) {
    const int lane = threadIdx.x & 31;
    const uint4 x4 = *reinterpret_cast<const uint4*>(q + 8 * lane);
    const uint32_t xw[4] = {x4.x, x4.y, x4.z, x4.w};
    float x[8], amax = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(xw[i] << 16);
        x[2 * i + 1] = __uint_as_float(xw[i] & 0xFFFF0000u);
        amax = fmaxf(amax, fmaxf(fabsf(x[2 * i]), fabsf(x[2 * i + 1])));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));  // block of 16 = lanes 2b, 2b+1
    const uint32_t sc = q_f32_to_e4m3(__fdiv_rn(amax, 6.0f));
    const float sv = __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)sc, __NV_E4M3)));
    uint32_t cw = 0;
    if (sv != 0.f) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            cw |= q_f32x2_to_e2m1x2(__fdiv_rn(x[2 * i], sv), __fdiv_rn(x[2 * i + 1], sv)) << (8 * i);
    }
    uint32_t pa = 0, pb = 0, na = 0, nb = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t va = e2m1_int2((cw >> (4 * j)) & 15), vb = e2m1_int2((cw >> (16 + 4 * j)) & 15);
        pa |= va << (8 * j);
        pb |= vb << (8 * j);
        na |= ((0u - va) & 0xFF) << (8 * j);
        nb |= ((0u - vb) & 0xFF) << (8 * j);
    }
    q4[lane] = make_uint4(pa, pb, na, nb);
    __syncwarp();
    return __shfl_sync(0xffffffffu, kf_lut[sc], 2 * (lane & 15));
}

// Signed dot product of 8 E2M1 codes (one 32-bit word, low nibble first) with 8 query values held
// as 2q in signed bytes (qa: codes 0..3, qb: codes 4..7; nqa, nqb negated): 4 * sum(code value * q).
// prmt's sign-replicate mode maps codes with the sign bit to 0, so one lookup takes the positive
// codes and a second, on the word with every sign bit flipped, the negative ones.
__device__ __forceinline__ int dot8p(uint32_t w, uint32_t qa, uint32_t qb, uint32_t nqa, uint32_t nqb, int acc,
                                     uint32_t t0, uint32_t t1) {
    const uint32_t wx = w ^ 0x88888888u;
    acc = __dp4a((int)prmt(t0, t1, w), (int)qa, acc);
    acc = __dp4a((int)prmt(t0, t1, wx), (int)nqa, acc);
    acc = __dp4a((int)prmt(t0, t1, __umulhi(w, 0x10000u)), (int)qb, acc);
    acc = __dp4a((int)prmt(t0, t1, __umulhi(wx, 0x10000u)), (int)nqb, acc);
    return acc;
}

template <bool RELU, bool POOL>
__global__ void __launch_bounds__(kSThreads, 2) score_kernel(IndexArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int kf_lut[256];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < 256; i += kSThreads) kf_lut[i] = e4m3_fixed(i);
    __syncthreads();
    wait_prior_grid();  // the cache and the zeroed histograms come from earlier kernels
    // the magnitude table lives in registers for the whole kernel
    uint32_t t0, t1;
    asm volatile("mov.b32 %0, 0x03020100;" : "=r"(t0));
    asm volatile("mov.b32 %0, 0x0C080604;" : "=r"(t1));
    uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + kHdrStatus);
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(a.ws + a.L.cand_key);
    unsigned long long* bmax = reinterpret_cast<unsigned long long*>(a.ws + a.L.bmax);
    unsigned int* hist = reinterpret_cast<unsigned int*>(a.ws + a.L.key_hist);
    const size_t row_keys = (size_t)a.plan.units_max * kBS;
    // static schedule: the rows' steps of 4 units, laid end to end, split evenly over the warps
    const int spr = (a.plan.units_max + kUnitsPerStep - 1) / kUnitsPerStep;
    const int row_units = spr * kUnitsPerStep;
    const long long total = (long long)a.plan.rows * spr;
    const long long gw = (long long)blockIdx.x * kSWarps + warp, nw = (long long)gridDim.x * kSWarps;
    const long long s0 = total * gw / nw, s1 = total * (gw + 1) / nw;
    const int nsteps = (int)(s1 - s0);
    unsigned char* wst = smem + (size_t)warp * kWarpBytes;
    uint4* q4 = reinterpret_cast<uint4*>(wst + kSStages * kStepBytes);
    StageLane SL;
    SL.m = lane >> 3;
    SL.idx = lane & 7;
    {
        const int cm = ((lane & 7) ^ (lane >> 3)) << 4;
        SL.dst0 = 128 * SL.m + cm;
        SL.dst1 = 512 + 128 * SL.m + (cm ^ 64);
    }
    // staging cursor (kSStages - 1 steps ahead of the compute cursor); in Reindex mode lanes 0..3
    // hold the pool ids of the next step to stage, loaded one step early
    int s_row = (int)(s0 / spr), s_su = (int)(s0 % spr) * kUnitsPerStep;
    int c_row = s_row, c_su = s_su;
    int srow_cached = -1, crow_cached = -1;
    DRow SR{}, CR{};
    bool sok = true;
    auto load_ids = [&](int row, int su) -> int {
        if (!a.reindex) return su + lane;
        const int u = su + lane;
        return (lane < kUnitsPerStep && row < a.plan.rows && u < a.pool_stride)
                   ? __ldg(a.pool + (size_t)row * a.pool_stride + u) : -1;
    };
    int ids = load_ids(s_row, s_su);
    auto stage = [&](int slot) -> int {
        if (s_row != srow_cached) { srow_cached = s_row; SR = drow(a, s_row, sok); }
        if (s_su == 0 && !sok && lane == 0) set_status(status, CSA2_DEV_BAD_POS);
        const int su = s_su;
        s_su += kUnitsPerStep;
        if (s_su >= row_units) { s_su = 0; ++s_row; }
        const int cur = ids;
        ids = load_ids(s_row, s_su);  // prefetch for the next call
        if (su >= SR.n_units) return -16;
        const int packed = lane < kUnitsPerStep ? unit_pack(a, SR, su + lane, cur, status) : -16;
        stage_step(a, SR.b, packed, wst + slot * kStepBytes, SL);
        return packed;
    };
    int pk0 = -16, pk1 = -16, pk2 = -16;
#pragma unroll
    for (int i = 0; i < kSStages - 1; ++i) {
        if (i < nsteps) {
            const int p = stage(i);
            if (i == 0) pk0 = p; else pk1 = p;
        }
        cp_async_commit();
    }
    int qf = 0;
    for (int i = 0; i < nsteps; ++i) {
        const int nx = i + kSStages - 1;
        if (nx < nsteps) {
            const int sl = nx % kSStages;
            const int p = stage(sl);
            if (sl == 0) pk0 = p; else if (sl == 1) pk1 = p; else pk2 = p;
        }
        cp_async_commit();
        const int row = c_row, su = c_su;
        c_su += kUnitsPerStep;
        if (c_su >= row_units) { c_su = 0; ++c_row; }
        if (row != crow_cached) {
            bool ok;
            crow_cached = row;
            CR = drow(a, row, ok);
            if (CR.n_units > 0) qf = quantize_query_warp(a.idx_q + (size_t)row * (kHI * kDI), q4, kf_lut);
        }
        cp_async_wait<kSStages - 1>();
        __syncwarp();
        if (su < CR.n_units) {
            const int sl = i % kSStages;
            const unsigned char* st = wst + sl * kStepBytes;
            const int packed = sl == 0 ? pk0 : (sl == 1 ? pk1 : pk2);
            const int P = lane;
            const uint4 sc4 = *reinterpret_cast<const uint4*>(st + 4096 + 16 * P);
            const uint32_t scw[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
            long long acc = 0, hacc = 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 kw = *reinterpret_cast<const uint4*>(st + 128 * P + ((c ^ (P & 7)) << 4));
                const uint4 a0 = q4[4 * c], a1 = q4[4 * c + 1], a2 = q4[4 * c + 2], a3 = q4[4 * c + 3];
                int d0 = dot8p(kw.x, a0.x, a0.y, a0.z, a0.w, 0, t0, t1);
                d0 = dot8p(kw.y, a1.x, a1.y, a1.z, a1.w, d0, t0, t1);
                int d1 = dot8p(kw.z, a2.x, a2.y, a2.z, a2.w, 0, t0, t1);
                d1 = dot8p(kw.w, a3.x, a3.y, a3.z, a3.w, d1, t0, t1);
                const uint32_t sw = scw[c >> 1] >> (16 * (c & 1));
                const int qf0 = __shfl_sync(0xffffffffu, qf, 2 * c), qf1 = __shfl_sync(0xffffffffu, qf, 2 * c + 1);
                const long long v = (long long)(d0 * kf_lut[sw & 0xFF]) * qf0 +
                                    (long long)(d1 * kf_lut[(sw >> 8) & 0xFF]) * qf1;
                if (RELU) {  // head h covers chunks 2h, 2h+1
                    hacc += v;
                    if (c & 1) { acc += hacc > 0 ? hacc : 0; hacc = 0; }
                } else {
                    acc += v;
                }
            }
            const int u = lane >> 3, idx = lane & 7;
            const int pk = __shfl_sync(0xffffffffu, packed, u);
            const bool valid = (pk >> 4) >= 0 && idx < (pk & 15);
            const unsigned long long key = valid ? ((unsigned long long)acc ^ 0x8000000000000000ull) : 0ull;
            const bool in_row = su + u < CR.n_units;  // keys past the row's last unit are never read
            unsigned int* hrow = hist + (size_t)row * kRowHist;
            if (in_row) {
                keys[(size_t)row * row_keys + (size_t)(su + u) * kBS + idx] = key;
                if (valid) atomicAdd(hrow + key_bin(key), 1u);
            }
            if (POOL) {
                unsigned long long bm = key, o;
                o = shfl_xor_u64(bm, 1); bm = o > bm ? o : bm;
                o = shfl_xor_u64(bm, 2); bm = o > bm ? o : bm;
                o = shfl_xor_u64(bm, 4); bm = o > bm ? o : bm;
                if (idx == 0 && in_row) {
                    bmax[(size_t)row * ((a.plan.units_max + 1) & ~1) + su + u] = bm;
                    if (bm) atomicAdd(hrow + kKeyBins + key_bin(bm), 1u);
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
}

// ---- select kernel ---------------------------------------------------------------------------------
// Grid: rows x slices, sized to one wave of resident CTAs. A slice is a run of batches of kBatch
// keys. Every CTA finds the row's cut bin from the histograms and appends the keys of its batches at
// or above it (with their element index and position) to the row's candidate list; the last CTA of
// the row to finish ranks the candidates exactly. The first batch is requested before the histograms
// are read, so a CTA waits for memory about once per batch, once for its ticket and (the last) once
// for the candidates.

struct SelScal {
    int digit, above, cnt, nemit, ntie, last;
    unsigned long long red_and[kQWarps], red_or[kQWarps];
    int nv[kQWarps], wsum[kQWarps];
};

// Position of element i of a row: 8 * pool[i / 8] + i % 8 in Reindex mode, else i.
struct PosMap {
    const int32_t* prow;
    __device__ __forceinline__ int operator()(int i) const {
        return prow ? __ldg(prow + (i >> 3)) * kBS + (i & 7) : i;
    }
};

struct SelSmem {
    unsigned long long* tk;  // keys of the second-level cut bin [kTie]
    int* ti;                 // their element index [kTie]
    int* tp;                 // their position [kTie]
    int* si;                 // selected element indices [kMaxK]
    int* list;               // selected positions [kMaxK]
    unsigned int* bitmap;    // selected elements of the row [ceil(n / 32)]
    unsigned short* wpre;    // selected elements before each bitmap word
    unsigned int* hist;      // radix histogram [256]
};

// Shared memory of a select CTA for rows of at most nmax elements (bitmap only up to kMapBits).
__host__ __device__ inline size_t sel_smem_bytes(int nmax) {
    const size_t words = nmax <= kMapBits ? (size_t)(nmax + 31) / 32 : 0;
    const size_t rank = (size_t)16 * kTie + (size_t)8 * kMaxK + 4 * 256 + 4 * words + ((2 * words + 15) & ~(size_t)15);
    const size_t lists = (size_t)32 * kCtaCand;  // the CTA's candidate lists, before the ranking
    return rank > lists ? rank : lists;
}

__device__ inline SelSmem sel_smem(unsigned char* p, int nmax) {
    const size_t words = nmax <= kMapBits ? (size_t)(nmax + 31) / 32 : 0;
    SelSmem M;
    M.tk = reinterpret_cast<unsigned long long*>(p); p += 8 * kTie;
    M.ti = reinterpret_cast<int*>(p); p += 4 * kTie;
    M.tp = reinterpret_cast<int*>(p); p += 4 * kTie;
    M.si = reinterpret_cast<int*>(p); p += 4 * kMaxK;
    M.list = reinterpret_cast<int*>(p); p += 4 * kMaxK;
    M.hist = reinterpret_cast<unsigned int*>(p); p += 4 * 256;
    M.bitmap = reinterpret_cast<unsigned int*>(p); p += 4 * words;
    M.wpre = reinterpret_cast<unsigned short*>(p);
    return M;
}

__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0;
    total = 0;
    for (int w = 0; w < kQWarps; ++w) {
        const int c = wsum[w];
        before += w < warp ? c : 0;
        total += c;
    }
    __syncthreads();
    return before + incl - v;
}

// Scan of a 256-bin histogram by warp 0: the bin where the running count (from the top bin when
// desc, else from bin 0) reaches kr; S.digit / S.above (count before it) / S.cnt (its count).
__device__ void scan_bins(const unsigned int* hist, int kr, bool desc, SelScal& S) {
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
                S.digit = desc ? 255 - 8 * lane - j : 8 * lane + j;
                S.above = (int)run;
                S.cnt = (int)c[j];
                break;
            }
            run += c[j];
        }
    }
}

// ---- exact radix select (the path for rows the histogram cut cannot settle) ------------------------
// Mode 0: at most K valid keys, all taken. Mode 1: exactly K keys have (key & mask) >= prefix.
// Mode 2: the K-th largest key equals prefix; kr of the keys equal to it are still to be taken.
struct Thr {
    unsigned long long prefix, mask;
    int kr, mode;
};

__device__ Thr kth_threshold(int n, int K, const unsigned long long* key, unsigned int* hist, SelScal& S) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned long long va = ~0ull, vo = 0ull;
    int nv = 0;
    for (int i = tid; i < n; i += kQThreads) {
        const unsigned long long k = key[i];
        if (k) { va &= k; vo |= k; ++nv; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        va &= shfl_xor_u64(va, o);
        vo |= shfl_xor_u64(vo, o);
        nv += __shfl_xor_sync(0xffffffffu, nv, o);
    }
    if (lane == 0) { S.red_and[warp] = va; S.red_or[warp] = vo; S.nv[warp] = nv; }
    __syncthreads();
    va = ~0ull; vo = 0ull; nv = 0;
    for (int w = 0; w < kQWarps; ++w) { va &= S.red_and[w]; vo |= S.red_or[w]; nv += S.nv[w]; }
    __syncthreads();
    Thr t{0ull, 0ull, K, 0};
    if (nv <= K) return t;
    const unsigned long long diff = va ^ vo;
    int top = diff ? 63 - __clzll((long long)diff) : -1;
    t.mask = top < 0 ? ~0ull : (top >= 63 ? 0ull : ~((2ull << top) - 1ull));
    t.prefix = va & t.mask;
    t.mode = 2;
    while (top >= 0) {
        const int shift = top >= 7 ? top - 7 : 0;
        const unsigned int dmask = (1u << (top - shift + 1)) - 1u;
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int base = 0; base < n; base += kQThreads) {
            const int i = base + tid;
            int d = -1;
            if (i < n) {
                const unsigned long long k = key[i];
                if (k && (k & t.mask) == t.prefix) d = (int)((k >> shift) & dmask);
            }
            const unsigned int peers = __match_any_sync(0xffffffffu, d);
            if (d >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (unsigned)__popc(peers));
        }
        __syncthreads();
        if (warp == 0) scan_bins(hist, t.kr, true, S);
        __syncthreads();
        t.kr -= S.above;
        t.prefix |= (unsigned long long)S.digit << shift;
        t.mask |= (unsigned long long)dmask << shift;
        const bool exact = S.cnt == t.kr;
        top = shift - 1;
        __syncthreads();
        if (exact) { t.mode = 1; break; }
    }
    return t;
}

// Mode 2: the largest position among the kr lowest positions whose key equals t.prefix.
__device__ unsigned int tie_threshold(int n, const Thr& t, const unsigned long long* key, PosMap pos,
                                      unsigned int* hist, SelScal& S) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned int pp = 0, pm = 0;
    int r = t.kr;
    for (int shift = 24; shift >= 0; shift -= 8) {
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int base = 0; base < n; base += kQThreads) {
            const int i = base + tid;
            int d = -1;
            if (i < n && key[i] == t.prefix) {
                const unsigned int p = (unsigned int)pos(i);
                if ((p & pm) == pp) d = (int)((p >> shift) & 255u);
            }
            const unsigned int peers = __match_any_sync(0xffffffffu, d);
            if (d >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (unsigned)__popc(peers));
        }
        __syncthreads();
        if (warp == 0) scan_bins(hist, r, false, S);
        __syncthreads();
        r -= S.above;
        pp |= (unsigned int)S.digit << shift;
        pm |= 0xFFu << shift;
        const bool fin = S.cnt == r;
        __syncthreads();
        if (fin) break;
    }
    return pp | ~pm;
}

// ascending bitonic sort of n <= kMaxK ints in a (room for the next power of two)
__device__ void sort_asc(int* a, int n) {
    int P = 1;
    while (P < n) P <<= 1;
    for (int i = n + threadIdx.x; i < P; i += kQThreads) a[i] = 0x7FFFFFFF;
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < P; i += kQThreads) {
                const int l = i ^ j;
                if (l > i) {
                    const int x = a[i], y = a[l];
                    if ((x > y) == ((i & k) == 0)) { a[i] = y; a[l] = x; }
                }
            }
            __syncthreads();
        }
    }
}

// Exact Top-K of the n keys key[0..n) by radix select; ascending positions to out, padded with -1.
__device__ int radix_topk(int n, int K, const unsigned long long* key, PosMap pos, int32_t* out, const SelSmem& M,
                          SelScal& S) {
    const int tid = threadIdx.x, lane = tid & 31;
    const Thr t = kth_threshold(n, K, key, M.hist, S);
    const unsigned int pthr = t.mode == 2 ? tie_threshold(n, t, key, pos, M.hist, S) : 0xFFFFFFFFu;
    if (tid == 0) S.nemit = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kQThreads) {
        const int i = base + tid;
        bool sel = false;
        int p = 0;
        if (i < n) {
            const unsigned long long k = key[i];
            if (k) {
                if (t.mode == 0) sel = true;
                else if (t.mode == 1) sel = (k & t.mask) >= t.prefix;
                else sel = k > t.prefix || (k == t.prefix && (unsigned int)pos(i) <= pthr);
                if (sel) p = pos(i);
            }
        }
        const unsigned int bal = __ballot_sync(0xffffffffu, sel);
        int wb = 0;
        if (lane == 0 && bal) wb = atomicAdd(&S.nemit, __popc(bal));
        wb = __shfl_sync(0xffffffffu, wb, 0);
        const int o = wb + __popc(bal & ((1u << lane) - 1));
        if (sel && o < K) M.list[o] = p;
    }
    __syncthreads();
    const int cnt = S.nemit < K ? S.nemit : K;
    sort_asc(M.list, cnt);
    for (int i = tid; i < K; i += kQThreads) out[i] = i < cnt ? M.list[i] : -1;
    return cnt;
}

// The cut bin of a histogram h[0..nbins) (nbins = 1024 or 2048): fewer than K counted keys lie
// above it, at least K at or above it. Returns -1 when at most K keys are counted; *above = the
// count above the cut bin.
__device__ int cut_bin(const unsigned int* h, int nbins, int K, SelScal& S, int* above) {
    const int tid = threadIdx.x;
    const int per = nbins / kQThreads;  // 8 or 16
    unsigned int hb[kKeyBins / kQThreads];
    int sum = 0;
    const uint4* hv = reinterpret_cast<const uint4*>(h + nbins - per * (tid + 1));  // 16-byte aligned
#pragma unroll
    for (int q = 0; q < kKeyBins / kQThreads / 4; ++q) {
        const uint4 v = 4 * q < per ? __ldcg(hv + q) : make_uint4(0u, 0u, 0u, 0u);
        hb[4 * q] = v.x; hb[4 * q + 1] = v.y; hb[4 * q + 2] = v.z; hb[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int j = 0; j < kKeyBins / kQThreads; ++j) sum += (int)hb[j];
    if (tid == 0) { S.digit = -1; S.above = 0; }
    int total;
    const int excl = block_excl_scan(sum, S.wsum, total);  // its barriers order the reset above
    if (total > K && excl < K && excl + sum >= K) {
        int run = excl;
        for (int j = per - 1; j >= 0; --j) {
            if (run + (int)hb[j] >= K) {
                S.digit = nbins - per * (tid + 1) + j;
                S.above = run;
                break;
            }
            run += (int)hb[j];
        }
    }
    __syncthreads();
    *above = S.above;
    const int d = S.digit;
    __syncthreads();
    return d;
}

// Warp-aggregated append of (element, position) to the selected list (at most K kept).
__device__ __forceinline__ void add_selected(bool sel, int i, int p, int K, bool in_order, const SelSmem& M, SelScal& S) {
    const int lane = threadIdx.x & 31;
    const unsigned int bal = __ballot_sync(0xffffffffu, sel);
    if (!bal) return;
    int wb = 0;
    if (lane == 0) wb = atomicAdd(&S.nemit, __popc(bal));
    wb = __shfl_sync(0xffffffffu, wb, 0);
    const int o = wb + __popc(bal & ((1u << lane) - 1));
    if (sel && o < K) {
        M.si[o] = i;
        M.list[o] = p;
        if (in_order) atomicOr(&M.bitmap[i >> 5], 1u << (i & 31));
    }
}

// Exact Top-K of a row from its candidate list (nc pairs (key, element << 32 | position), all keys
// in bins >= bstar; `above` keys lie above bstar). Keys above the cut bin are taken; inside it the
// second-level histogram hsub places the cut at bin s*: keys above s* are taken and the keys in s*
// are ranked exactly, pairwise, ties to the lower position. A list that overflowed kSelCand or more
// than kTie keys in s* are settled by radix select over all n keys g[0..n) instead.
// in_order (positions ascend with the element index): each selected element's output slot is the
// number of selected elements before it, read from a bitmap over the n elements; otherwise the
// positions are sorted. Ascending positions to out, padded with -1; returns the count.
__device__ int rank_row(const unsigned long long* ck, const unsigned long long* cip, int nc, int bstar, int above,
                        const unsigned int* hsub, const unsigned long long* g, int n, int K, PosMap pos,
                        bool in_order, int32_t* out, const SelSmem& M, SelScal& S) {
    const int tid = threadIdx.x, lane = tid & 31;
    if (nc > kSelCand) return radix_topk(n, K, g, pos, out, M, S);
    int above2 = 0;
    const int sstar = bstar >= 0 ? cut_bin(hsub, kSubBins, K - above, S, &above2) : -1;
    const int words = (n + 31) >> 5;
    if (in_order)
        for (int w = tid; w < words; w += kQThreads) M.bitmap[w] = 0u;
    if (tid == 0) { S.nemit = 0; S.ntie = 0; }
    __syncthreads();
    constexpr int kRU = 4;  // candidates per thread requested together
    for (int base0 = 0; base0 < nc; base0 += kQThreads * kRU) {
    unsigned long long kr[kRU], ir[kRU];
#pragma unroll
    for (int r = 0; r < kRU; ++r) {
        const int c = base0 + r * kQThreads + tid;
        kr[r] = c < nc ? __ldcg(ck + c) : 0ull;
        ir[r] = c < nc ? __ldcg(cip + c) : 0ull;
    }
#pragma unroll
    for (int r = 0; r < kRU; ++r) {
        const int c = base0 + r * kQThreads + tid;
        bool sel = false, tie = false;
        const unsigned long long k = kr[r], ip = ir[r];
        if (c < nc) {
            const int b = key_bin(k);
            if (bstar < 0 || b > bstar) {
                sel = true;
            } else if (b == bstar) {
                const int sb = sub_bin(k);
                sel = sstar < 0 || sb > sstar;
                tie = sstar >= 0 && sb == sstar;
            }
        }
        add_selected(sel, (int)(ip >> 32), (int)(unsigned int)ip, K, in_order, M, S);
        const unsigned int tb = __ballot_sync(0xffffffffu, tie);
        if (tb) {
            int wb = 0;
            if (lane == 0) wb = atomicAdd(&S.ntie, __popc(tb));
            wb = __shfl_sync(0xffffffffu, wb, 0);
            const int o = wb + __popc(tb & ((1u << lane) - 1));
            if (tie && o < kTie) { M.tk[o] = k; M.ti[o] = (int)(ip >> 32); M.tp[o] = (int)(unsigned int)ip; }
        }
    }
    }
    __syncthreads();
    const int m = S.ntie;
    if (m > kTie) return radix_topk(n, K, g, pos, out, M, S);
    const int need = K - above - above2;
    for (int base = 0; base < m; base += kQThreads) {
        const int t = base + tid;
        bool sel = false;
        if (t < m) {
            const unsigned long long kt = M.tk[t];
            const int pt = M.tp[t];
            int rank = 0;
            for (int f = 0; f < m; ++f) {
                const unsigned long long kf = M.tk[f];
                rank += (kf > kt) || (kf == kt && M.tp[f] < pt);
            }
            sel = rank < need;
        }
        add_selected(sel, t < m ? M.ti[t] : 0, t < m ? M.tp[t] : 0, K, in_order, M, S);
    }
    __syncthreads();
    const int cnt = S.nemit < K ? S.nemit : K;
    if (!in_order) {
        sort_asc(M.list, cnt);
        for (int i = tid; i < K; i += kQThreads) out[i] = i < cnt ? M.list[i] : -1;
        return cnt;
    }
    // slot of element i = selected elements in words before i's word + those below i in it
    const int per = (words + kQThreads - 1) / kQThreads;
    const int w0 = min(tid * per, words), w1 = min(w0 + per, words);
    int wc = 0;
    for (int w = w0; w < w1; ++w) wc += __popc(M.bitmap[w]);
    int total;
    int run = block_excl_scan(wc, S.wsum, total);
    for (int w = w0; w < w1; ++w) {
        M.wpre[w] = (unsigned short)run;
        run += __popc(M.bitmap[w]);
    }
    __syncthreads();
    for (int e = tid; e < cnt; e += kQThreads) {
        const int i = M.si[e];
        const int slot = M.wpre[i >> 5] + __popc(M.bitmap[i >> 5] & ((1u << (i & 31)) - 1u));
        out[slot] = M.list[e];
    }
    for (int i = cnt + tid; i < K; i += kQThreads) out[i] = -1;
    return cnt;
}

// Appends the flagged (key, element << 32 | position) pairs to the CTA's shared list (cap entries);
// a warp whose entries no longer fit appends the rest to the row's global list itself.
template <int N>
__device__ __forceinline__ void local_append(const bool (&take)[N], const unsigned long long (&key)[N],
                                             const unsigned long long (&ip)[N], int* nloc, unsigned long long* lk,
                                             unsigned long long* lip, unsigned int* gcounter,
                                             unsigned long long* gk, unsigned long long* gip) {
    const int lane = threadIdx.x & 31;
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < N; ++j) cnt += take[j];
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    const int wtotal = __shfl_sync(0xffffffffu, incl, 31);
    if (wtotal == 0) return;
    int base = 0;
    if (lane == 31) base = atomicAdd(nloc, wtotal);
    base = __shfl_sync(0xffffffffu, base, 31);
    const int spill = base + wtotal - kCtaCand;  // entries past the shared list
    int gbase = 0;
    if (spill > 0) {
        if (lane == 31) gbase = (int)atomicAdd(gcounter, (unsigned)min(spill, wtotal));
        gbase = __shfl_sync(0xffffffffu, gbase, 31);
    }
    int o = base + incl - cnt;
#pragma unroll
    for (int j = 0; j < N; ++j) {
        if (take[j]) {
            if (o < kCtaCand) {
                lk[o] = key[j];
                lip[o] = ip[j];
            } else {
                const int g = gbase + (o - max(base, kCtaCand));
                if (g < kSelCand) { gk[g] = key[j]; gip[g] = ip[j]; }
            }
            ++o;
        }
    }
}

// Moves the CTA's shared list to the row's global list with one atomic on the row's counter.
__device__ void flush_local(int nloc, const unsigned long long* lk, const unsigned long long* lip,
                            unsigned int* gcounter, unsigned long long* gk, unsigned long long* gip, SelScal& S) {
    const int n = min(nloc, kCtaCand);
    if (n == 0) return;
    if (threadIdx.x == 0) S.cnt = (int)atomicAdd(gcounter, (unsigned)n);
    __syncthreads();
    const int base = S.cnt;
    for (int j = threadIdx.x; j < n; j += kQThreads)
        if (base + j < kSelCand) { gk[base + j] = lk[j]; gip[base + j] = lip[j]; }
}

__global__ void __launch_bounds__(kQThreads, 8) select_kernel(IndexArgs a, int slices) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ SelScal S;
    const int row = blockIdx.x / slices, slice = blockIdx.x % slices;
    const int tid = threadIdx.x;
    wait_prior_grid();  // keys and histograms come from the score kernel
    const bool pool_on = a.plan.pool_blocks > 0 && !a.reindex;
    const int nmax = a.plan.units_max * kBS;
    const int bstride = (a.plan.units_max + 1) & ~1;
    const unsigned long long* gk = reinterpret_cast<const unsigned long long*>(a.ws + a.L.cand_key) + (size_t)row * nmax;
    const unsigned long long* gb = reinterpret_cast<const unsigned long long*>(a.ws + a.L.bmax) + (size_t)row * bstride;
    unsigned int* hrow = reinterpret_cast<unsigned int*>(a.ws + a.L.key_hist) + (size_t)row * kRowHist;
    unsigned int* hsub = hrow + 2 * kKeyBins;
    unsigned long long* ck = reinterpret_cast<unsigned long long*>(a.ws + a.L.sel_key) + (size_t)row * (2 * kSelCand);
    unsigned long long* cip = reinterpret_cast<unsigned long long*>(a.ws + a.L.sel_pos) + (size_t)row * (2 * kSelCand);
    // a row's counters sit on their own 128-byte line when the rows allow it
    RowCtr* rc = reinterpret_cast<RowCtr*>(a.ws + a.L.row_ctr) + (size_t)row * ctr_stride(a.plan.rows);
    unsigned int* pool_cnt = reinterpret_cast<unsigned int*>(&rc->tau);  // low word: pool candidates
    unsigned int* row_flags = pool_cnt + 1;                                // high word: 1 = pool out of order
    // the CTA's candidate lists (the ranking reuses this memory afterwards)
    unsigned long long* lk = reinterpret_cast<unsigned long long*>(smem);
    unsigned long long* lip = lk + kCtaCand;
    unsigned long long* plk = lip + kCtaCand;
    unsigned long long* plip = plk + kCtaCand;
    if (tid == 0) { S.nemit = 0; S.ntie = 0; }  // local list counts
    const int nbatch = (nmax + kBatch - 1) / kBatch;
    const int b0 = (int)((long long)nbatch * slice / slices), b1 = (int)((long long)nbatch * (slice + 1) / slices);
    // the first batch's keys are requested before anything else
    const int32_t* prow = a.reindex ? a.pool + (size_t)row * a.pool_stride : nullptr;
    // thread t of batch bt owns unit u = bt * kQThreads + t: its 8 keys (64 contiguous bytes), its
    // block maximum and its pool id
    unsigned long long kk[kPerT];
    int pid = 0, pid_next = 0;
    unsigned long long bmv = 0;
    auto load_unit = [&](int bt) {
        const int u = bt * kQThreads + tid;
        if (u < a.plan.units_max) {
            const uint4* src = reinterpret_cast<const uint4*>(gk + (size_t)u * kBS);
#pragma unroll
            for (int q = 0; q < kPerT / 2; ++q) {
                const uint4 v = __ldcg(src + q);
                kk[2 * q] = ((unsigned long long)v.y << 32) | v.x;
                kk[2 * q + 1] = ((unsigned long long)v.w << 32) | v.z;
            }
            pid = prow ? __ldg(prow + u) : u;
            pid_next = (prow && u + 1 < a.plan.units_max) ? __ldg(prow + u + 1) : 0x7FFFFFFF;
            bmv = pool_on ? __ldcg(gb + u) : 0ull;
        } else {
#pragma unroll
            for (int j = 0; j < kPerT; ++j) kk[j] = 0ull;
            pid = 0;
            pid_next = 0x7FFFFFFF;
            bmv = 0ull;
        }
    };
    if (b0 < b1) load_unit(b0);
    bool ok;
    const DRow R = drow(a, row, ok);
    const int n = R.n_units * kBS;
    const int K = a.plan.k, P = a.plan.pool_blocks;
    int above, pabove = 0, pstar = -1;
    const int bstar = cut_bin(hrow, kKeyBins, K, S, &above);  // its barriers order the resets above
    if (pool_on) pstar = cut_bin(hrow + kKeyBins, kKeyBins, P, S, &pabove);
    int unsorted = 0;
    for (int bt = b0; bt < b1; ++bt) {
        if (bt > b0) load_unit(bt);
        const int u = bt * kQThreads + tid;
        if (prow && u + 1 < R.n_units) unsorted |= pid >= pid_next;
        bool take[kPerT];
        unsigned long long ip[kPerT];
#pragma unroll
        for (int j = 0; j < kPerT; ++j) {
            const int i = u * kBS + j;
            const int b = kk[j] ? key_bin(kk[j]) : -2;
            take[j] = i < n && b >= bstar && b >= -1;
            const int p = pid * kBS + j;  // Full mode: pid == u
            ip[j] = ((unsigned long long)(unsigned int)i << 32) | (unsigned int)p;
            if (take[j] && b == bstar) atomicAdd(hsub + sub_bin(kk[j]), 1u);
        }
        local_append(take, kk, ip, &S.nemit, lk, lip, &rc->ncand, ck, cip);
        if (pool_on) {
            const int b = bmv ? key_bin(bmv) : -2;
            const bool pt[1] = {u < R.n_units && b >= pstar && b >= -1};
            if (pt[0] && b == pstar) atomicAdd(hsub + kSubBins + sub_bin(bmv), 1u);
            const unsigned long long pk[1] = {bmv};
            const unsigned long long pu[1] = {((unsigned long long)(unsigned int)u << 32) | (unsigned int)u};
            local_append(pt, pk, pu, &S.ntie, plk, plip, pool_cnt, ck + kSelCand, cip + kSelCand);
        }
    }
    if (__syncthreads_or(unsorted) && tid == 0) atomicOr(row_flags, 1u);
    const int nloc = S.nemit, ploc = S.ntie;
    flush_local(nloc, lk, lip, &rc->ncand, ck, cip, S);
    __syncthreads();
    if (pool_on) flush_local(ploc, plk, plip, pool_cnt, ck + kSelCand, cip + kSelCand, S);
    // 3. the last CTA of the row ranks its candidates
    __threadfence();
    __syncthreads();
    if (tid == 0) S.last = atomicAdd(&rc->ticket, 1u) == (unsigned)slices - 1;
    __syncthreads();
    if (!S.last) return;
    __threadfence();
    const int nc = (int)*reinterpret_cast<volatile unsigned int*>(&rc->ncand);
    const int pnc = (int)*reinterpret_cast<volatile unsigned int*>(pool_cnt);
    const bool pool_sorted = *reinterpret_cast<volatile unsigned int*>(row_flags) == 0u;
    const SelSmem M = sel_smem(smem, nmax);
    const bool fits = nmax <= kMapBits;  // the bitmap is sized for the longest row
    rank_row(ck, cip, nc, bstar, above, hsub, gk, n, K, PosMap{prow}, pool_sorted && fits,
             a.out_idx + (size_t)row * K, M, S);
    if (pool_on) {
        __syncthreads();
        const int cnt = rank_row(ck + kSelCand, cip + kSelCand, pnc, pstar, pabove, hsub + kSubBins, gb, R.n_units,
                                 P, PosMap{nullptr}, fits, a.out_pool + (size_t)row * P, M, S);
        if (tid == 0) a.out_pool_n[row] = cnt;
    }
    // leave the row's counters and histograms zeroed for the next call
    for (int j = tid; j < kRowHist; j += kQThreads) hrow[j] = 0u;
    if (tid == 0) { rc->ticket = 0; rc->ncand = 0; rc->tau = 0; }
}

__global__ void zero_kernel(uint4* p, size_t n16) {
    wait_prior_grid();  // the previous select may still read these histograms
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
        p[i] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace

cudaError_t launch_index_decode(const IndexArgs& a, cudaStream_t s) {
    const bool relu = (a.flags & CSA2_SCORE_RELU) != 0;
    const bool pool = a.plan.pool_blocks > 0 && !a.reindex;
    const void* fn = relu ? (pool ? (const void*)score_kernel<true, true> : (const void*)score_kernel<true, false>)
                          : (pool ? (const void*)score_kernel<false, true> : (const void*)score_kernel<false, false>);
    const size_t smem = (size_t)kSWarps * kWarpBytes;
    // the score histograms start from zero (kRowHist * 4 bytes per row: a multiple of 16)
    const size_t n16 = (size_t)a.plan.rows * kRowHist / 4;
    cudaError_t e = launch_after_prior(zero_kernel, dim3((unsigned)((n16 + 1023) / 1024 < 1184 ? (n16 + 1023) / 1024 : 1184)),
                                       dim3(256), 0, s, reinterpret_cast<uint4*>(a.ws + a.L.key_hist), n16);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kSThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    // one warp per step at most; otherwise every resident warp gets an equal share of the steps
    const long long steps = (long long)a.plan.rows * ((a.plan.units_max + kUnitsPerStep - 1) / kUnitsPerStep);
    long long grid = (long long)sms * per_sm;
    const long long need = (steps + kSWarps - 1) / kSWarps;
    if (grid > need) grid = need;
    if (grid < 1) grid = 1;
    void (*sk)(IndexArgs) = relu ? (pool ? score_kernel<true, true> : score_kernel<true, false>)
                                 : (pool ? score_kernel<false, true> : score_kernel<false, false>);
    e = launch_after_prior(sk, dim3((unsigned)grid), dim3(kSThreads), smem, s, a);
    if (e != cudaSuccess) return e;
    const size_t qsmem = sel_smem_bytes(a.plan.units_max * kBS);
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qsmem);
    if (e != cudaSuccess) return e;
    // as many slices per row as one wave of resident CTAs allows (at most one batch each)
    int qper = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&qper, select_kernel, kQThreads, qsmem);
    if (e != cudaSuccess) return e;
    const int nbatch = (a.plan.units_max * kBS + kBatch - 1) / kBatch;
    long long slices = (long long)sms * (qper > 0 ? qper : 1) / a.plan.rows;
    if (slices > nbatch) slices = nbatch;
    if (slices < 1) slices = 1;
    return launch_after_prior(select_kernel, dim3((unsigned)((long long)a.plan.rows * slices)), dim3(kQThreads), qsmem,
                              s, a, (int)slices);
}

}  // namespace csa2
