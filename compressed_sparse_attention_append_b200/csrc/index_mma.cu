// index_mma.cu -- indexer scores on the tensor cores for several query rows per sequence (a prefill
// chunk, where row i sees positions <= i; the draft tokens of multi-token decode): tcgen05
// block-scaled FP4 MMA (kind::mxf4nvf4, one E4M3 scale per 16 channels, fp32 accumulation) of
// 128-position key tiles against tiles of 16 or 256 query rows, each key tile read once per query
// tile.
//
// [B] "DeepSeek Cuts KV Cache Footprint Fourfold", "Technical Approach": Full mode ranks every
// position. [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token", sec. IX
// (the indexer scores every visible position), sec. XI (indexer queries and keys in FP4 with one
// E4M3 scale per 16 channels).
//
// The selection stays exact. The MMA gives approximate scores S^ with |S^ - S| <= eps_i for every
// position (S the exact score; eps_i from a bound on the accumulation error, below), and:
//   1. a sampled pass (this file): for about one key tile in 32, the largest S^ of each query row
//      over the tile; a row's admission estimate tau_i is the R-th largest of its sampled maxima,
//      R chosen so that about kMmaTarget positions of the row lie above it;
//   2. the full pass (this file): every visible position with S^ >= tau_i - 2 eps_i joins the row's
//      candidate list (at most kMmaCap);
//   3. per row (index.cu): if at least k candidates have S^ >= tau_i, every true Top-k position is
//      a candidate (k positions score >= tau_i - eps_i exactly, so the k-th best exact score does
//      too, and a position scoring that well has S^ >= tau_i - 2 eps_i); with A the k-th largest
//      S^ among the candidates, the Top-k lies in {S^ >= A - 2 eps_i}, which is rescored with the
//      exact integer arithmetic of index.cu and ranked exactly. A row whose list overflowed, held
//      fewer than k positions above tau_i, or showed a rescored |S^ - S| > eps_i is handed to the
//      exact CUDA-core scan of index.cu.
// Error bound: the MMA's products of E2M1 codes and E4M3 scales are exact in fp32; only the
// accumulation rounds. eps_i = 2^-14 * 576 * sum_b s_q[i,b] * max_p s_k[p,b] bounds 2^-14 times the
// sum of |terms| (576 = 16 channels x 6 x 6), far above the rounding of fp32 accumulation of 256
// terms (about 2^-23 of that sum, as measured).
//
// Kernel roles (one CTA of 14 warps per SM with 256 query columns, two of 10 with 16): warp 0 issues
// the TMA copies of key tiles (codes through a 128-byte-swizzled tensor map, scales by a bulk copy)
// into a ring of 4 stages (3 with 16 queries); warp 1 turns the scales into tensor-core scale-factor matrices
// (tcgen05.cp, replicated over the four lane quadrants) and issues the MMAs into tensor-memory
// accumulator slots; the other warps, in sets of four (one per lane quadrant) taking the slots in
// turn, read the accumulators (tcgen05.ld) and either admit candidates or reduce tile maxima. A
// candidate goes to the list its row keeps for this work item, counted in shared memory: each
// (row, item) list has one writer CTA, so no global atomics are needed. Every wait is bounded: one
// that runs out sets CSA2_DEV_TIMEOUT, and the CTA winds down (the producer waits for its copies in
// flight and the MMA warp for its MMAs, with the same bound) and frees its tensor memory.
#include <mutex>

#include "csa2_internal.cuh"
#include "tc.cuh"

namespace csa2 {

namespace {

using namespace tc;

constexpr int kTP = kMmaTile;                  // key positions per tile (MMA M)
constexpr int kCodeB = kTP * kIKBytes;         // 16384
constexpr int kScB = kTP * kIKScales;          // 2048
constexpr int kStageB = kCodeB + 2 * kScB;     // codes | raw scales | scale-factor matrices
constexpr uint64_t kWaitNs = 200000000ull;     // bound of one pipeline wait
constexpr float kEpsRel = 1.0f / 16384.0f;     // 2^-14

template <int NQ>
struct Cfg {
    static constexpr int ST = NQ > 128 ? 4 : 3;     // key tile stages (two 16-query CTAs share an SM)
    static constexpr int W = NQ > 128 ? 128 : NQ;   // MMA N
    static constexpr int H = NQ / W;                // MMAs per K step
    static constexpr int TPS = NQ > 128 ? 1 : 4;    // key tiles per accumulator slot (W columns each)
    static constexpr int SW = W * TPS;              // slot width in columns
    static constexpr int NSLOT = NQ > 128 ? 3 : 2;  // accumulator slots
    static constexpr int SETS = NQ > 128 ? 3 : 2;   // sets of four accumulator-reading warps (one per
                                                    // lane quadrant); set u % SETS reads slot use u
    static constexpr int EPI = 4 * SETS;
    static constexpr int THREADS = 32 * (2 + EPI);
    static constexpr int SFA = NSLOT * SW;          // key scale factors: 16 columns per stage
    static constexpr int SFB = SFA + 16 * ST;      // query scale factors: 16 columns per half
    static constexpr int COLS = SFB + 16 * H <= 256 ? 256 : 512;
    static constexpr int BQ = NQ * kIKBytes;        // query tile bytes
    static constexpr int CH = W < 32 ? W : 32;      // accumulator columns per tcgen05.ld
    static constexpr int HS = (TPS > 1 ? 32 : CH) + 4;  // floats per lane of a warp's hit staging row
                                                        // (one 32-column load; padded against bank
                                                        // conflicts of its 16-byte stores)
    static constexpr size_t SMEM = 1024 + BQ + (size_t)ST * kStageB + (size_t)NQ * 12 + 128 + (NQ < 32 ? 64 : NQ * 2) +
                                   (size_t)EPI * 32 * HS * 4 + 8 * (2 * ST + 2 * NSLOT + 2);
};

template <int EPI>
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * EPI) : "memory"); }

// tcgen05.cp of a 32-row x 16-byte matrix (rows 16 bytes apart in shared memory) into 32 lanes x 4
// columns of tensor memory, replicated to the four lane quadrants.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint32_t saddr) {
    const uint64_t desc = (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) |
                          ((uint64_t)(128u >> 4) << 32) | (1ull << 46);
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

// Tiles of work item `it`: sequence b, query tile j, first tile (or first sample) t0, count nt.
template <bool SAMPLE>
__device__ __forceinline__ void item_range(const IndexArgs& a, const uint32_t* tend, int it, int& b, int& j, int& t0,
                                           int& nt) {
    const MmaPlan& P = a.plan.mma;
    const int nch = SAMPLE ? P.nschunks : P.nchunks;
    j = it % P.nqt;
    const int r = it / P.nqt;
    const int c = r % nch;
    b = r / nch;
    const int te = (int)tend[b * P.nqt + j];
    if (!SAMPLE) {
        t0 = c * P.kc;
        nt = min(P.kc, te - t0);
    } else {
        t0 = c * P.sc;
        const int e = min(P.ns, t0 + P.sc);
        nt = 0;
        for (int s = t0; s < e; ++s) nt += mma_sample_tile(P.st, s) < te;  // a prefix: tiles grow with s
    }
    if (nt < 0) nt = 0;
}

// Max over the warp's lanes of x[lane % N], left in x[0] of every lane (reduce-scatter).
template <int N>
__device__ __forceinline__ float lane_col_max(float (&x)[N]) {
    const int lane = threadIdx.x & 31;
    if (N == 16) {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = fmaxf(x[i], __shfl_xor_sync(0xffffffffu, x[i], 16));
    }
#pragma unroll
    for (int w = N / 2; w >= 1; w >>= 1) {
        const bool up = (lane & w) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float keep = up ? x[i + w] : x[i], send = up ? x[i] : x[i + w];
            x[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, w));
        }
    }
    return x[0];
}

template <int CH>
__device__ __forceinline__ void tmem_ld_ch(uint32_t taddr, uint32_t (&r)[CH]);
template <>
__device__ __forceinline__ void tmem_ld_ch<32>(uint32_t taddr, uint32_t (&r)[32]) { tmem_ld32(taddr, r); }
template <>
__device__ __forceinline__ void tmem_ld_ch<16>(uint32_t taddr, uint32_t (&r)[16]) { tmem_ld16(taddr, r); }

template <int NQ, bool SAMPLE>
__global__ void __launch_bounds__(Cfg<NQ>::THREADS, Cfg<NQ>::COLS <= 256 ? 2 : 1) mma_score_kernel(const IndexArgs a, const __grid_constant__ CUtensorMap tmap) {
    using G = Cfg<NQ>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    // 1024-byte aligned by offsetting the shared array itself (not through an integer), so that the
    // compiler keeps every access below in the shared state space
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    unsigned char* bq = sm;
    unsigned char* stg = sm + G::BQ;
    float* thr_s = reinterpret_cast<float*>(stg + G::ST * kStageB);
    int* ql_s = reinterpret_cast<int*>(thr_s + NQ);
    unsigned int* cnt_s = reinterpret_cast<unsigned int*>(ql_s + NQ);
    float* thr2 = reinterpret_cast<float*>(cnt_s + NQ);     // 32 columns: thresholds of column % NQ
    // thresholds rounded down to fp16, paired for the packed test: entry 16 g + p of a 32-column
    // load holds columns 32 g + p and 32 g + p + 16
    __half2* thh = reinterpret_cast<__half2*>(thr2 + 32);
    float* hstage = reinterpret_cast<float*>(thh + (NQ < 32 ? 16 : NQ / 2));  // [EPI warps][32 lanes][HS]
    uint64_t* full = reinterpret_cast<uint64_t*>(hstage + G::EPI * 32 * G::HS);
    uint64_t* empty = full + G::ST;
    uint64_t* dfull = empty + G::ST;
    uint64_t* dfree = dfull + G::NSLOT;
    uint64_t* qready = dfree + G::NSLOT;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(qready + 1);
    __shared__ volatile int abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const MmaPlan& P = a.plan.mma;
    uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + kHdrStatus);
    const uint32_t* tend = reinterpret_cast<const uint32_t*>(a.ws + a.L.mma_tend);
    if (tid == 0) {
        for (int s = 0; s < G::ST; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int k = 0; k < G::NSLOT; ++k) { mbar_init(&dfull[k], 1); mbar_init(&dfree[k], 4); }
        mbar_init(qready, 1);
        abort_s = 0;
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(tslot, G::COLS);
    if (tid == 0) prefetch_tmap(&tmap);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    const int nitems = P.nseq * P.nqt * (SAMPLE ? P.nschunks : P.nchunks);
    auto fail = [&]() {
        set_status(status, CSA2_DEV_TIMEOUT);
        abort_s = 1;
    };

    if (warp == 0) {
        // ---- TMA producer ----
        if (lane == 0) {
            int kk = 0;
            for (int it = blockIdx.x; it < nitems && !abort_s; it += gridDim.x) {
                int b, j, t0, nt;
                item_range<SAMPLE>(a, tend, it, b, j, t0, nt);
                for (int k = 0; k < nt; ++k, ++kk) {
                    const int s = kk % G::ST;
                    const uint32_t ph = (uint32_t)(kk / G::ST) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, kWaitNs)) { fail(); break; }
                    const int t = SAMPLE ? mma_sample_tile(P.st, t0 + k) : t0 + k;
                    const int64_t p0 = (int64_t)t * kTP;
                    const int64_t left = a.c.cap - p0;
                    const int nvalid = left < kTP ? (int)left : kTP;
                    unsigned char* st = stg + s * kStageB;
                    mbar_expect_tx(&full[s], (uint32_t)(kCodeB + nvalid * kIKScales));
                    tma_3d_g2s(st, &tmap, 0, (int)p0, b, &full[s]);
                    bulk_g2s(st + kCodeB, a.c.ik_scale + ((size_t)b * a.c.cap + p0) * kIKScales,
                             (uint32_t)(nvalid * kIKScales), &full[s]);
                }
            }
            // wait for the copies still in flight (all landed already unless a wait ran out)
            for (int s = 0; s < G::ST && s < kk; ++s) {
                const int n = (kk - s + G::ST - 1) / G::ST;
                if (!mbar_wait(&full[s], (uint32_t)(n - 1) & 1u, kWaitNs)) set_status(status, CSA2_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ---- scale factors and MMA issue ----
        const uint32_t idesc = mxf4_idesc(kTP, G::W);
        int kk = 0, u = 0, itn = 0, last_s = -1;
        uint32_t last_ph = 0;
        for (int it = blockIdx.x; it < nitems && !abort_s; it += gridDim.x) {
            int b, j, t0, nt;
            item_range<SAMPLE>(a, tend, it, b, j, t0, nt);
            if (nt == 0) continue;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(qready, (uint32_t)itn & 1u, kWaitNs);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            ++itn;
            if (!ok) { if (lane == 0) fail(); break; }
            tc_fence_after();
            for (int k = 0; k < nt; ++k, ++kk) {
                const int s = kk % G::ST;
                const uint32_t ph = (uint32_t)(kk / G::ST) & 1u;
                ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph, kWaitNs));
                if (!ok) { if (lane == 0) fail(); break; }
                unsigned char* st = stg + s * kStageB;
                // scale-factor matrix of K step j: row l = scale word j of key rows l, l+32, l+64, l+96
                const uint4* raw = reinterpret_cast<const uint4*>(st + kCodeB);
                uint4* sf = reinterpret_cast<uint4*>(st + kCodeB + kScB);
                const uint4 r0 = raw[lane], r1 = raw[lane + 32], r2 = raw[lane + 64], r3 = raw[lane + 96];
                sf[lane] = make_uint4(r0.x, r1.x, r2.x, r3.x);
                sf[32 + lane] = make_uint4(r0.y, r1.y, r2.y, r3.y);
                sf[64 + lane] = make_uint4(r0.z, r1.z, r2.z, r3.z);
                sf[96 + lane] = make_uint4(r0.w, r1.w, r2.w, r3.w);
                fence_async_smem();
                __syncwarp();
                const uint32_t sfa = tbase + (uint32_t)(G::SFA + 16 * s);
                if (lane == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int q = 0; q < 4; ++q) tmem_cp_sf(sfa + 4 * q, smem_u32(sf) + 512 * q);
                }
                // slot use u takes the H halves of one tile (256 queries) or TPS consecutive tiles of
                // an item (16 queries: tile k % TPS at column W * (k % TPS) of the slot)
                const int sub = G::TPS > 1 ? k % G::TPS : 0;
                const bool close = G::TPS == 1 || sub == G::TPS - 1 || k == nt - 1;
                for (int h = 0; h < G::H; ++h) {
                    const int slot = u % G::NSLOT;
                    const uint32_t uph = (uint32_t)(u / G::NSLOT) & 1u;
                    if (sub == 0) {
                        if (lane == 0) ok = mbar_wait(&dfree[slot], uph ^ 1u, kWaitNs);
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                    }
                    if (lane == 0) {
                        tc_fence_after();
                        const uint32_t d = tbase + (uint32_t)(slot * G::SW + sub * G::W);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint64_t ad = sw128_desc(smem_u32(st) + 32 * q);
                            const uint64_t bd = sw128_desc(smem_u32(bq + h * G::W * kIKBytes) + 32 * q);
                            mma_mxf4(d, ad, bd, idesc, sfa + 4 * q, tbase + (uint32_t)(G::SFB + 16 * h + 4 * q), q > 0);
                        }
                        if (close) mma_commit(&dfull[slot]);
                    }
                    if (close) ++u;
                }
                if (lane == 0) mma_commit(&empty[s]);
                last_s = s;
                last_ph = ph;
                if (!ok) { if (lane == 0) fail(); break; }
            }
            if (!ok) break;
        }
        // every MMA issued has completed before the tensor memory is freed
        if (lane == 0 && last_s >= 0 && !mbar_wait(&empty[last_s], last_ph, kWaitNs))
            set_status(status, CSA2_DEV_TIMEOUT);
        __syncwarp();
    } else {
        // ---- accumulator readers ----
        const int ew = warp - 2;
        const int set = ew >> 2;                 // set u % SETS reads slot use u
        const int quad = warp & 3;               // the lane quadrant this warp may access
        const int et = tid - 64;                 // 0..255
        const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
        const int sub = P.subcap;
        uint32_t* cnt = reinterpret_cast<uint32_t*>(a.ws + a.L.mma_cnt);
        int32_t* cpos = reinterpret_cast<int32_t*>(a.ws + a.L.mma_cpos);
        float* cval = reinterpret_cast<float*>(a.ws + a.L.mma_cval);
        uint32_t* tm = reinterpret_cast<uint32_t*>(a.ws + a.L.mma_tm);
        const uint8_t* qc = a.ws + a.L.mma_qc;
        const uint8_t* qs = a.ws + a.L.mma_qs;
        const float4* rowp = reinterpret_cast<const float4*>(a.ws + a.L.mma_row);
        int u = 0;
        // every item is visited even after a wait ran out (its tiles are then skipped), so that the
        // eight warps pass the same named barriers
        for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
            int b, j, t0, nt;
            item_range<SAMPLE>(a, tend, it, b, j, t0, nt);
            if (nt == 0) continue;
            const int tq = a.tq;
            const int rbase = b * tq + j * NQ;
            const int nrow = min(NQ, tq - j * NQ);
            const int chunk = SAMPLE ? 0 : t0 / P.kc;
            // the previous item's accumulators are all read (so its MMAs are done) before the query
            // tile and its scale factors are replaced
            epi_sync<G::EPI>();
            for (int e = et; e < NQ * 8; e += 32 * G::EPI) {
                const int r = e >> 3, c = e & 7;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (r < nrow) v = *reinterpret_cast<const uint4*>(qc + (size_t)(rbase + r) * kIKBytes + 16 * c);
                *reinterpret_cast<uint4*>(bq + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) = v;
            }
            for (int e = et; e < NQ; e += 32 * G::EPI) {
                int ql = -1;
                float th = __int_as_float(0x7f800000);
                if (e < nrow) {
                    const int64_t q = index_row_last(a, rbase + e);
                    ql = q < 0 ? -1 : (int)q;
                    if (!SAMPLE && ql >= 0) th = rowp[rbase + e].z;
                }
                ql_s[e] = ql;
                thr_s[e] = th;
                cnt_s[e] = 0;
            }
            if (G::TPS > 1 && !SAMPLE) {  // a 32-column load spans 32 / NQ tiles of the same queries
                for (int e = et; e < 32; e += 32 * G::EPI) {
                    const int c = e % NQ;
                    float th = __int_as_float(0x7f800000);
                    if (c < nrow && index_row_last(a, rbase + c) >= 0) th = rowp[rbase + c].z;
                    thr2[e] = th;
                }
            }
            if (!SAMPLE) {
                constexpr int NP = NQ < 32 ? 16 : NQ / 2;
                for (int e = et; e < NP; e += 32 * G::EPI) {
                    const int g = e >> 4, pp = e & 15;
                    const int c0 = (32 * g + pp) % NQ, c1 = (32 * g + pp + 16) % NQ;
                    float t0 = __int_as_float(0x7f800000), t1 = t0;
                    if (c0 < nrow && index_row_last(a, rbase + c0) >= 0) t0 = rowp[rbase + c0].z;
                    if (c1 < nrow && index_row_last(a, rbase + c1) >= 0) t1 = rowp[rbase + c1].z;
                    thh[e] = __halves2half2(__float2half_rd(t0), __float2half_rd(t1));
                }
            }
            if (set < G::H) {
                // query scale factors of half `set`: column 4q + g, lane l <- scale word q of row l + 32 g
                uint32_t w[16];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int r = set * G::W + lane + 32 * g;
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (r < G::W * (set + 1) && r < nrow)
                        v = *reinterpret_cast<const uint4*>(qs + (size_t)(rbase + r) * kIKScales);
                    w[g] = v.x; w[4 + g] = v.y; w[8 + g] = v.z; w[12 + g] = v.w;
                }
                tmem_st16(tbase + lane_off + (uint32_t)(G::SFB + 16 * set), w);
                tmem_st_wait();
            }
            fence_async_smem();
            tc_fence_before();
            epi_sync<G::EPI>();
            if (et == 0) mbar_arrive(qready);
            for (int k = 0; k < nt && !abort_s; k += G::TPS) {
                const int t = SAMPLE ? mma_sample_tile(P.st, t0 + k) : t0 + k;
                const int p = t * kTP + 32 * quad + lane;
                const int ng = min(G::TPS, nt - k);  // tiles in this slot use
                for (int h = 0; h < G::H; ++h, ++u) {
                    if (u % G::SETS != set) continue;
                    const int slot = u % G::NSLOT;
                    const uint32_t ph = (uint32_t)(u / G::NSLOT) & 1u;
                    const bool ok = __all_sync(0xffffffffu, mbar_wait(&dfull[slot], ph, kWaitNs));
                    if (!ok) { if (lane == 0) fail(); break; }
                    tc_fence_after();
                    // sampling: the column maxima of one chunk of CH accumulator columns (queries)
                    auto sample = [&](const uint32_t (&v)[G::CH], int colb) {
                        float x[G::CH];
#pragma unroll
                        for (int i = 0; i < G::CH; ++i)
                            x[i] = p <= ql_s[colb + i] ? __uint_as_float(v[i]) : -__int_as_float(0x7f800000);
                        const float m = lane_col_max<G::CH>(x);
                        const int col = colb + (lane % G::CH);
                        if (lane < G::CH && ql_s[col] >= 0)
                            atomicMax(&tm[(size_t)(rbase + col) * P.ns + (t0 + k)], f32_order(m));
                    };
                    // filtering: this thread's columns at or above their thresholds, as a bit mask
                    // (independent 4-bit groups, then an OR tree: no serial dependency chain)
                    // A superset test in fp16: values p and p + 16 of a 32-column load are packed and
                    // compared with thresholds rounded down (a value at or above its fp32 threshold
                    // rounds to at least the rounded-down threshold); admitted values are checked
                    // again exactly. Four independent partial masks.
                    auto packed_mask = [&](const uint32_t (&v)[32], const __half2* th) -> uint32_t {
                        uint32_t mk[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                        for (int pp = 0; pp < 16; ++pp) {
                            const __half2 hv = __floats2half2_rn(__uint_as_float(v[pp]), __uint_as_float(v[pp + 16]));
                            mk[pp & 3] |= __hge2_mask(hv, th[pp]) & (0x00010001u << pp);
                        }
                        return (mk[0] | mk[1]) | (mk[2] | mk[3]);
                    };
                    auto hitmask = [&](const uint32_t (&v)[G::CH], int colb) -> uint32_t {
                        if constexpr (G::CH == 32) return packed_mask(v, thh + (colb >> 5) * 16);
                        const float4* t4 = reinterpret_cast<const float4*>(thr_s + colb);
                        uint32_t mk[G::CH / 4];
#pragma unroll
                        for (int i4 = 0; i4 < G::CH / 4; ++i4) {
                            const float4 tt = t4[i4];
                            const uint32_t g = (__uint_as_float(v[4 * i4 + 0]) >= tt.x ? 1u : 0u) |
                                               (__uint_as_float(v[4 * i4 + 1]) >= tt.y ? 2u : 0u) |
                                               (__uint_as_float(v[4 * i4 + 2]) >= tt.z ? 4u : 0u) |
                                               (__uint_as_float(v[4 * i4 + 3]) >= tt.w ? 8u : 0u);
                            mk[i4] = g << (4 * i4);
                        }
#pragma unroll
                        for (int w = G::CH / 8; w >= 1; w >>= 1)
#pragma unroll
                            for (int i = 0; i < w; ++i) mk[i] |= mk[i + w];
                        return mk[0];
                    };
                    auto hitmask2 = [&](const uint32_t (&v)[32]) -> uint32_t { return packed_mask(v, thh); };
                    // the admitted positions of one chunk go to their rows' lists of this item
                    auto admit = [&](const uint32_t (&v)[G::CH], int colb, uint32_t m) {
                        if (!m) return;
                        // the values go through this lane's staging row, read back by index
                        float* hs = hstage + ((size_t)ew * 32 + lane) * G::HS;
#pragma unroll
                        for (int i4 = 0; i4 < G::CH / 4; ++i4)
                            *reinterpret_cast<float4*>(hs + 4 * i4) =
                                make_float4(__uint_as_float(v[4 * i4]), __uint_as_float(v[4 * i4 + 1]),
                                            __uint_as_float(v[4 * i4 + 2]), __uint_as_float(v[4 * i4 + 3]));
                        do {
                            const int i = __ffs(m) - 1;
                            m &= m - 1;
                            const int col = colb + i;
                            if (p > ql_s[col] || !(hs[i] >= thr_s[col])) continue;
                            // this CTA alone fills the row's list of this item: a shared counter
                            const unsigned int o = atomicAdd(&cnt_s[col], 1u);
                            if (o < (unsigned)sub) {
                                const size_t off = ((size_t)(rbase + col) * P.nchunks + chunk) * sub + o;
                                cpos[off] = p;
                                cval[off] = hs[i];
                            }
                        } while (m);
                    };
                    const uint32_t dcol = tbase + lane_off + (uint32_t)(slot * G::SW);
                    if (G::TPS > 1) {
                        // TPS tiles of W = 16 queries: column c <-> tile k + c / 16, query c % 16
                        static_assert(G::TPS == 1 || (G::W == 16 && G::TPS == 4), "grouped slots: 4 tiles x 16");
                        uint32_t v0[32], v1[32];
                        tmem_ld32(dcol, v0);
                        tmem_ld32(dcol + 32u, v1);
                        tmem_ld_wait();
                        // key position of this thread in tile k + sb
                        auto pos_of = [&](int sb) {
                            const int tt = SAMPLE ? mma_sample_tile(P.st, t0 + k + sb) : t0 + k + sb;
                            return tt * kTP + 32 * quad + lane;
                        };
                        auto grouped = [&](const uint32_t (&v)[32], int c) {  // tiles 2c, 2c + 1
                            const int pa = pos_of(2 * c), pb = pos_of(2 * c + 1);
                            const bool va = 2 * c < ng, vb = 2 * c + 1 < ng;
                            if (SAMPLE) {
                                float x[32];
#pragma unroll
                                for (int i = 0; i < 32; ++i) {
                                    const bool ok2 = i < 16 ? (va && pa <= ql_s[i & 15]) : (vb && pb <= ql_s[i & 15]);
                                    x[i] = ok2 ? __uint_as_float(v[i]) : -__int_as_float(0x7f800000);
                                }
                                const float m = lane_col_max<32>(x);
                                const int q = lane & 15, sb = 2 * c + (lane >> 4);
                                if (sb < ng && ql_s[q] >= 0)
                                    atomicMax(&tm[(size_t)(rbase + q) * P.ns + (t0 + k + sb)], f32_order(m));
                            } else {
                                uint32_t m = hitmask2(v);
                                m &= (va ? 0x0000FFFFu : 0u) | (vb ? 0xFFFF0000u : 0u);
                                if (!m) return;
                                float* hs = hstage + ((size_t)ew * 32 + lane) * G::HS;
#pragma unroll
                                for (int i4 = 0; i4 < 8; ++i4)
                                    *reinterpret_cast<float4*>(hs + 4 * i4) =
                                        make_float4(__uint_as_float(v[4 * i4]), __uint_as_float(v[4 * i4 + 1]),
                                                    __uint_as_float(v[4 * i4 + 2]), __uint_as_float(v[4 * i4 + 3]));
                                do {
                                    const int i = __ffs(m) - 1;
                                    m &= m - 1;
                                    const int q = i & 15;
                                    const int pp = i < 16 ? pa : pb;
                                    if (pp > ql_s[q] || !(hs[i] >= thr2[i])) continue;
                                    const unsigned int o = atomicAdd(&cnt_s[q], 1u);
                                    if (o < (unsigned)sub) {
                                        const size_t off = ((size_t)(rbase + q) * P.nchunks + chunk) * sub + o;
                                        cpos[off] = pp;
                                        cval[off] = hs[i];
                                    }
                                } while (m);
                            }
                        };
                        grouped(v0, 0);
                        if (ng > 2) grouped(v1, 1);
                    } else if (G::W >= 2 * G::CH) {
#pragma unroll 1
                        for (int c0 = 0; c0 < G::W; c0 += 2 * G::CH) {
                            uint32_t v0[G::CH], v1[G::CH];
                            tmem_ld_ch<G::CH>(dcol + (uint32_t)c0, v0);
                            tmem_ld_ch<G::CH>(dcol + (uint32_t)(c0 + G::CH), v1);
                            tmem_ld_wait();
                            const int cb = h * G::W + c0;
                            if (SAMPLE) {
                                sample(v0, cb);
                                sample(v1, cb + G::CH);
                            } else {
                                const uint32_t m0 = hitmask(v0, cb), m1 = hitmask(v1, cb + G::CH);
                                admit(v0, cb, m0);
                                admit(v1, cb + G::CH, m1);
                            }
                        }
                    } else {
                        uint32_t v0[G::CH];
                        tmem_ld_ch<G::CH>(dcol, v0);
                        tmem_ld_wait();
                        if (SAMPLE) sample(v0, h * G::W);
                        else admit(v0, h * G::W, hitmask(v0, h * G::W));
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&dfree[slot]);
                }
            }
            if (!SAMPLE) {
                // the item's candidate counts (a count above subcap marks an overflowed list)
                epi_sync<G::EPI>();
                for (int e = et; e < nrow; e += 32 * G::EPI) cnt[(size_t)(rbase + e) * P.nchunks + chunk] = cnt_s[e];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, G::COLS);
}

// Query quantisation (the cache codec), the key tiles each query tile sees, and the largest key
// scale of every 16-channel block of each sequence.
__global__ void __launch_bounds__(256) mma_prep_kernel(const IndexArgs a, int qblocks, int sblocks) {
    const MmaPlan& P = a.plan.mma;
    const int tid = threadIdx.x;
    if ((int)blockIdx.x < qblocks) {
        const int row = blockIdx.x * 16 + (tid >> 4), blk = tid & 15;
        if (row >= a.rows) return;
        float x[16];
        load16_bf16(a.idx_q + (size_t)row * (kHI * kDI) + 16 * blk, x);
        uint2 codes;
        uint8_t sc;
        quantize_block(x, codes, sc);
        *reinterpret_cast<uint2*>(a.ws + a.L.mma_qc + (size_t)row * kIKBytes + 8 * blk) = codes;
        a.ws[a.L.mma_qs + (size_t)row * kIKScales + blk] = sc;
        if (blk == 0) {
            const int64_t q = index_row_last(a, row);
            if (q >= 0) {
                const int b = row / a.tq, j = (row % a.tq) / P.nq;
                atomicMax(reinterpret_cast<uint32_t*>(a.ws + a.L.mma_tend) + b * P.nqt + j,
                          (uint32_t)(q / kTP + 1));
            }
        }
        return;
    }
    __shared__ uint32_t red[8][4];
    const int sb = blockIdx.x - qblocks;
    const int b = sb / sblocks, part = sb % sblocks;
    int64_t n = (int64_t)P.nt * kTP;
    if (n > a.c.cap) n = a.c.cap;
    const uint4* sc = reinterpret_cast<const uint4*>(a.c.ik_scale + (size_t)b * a.c.cap * kIKScales);
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
#pragma unroll 4
    for (int64_t p = (int64_t)part * 256 + tid; p < n; p += (int64_t)sblocks * 256) {
        const uint4 v = __ldg(sc + p);
        m0 = __vmaxu4(m0, v.x & 0x7F7F7F7Fu);
        m1 = __vmaxu4(m1, v.y & 0x7F7F7F7Fu);
        m2 = __vmaxu4(m2, v.z & 0x7F7F7F7Fu);
        m3 = __vmaxu4(m3, v.w & 0x7F7F7F7Fu);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        m0 = __vmaxu4(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = __vmaxu4(m1, __shfl_xor_sync(0xffffffffu, m1, o));
        m2 = __vmaxu4(m2, __shfl_xor_sync(0xffffffffu, m2, o));
        m3 = __vmaxu4(m3, __shfl_xor_sync(0xffffffffu, m3, o));
    }
    if ((tid & 31) == 0) { red[tid >> 5][0] = m0; red[tid >> 5][1] = m1; red[tid >> 5][2] = m2; red[tid >> 5][3] = m3; }
    __syncthreads();
    if (tid < 16) {
        uint32_t m = 0;
        for (int w = 0; w < 8; ++w) m = __vmaxu4(m, red[w][tid >> 2]);
        atomicMax(reinterpret_cast<uint32_t*>(a.ws + a.L.mma_smax) + b * 16 + tid, (m >> (8 * (tid & 3))) & 0xFFu);
    }
}

// Per row: the error bound eps, the threshold estimate tau (R-th largest sampled tile maximum) and
// the admission threshold tau - 2 eps (rounded down); -inf admits every visible position when they
// fit the candidate list. One warp per row.
__global__ void __launch_bounds__(256) mma_tau_kernel(const IndexArgs a) {
    const MmaPlan& P = a.plan.mma;
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= a.rows) return;
    const int b = row / a.tq;
    const int64_t ql = index_row_last(a, row);
    float4 out = make_float4(0.f, 0.f, __int_as_float(0x7f800000), 0.f);
    double e = 0.0;
    if (lane < 16) {
        const double sq = (double)e4m3_to_f32(a.ws[a.L.mma_qs + (size_t)row * kIKScales + lane]);
        const uint32_t mb = reinterpret_cast<const uint32_t*>(a.ws + a.L.mma_smax)[b * 16 + lane];
        e = sq * (double)e4m3_to_f32((uint8_t)mb);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
    const double eps = e * 576.0 * (double)kEpsRel;
    if (ql >= kMmaCap) {  // rows seeing at most kMmaCap positions are rescored whole, unfiltered
        const int64_t n = ql + 1;
        out.y = __double2float_ru(eps);
        {
            // samples whose tile starts at or before the row's last visible position (a prefix)
            const int tl = (int)(ql / kTP);
            int s1 = tl / P.st;
            if (mma_sample_tile(P.st, s1) > tl) --s1;
            const int ns_i = min(P.ns, s1 + 1);
            const float f = 1.f - expf(128.f * log1pf(-(float)kMmaTarget / (float)n));
            int R = (int)ceilf(f * (float)ns_i);
            R = R < 1 ? 1 : (R > ns_i ? ns_i : R);
            const uint32_t* tm = reinterpret_cast<const uint32_t*>(a.ws + a.L.mma_tm) + (size_t)row * P.ns;
            uint32_t v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = (lane + 32 * i < ns_i) ? tm[lane + 32 * i] : 0u;
            // the largest x with #{v >= x} >= R is the R-th largest value
            uint32_t x = 0;
            for (int bit = 31; bit >= 0; --bit) {
                const uint32_t y = x | (1u << bit);
                int c = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) c += v[i] >= y;
                c = __reduce_add_sync(0xffffffffu, (unsigned)c);
                if (c >= R) x = y;
            }
            const float tau = f32_unorder(x);
            out.x = tau;
            out.z = __double2float_rd((double)tau - 2.0 * eps);
        }
    }
    if (lane == 0) reinterpret_cast<float4*>(a.ws + a.L.mma_row)[row] = out;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

template <int NQ, bool SAMPLE>
cudaError_t launch_score(const IndexArgs& a, const CUtensorMap& map, int sms, cudaStream_t s) {
    using G = Cfg<NQ>;
    auto k = mma_score_kernel<NQ, SAMPLE>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::SMEM);
    if (e != cudaSuccess) return e;
    // the largest shared-memory carveout, so that two 16-column CTAs fit on an SM
    e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const MmaPlan& P = a.plan.mma;
    const long long items = (long long)P.nseq * P.nqt * (SAMPLE ? P.nschunks : P.nchunks);
    int fit = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fit, k, G::THREADS, G::SMEM);
    if (e != cudaSuccess) return e;
    if (fit < 1) return cudaErrorInvalidConfiguration;
    // two CTAs share an SM's tensor memory when each takes 256 columns; their registers (launch
    // bounds) and shared memory (with the largest carveout) are sized for two per SM
    const int per_sm = G::COLS <= 256 ? 2 : 1;
    long long grid = (long long)sms * per_sm;
    if (grid > items) grid = items;
    if (grid < 1) return cudaSuccess;
    k<<<(unsigned)grid, G::THREADS, G::SMEM, s>>>(a, map);
    return cudaGetLastError();
}

template <int NQ>
cudaError_t launch_passes(const IndexArgs& a, const CUtensorMap& map, int sms, cudaStream_t s) {
    cudaError_t e = launch_score<NQ, true>(a, map, sms, s);
    if (e != cudaSuccess) return e;
    mma_tau_kernel<<<(unsigned)((a.rows + 7) / 8), 256, 0, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_score<NQ, false>(a, map, sms, s);
}

}  // namespace

cudaError_t launch_index_mma(const IndexArgs& a, cudaStream_t s) {
    const MmaPlan& P = a.plan.mma;
    if (!P.on || a.rows < 1) return cudaErrorInvalidValue;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    // the indexer code plane as [sequence][position][128 bytes]; a box is one key tile; positions
    // past the capacity read as zeros
    CUtensorMap map;
    const cuuint64_t gdim[3] = {(cuuint64_t)kIKBytes, (cuuint64_t)a.c.cap, (cuuint64_t)P.nseq};
    const cuuint64_t gstr[2] = {(cuuint64_t)kIKBytes, (cuuint64_t)a.c.cap * kIKBytes};
    const cuuint32_t box[3] = {(cuuint32_t)kIKBytes, (cuuint32_t)kTP, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.c.ik_data, gdim, gstr, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaMemsetAsync(a.ws + a.L.mma_zero, 0, a.L.mma_zero_bytes, s);
    if (e != cudaSuccess) return e;
    const int qblocks = (a.rows + 15) / 16;
    int64_t n = (int64_t)P.nt * kTP;
    int64_t sb = (n + 2047) / 2048;                 // about 8 positions per thread
    const int64_t sb_max = 4096 / P.nseq > 1 ? 4096 / P.nseq : 1;
    const int sblocks = (int)(sb < sb_max ? sb : sb_max);
    mma_prep_kernel<<<(unsigned)(qblocks + P.nseq * sblocks), 256, 0, s>>>(a, qblocks, sblocks);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return P.nq == 16 ? launch_passes<16>(a, map, sms, s) : launch_passes<256>(a, map, sms, s);
}

}  // namespace csa2
