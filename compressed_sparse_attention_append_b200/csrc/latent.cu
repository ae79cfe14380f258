// latent.cu -- sparse attention in the pages' own shape on the tensor cores: 64 query heads of 512
// channels over a 512-channel latent that is both key and value.
//
// [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token":
//   sec. VII: the main KV is one 512-channel latent per entry (288 B: E2M1 codes and an E4M3 scale
//   per 16 channels); the configuration list: 64 query heads of dimension 512;
//   sec. VI: the query attends to its selected entries plus its own recent window;
//   sec. XI: cached values are dequantised before attention (E2M1 x E4M3 products and E4M3 window
//   values are exact in fp16);
//   sec. XII: a query at token i sees window tokens [max(s, i - win + 1), i].
// Reading taken here: one softmax over selected and window entries, the latent serving as K and
// V (no separate value projection), default scale 1/sqrt(512).
//
// One CTA per query row, 16 warps. The row's keys come in tiles of 128: ceil(k / 128) tiles of
// selected entries (-1 or invalid entries are zero rows, masked), then one tile of up to 128 window
// rows. Per tile:
//   1. the tile's raw rows (loaded into registers while the previous tile was being processed) are
//      dequantised ONCE into a 128 x 512 fp16 tile L in shared memory (K-major rows of 128-byte
//      swizzled 64-channel blocks);
//   2. S^T = L Q^T on tcgen05 (kind::f16, M = 128 keys, N = 64 heads, K = 512), fp32 in tensor
//      memory;
//   3. softmax: each thread holds one key's logits for 16 heads; the tile's per-head maxima are
//      reduced across the CTA (a warp reduction per head, then the four lane quarters through
//      shared memory); the running maximum m of a head moves only when the tile exceeds it
//      by more than 8 (in log2 units), and then the head's accumulated O and l are rescaled (in
//      tensor memory), so P = exp2(logit - m) <= 2^8 stays well inside fp16; P is rounded to fp16
//      into shared memory, [key][head] (MN-major);
//   4. O^T += L^T P^T on tcgen05 (M = 128 channels, four M tiles, N = 64 heads, K = 128 keys): the
//      same shared-memory bytes of L, read MN-major (channels contiguous), so the latent is
//      dequantised once for both products.
// The two channel halves of L (64-channel blocks 0..3 and 4..7) are dequantised by separate halves
// of the CTA, each as soon as the O^T MMAs of the previous tile that read it have completed, and the
// S^T k-steps of a half are issued as soon as that half is in place (mbarriers between the threads
// and the MMA issuer), so dequantisation overlaps the tensor pipe. The row's indices are checked
// and staged in shared memory once, so no tile waits on a dependent index load.
// Tensor memory: S^T in columns 0..63, O^T in columns 64..319 (channels on the lanes).
// The result is normalised by the per-head sum of P at the end: out = O / l, lse = m ln 2 + ln l.
// Every wait on the tensor cores is bounded; one that runs out sets CSA2_DEV_TIMEOUT.
#include "csa2_internal.cuh"
#include "tc.cuh"

namespace csa2 {

namespace {

using namespace tc;

constexpr int kT = 512;                       // threads: key = tid & 127, channels 128 (tid >> 7) .. +127
constexpr int kTile = 128;                    // keys per tile (MMA M of S^T)
constexpr int kBlk = kTile * 128;             // 16384: one 64-channel block of the L tile
constexpr int kLTile = 8 * kBlk;              // 131072: the fp16 L tile
constexpr int kQBlk = kLatHQ * 128;           // 8192: one 64-channel block of Q (64 heads)
constexpr int kQBytes = 8 * kQBlk;            // 65536
constexpr int kPBytes = kTile * 128;          // 16384: P, 128 keys x 64 heads fp16
constexpr uint32_t kCols = 512;               // tensor memory allocated (power of two >= 320)
constexpr uint32_t kSCol = 0, kOCol = 64;
constexpr float kLazy = 8.f;
constexpr uint64_t kWaitNs = 200000000ull;
// f16 x f16 -> f32, M 128, N 64; S^T: both operands K-major; O^T: both MN-major (bits 15, 16)
constexpr uint32_t kIdescS = (1u << 4) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescO = kIdescS | (1u << 15) | (1u << 16);
constexpr size_t kOffQ = kLTile, kOffP = kOffQ + kQBytes, kOffIdx = kOffP + kPBytes;
constexpr size_t kOffRed = kOffIdx + 4 * kMaxK;
constexpr size_t kOffM = kOffRed + 4 * 64 * 4, kOffAl = kOffM + 64 * 4, kOffL = kOffAl + 64 * 4;
constexpr size_t kOffBar = kOffL + 64 * 4, kOffSlot = kOffBar + 8 * 8;
constexpr size_t kUsed = kOffSlot + 16;
// the whole 227 KB: one CTA per SM (tensor memory and the L tile allow no second one)
constexpr size_t kSmem = 232448;
static_assert(kUsed + 1024 <= kSmem, "shared memory plan");
// mbarriers: S^T done; O^T of channel half 0 / 1 done; channel half 0 / 1 of L dequantised
enum { kBarS = 0, kBarO0 = 1, kBarO1 = 2, kBarH0 = 3, kBarH1 = 4 };

__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d), "l"(ad), "l"(bd), "r"(idesc), "r"((uint32_t)acc)
        : "memory");
}

// MN-major operand in the 128-byte swizzle pattern: 64-element groups of the M (or N) dimension
// `lbo` bytes apart, 8-row groups of K 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc_mn(uint32_t addr, uint32_t lbo) {
    return sw128_desc(addr) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16);
}

// byte offset of 16-byte chunk c of row r in a 128-byte-swizzled block (8-row groups of 1024 bytes)
__device__ __forceinline__ uint32_t sw(int r, int c) { return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t scale_h2(uint32_t s) { return e4m3x2_to_h2((uint16_t)(s | (s << 8))); }

// the largest value of v over the warp, in every lane (sm_100a warp reduction)
__device__ __forceinline__ float warp_max(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}
// 2^x (the hardware approximation: relative error about 2^-22; results below 2^-126 flush to 0)
__device__ __forceinline__ float ex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// 16 lanes' worth of sums reduced across the warp: lane L < 16 ends with the sum over all 32 lanes
// of element L (the transposing butterfly: each step halves the elements a lane keeps).
__device__ __forceinline__ float warp_sum16(float (&v)[16], int lane) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], 16);
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1) {
        const bool up = (lane & w) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float keep = up ? v[i + w] : v[i], send = up ? v[i] : v[i + w];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
    }
    return v[0];
}

__global__ void __launch_bounds__(kT, 1) latent_attend_kernel(LatentAttendArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    unsigned char* Lt = sm;
    unsigned char* Qs = sm + kOffQ;
    unsigned char* Ps = sm + kOffP;
    int* sidx = reinterpret_cast<int*>(sm + kOffIdx);       // the row's selected entries, -1 if unusable
    float* red = reinterpret_cast<float*>(sm + kOffRed);   // [4 lane quarters][64 heads]
    float* s_m = reinterpret_cast<float*>(sm + kOffM);     // running maximum per head (log2 units)
    float* s_al = reinterpret_cast<float*>(sm + kOffAl);   // this tile's rescale factor per head
    float* s_l = reinterpret_cast<float*>(sm + kOffL);     // final sum per head
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kOffSlot);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int key = tid & 127, qq = tid >> 7;      // load / dequantise: key, channels 128 qq ..
    const int half = qq >> 1;                      // channel half (blocks 4 half .. 4 half + 3)
    const int quad = warp & 3, cg = warp >> 2;     // softmax / epilogue: lanes 32 quad .., heads 16 cg ..
    const int row = blockIdx.x, K = a.k;
    wait_prior_grid();  // indices, cache and queries come from earlier work on the stream

    const int b = row / a.tq;
    const int64_t qpos = a.qpos[row];
    const int64_t qlast = qpos < 0 ? -1 : (qpos + 1) / a.ratio - 1;  // the last visible entry
    const bool row_ok = qpos >= 0 && qlast < a.c.cap;
    int64_t lo = qpos - a.win + 1;
    {
        const int64_t sb = a.swa_begin ? a.swa_begin[b] : 0;
        if (lo < sb) lo = sb;
        if (lo < 0) lo = 0;
    }
    const int nwin = (row_ok && qpos >= lo) ? (int)(qpos - lo + 1) : 0;
    const int ft = row_ok ? (K + kTile - 1) / kTile : 0;
    const int nt = ft + (nwin > 0 ? 1 : 0);
    const float scale2 = a.sm_scale * 1.4426950408889634f;  // logits in log2 units
    uint32_t* status = a.status;

    if (tid == 0) {
        mbar_init(&bars[kBarS], 1);
        mbar_init(&bars[kBarO0], 1);
        mbar_init(&bars[kBarO1], 1);
        mbar_init(&bars[kBarH0], kT / 2);
        mbar_init(&bars[kBarH1], kT / 2);
        mbar_fence_init();
    }
    if (tid < 64) s_m[tid] = -INFINITY;
    if (warp == 0) tmem_alloc(tslot, kCols);
    // Q (this thread: head tid >> 3, channels 64 (tid & 7) ..) requested first; it is converted once
    // the row's indices are staged and tile 0's rows requested, so that the three loads overlap
    uint4 qv[8];
    {
        const uint4* src = reinterpret_cast<const uint4*>(a.q + ((size_t)row * kLatHQ + (tid >> 3)) * kLatD + 64 * (tid & 7));
#pragma unroll
        for (int c = 0; c < 8; ++c) qv[c] = __ldg(src + c);
    }
    // the row's indices, checked once (an entry that is -1, not visible or out of range becomes -1)
    for (int i = tid; i < (row_ok ? K : 0); i += kT) {
        const int v = __ldg(a.idx + (size_t)row * K + i);
        const bool ok = v >= 0 && (int64_t)v <= qlast && (int64_t)v < a.c.cap;
        if (!ok && v != -1) set_status(status, CSA2_DEV_BAD_INDEX);
        sidx[i] = ok ? v : -1;
    }

    const size_t seq_row0 = (size_t)b * a.c.cap;
    const size_t swa_row0 = (size_t)b * a.c.swa_cap;
    bool ok_all = true;
    auto wait_bar = [&](int i, uint32_t parity) {
        if (!mbar_wait(&bars[i], parity, kWaitNs)) {
            if (ok_all) set_status(status, CSA2_DEV_TIMEOUT);
            ok_all = false;
        }
    };

    // this thread's window row (key `key` of the window tile), channels 128 qq ..
    auto win_src = [&]() {
        const int64_t p = lo + key;
        return reinterpret_cast<const uint4*>(a.c.swa + (swa_row0 + (size_t)(p & (a.c.swa_cap - 1))) * kLatSwa +
                                              128 * qq);
    };
    // ---- raw rows of tile j into registers (this thread: key `key`, channels 128 qq .. +127) ----
    // (of a window row only the first 64 channels: the other 64 are loaded while it is dequantised,
    // so that no more than 18 registers of raw data stay live across the softmax of the tile before)
    uint4 raw[4];
    uint2 rsc;
    bool kvalid = false;  // the key of this thread in the tile being loaded
    auto load_tile = [&](int j) {
#pragma unroll
        for (int i = 0; i < 4; ++i) raw[i] = make_uint4(0, 0, 0, 0);
        rsc = make_uint2(0, 0);
        kvalid = false;
        if (j < ft) {
            const int i = j * kTile + key;
            const int v = i < K ? sidx[i] : -1;
            if (v >= 0) {
                kvalid = true;
                const uint4* src = reinterpret_cast<const uint4*>(a.c.l_data + (seq_row0 + (size_t)v) * kLatBytes + 64 * qq);
#pragma unroll
                for (int c = 0; c < 4; ++c) raw[c] = __ldg(src + c);
                rsc = __ldg(reinterpret_cast<const uint2*>(a.c.l_scale + (seq_row0 + (size_t)v) * kLatScales + 8 * qq));
            }
        } else if (j < nt && key < nwin) {
            kvalid = true;
#pragma unroll
            for (int c = 0; c < 4; ++c) raw[c] = __ldg(win_src() + c);  // channels 128 qq .. +63
        }
    };
    // dequantise the registers into the L tile: channel 128 qq + 8 c lands in 64-channel block
    // 2 qq + c / 8, chunk c % 8, of row `key`
    auto dequant = [&](bool fp4, bool kvalid_dq) {
        if (fp4) {
#pragma unroll
            for (int bk = 0; bk < 8; ++bk) {  // 16-channel scale block bk: code words 2 bk, 2 bk + 1
                const uint32_t s2 = scale_h2(((bk < 4 ? rsc.x : rsc.y) >> (8 * (bk & 3))) & 0xFFu);
                const uint4 rw = raw[bk >> 1];
                const uint32_t w0 = (bk & 1) ? rw.z : rw.x, w1 = (bk & 1) ? rw.w : rw.y;
                uint32_t h0[4], h1[4];
                e2m1x8_to_h2x4(w0, h0);
                e2m1x8_to_h2x4(w1, h1);
#pragma unroll
                for (int i = 0; i < 4; ++i) { h0[i] = hmul2(h0[i], s2); h1[i] = hmul2(h1[i], s2); }
                const int c0 = 2 * bk;  // chunk index among the thread's 16 chunks of 8 channels
                *reinterpret_cast<uint4*>(Lt + (2 * qq + (c0 >> 3)) * kBlk + sw(key, c0 & 7)) = make_uint4(h0[0], h0[1], h0[2], h0[3]);
                *reinterpret_cast<uint4*>(Lt + (2 * qq + ((c0 + 1) >> 3)) * kBlk + sw(key, (c0 + 1) & 7)) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
            }
        } else {
            // window row: channels 128 qq .. +63 from the registers, then the other 64 channels
            // (loaded here, once per row, to keep register pressure below the limit)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                if (hh == 1) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) raw[c] = kvalid_dq ? __ldg(win_src() + 4 + c) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) {  // 8 window channels per chunk
                    const uint4 rw = raw[c >> 1];
                    const uint32_t w0 = (c & 1) ? rw.z : rw.x, w1 = (c & 1) ? rw.w : rw.y;
                    const uint4 h = make_uint4(e4m3x2_to_h2((uint16_t)(w0 & 0xFFFFu)), e4m3x2_to_h2((uint16_t)(w0 >> 16)),
                                               e4m3x2_to_h2((uint16_t)(w1 & 0xFFFFu)), e4m3x2_to_h2((uint16_t)(w1 >> 16)));
                    *reinterpret_cast<uint4*>(Lt + (2 * qq + hh) * kBlk + sw(key, c)) = h;
                }
            }
        }
    };

    __syncthreads();  // barriers, s_m, indices
    load_tile(0);
    {   // Q -> fp16 (B operand of S^T, K-major: row = head, 64-channel blocks)
        const int h = tid >> 3, cb = tid & 7;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t w[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
            uint32_t hv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) hv[i] = pack_h2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
            *reinterpret_cast<uint4*>(Qs + cb * kQBlk + sw(h, c)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();  // Q, tensor memory address
    tc_fence_after();
    const uint32_t tb = *tslot;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;

    float lsum[16];  // this thread's key slot: sum of P per head 16 cg + i over the tiles so far
#pragma unroll
    for (int i = 0; i < 16; ++i) lsum[i] = 0.f;

    // Per tile j: each channel half of L is dequantised by its 256 threads as soon as the O^T MMAs
    // of tile j - 1 that read that half have completed (O^T m-tiles 0, 1 read half 0, m-tiles 2, 3
    // half 1), and the S^T k-steps of a half are issued as soon as the half is in shared memory, so
    // that dequantisation overlaps the tensor pipe. The softmax then runs on all 16 warps.
    for (int j = 0; j < nt; ++j) {
        const bool fp4 = j < ft;  // CTA-uniform
        const bool valid = kvalid;
        if (j > 0) wait_bar(half ? kBarO1 : kBarO0, (uint32_t)(j - 1) & 1u);
        dequant(fp4, valid);
        fence_async_smem();
        mbar_arrive(&bars[half ? kBarH1 : kBarH0]);
        if (j + 1 < nt) load_tile(j + 1);  // in flight during this tile's MMAs and softmax
        if (tid == 0) {
            wait_bar(kBarH0, (uint32_t)j & 1u);
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
                const uint32_t off = (uint32_t)((kk >> 2) * kBlk + 32 * (kk & 3));
                const uint32_t qoff = (uint32_t)((kk >> 2) * kQBlk + 32 * (kk & 3));
                mma_f16(tb + kSCol, sw128_desc(smem_u32(Lt) + off), sw128_desc(smem_u32(Qs) + qoff), kIdescS, kk > 0);
            }
            wait_bar(kBarH1, (uint32_t)j & 1u);
            tc_fence_after();
#pragma unroll
            for (int kk = 16; kk < 32; ++kk) {
                const uint32_t off = (uint32_t)((kk >> 2) * kBlk + 32 * (kk & 3));
                const uint32_t qoff = (uint32_t)((kk >> 2) * kQBlk + 32 * (kk & 3));
                mma_f16(tb + kSCol, sw128_desc(smem_u32(Lt) + off), sw128_desc(smem_u32(Qs) + qoff), kIdescS, true);
            }
            mma_commit(&bars[kBarS]);
        }
        __syncwarp();
        wait_bar(kBarS, (uint32_t)j & 1u);  // also every earlier MMA (the O^T of tile j - 1)
        tc_fence_after();

        // ---- softmax of the tile: this thread's key 32 quad + lane (= key), heads 16 cg .. +15 ----
        float lg[16];  // raw logits q . l (the scale is applied inside the exponent)
        {
            uint32_t v[16];
            tmem_ld16(tb + lane_base + kSCol + 16 * cg, v);
            tmem_ld_wait();
            float r[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                lg[i] = __uint_as_float(v[i]);
                r[i] = warp_max(valid ? lg[i] * scale2 : -INFINITY);  // (any sign of the scale)
            }
            if (lane == 0) {
                float4* d = reinterpret_cast<float4*>(red + quad * 64 + 16 * cg);
                d[0] = make_float4(r[0], r[1], r[2], r[3]);
                d[1] = make_float4(r[4], r[5], r[6], r[7]);
                d[2] = make_float4(r[8], r[9], r[10], r[11]);
                d[3] = make_float4(r[12], r[13], r[14], r[15]);
            }
        }
        __syncthreads();
        int resc = 0;
        if (tid < 64) {
            const float tmax = fmaxf(fmaxf(red[tid], red[64 + tid]), fmaxf(red[128 + tid], red[192 + tid]));
            const float m_old = s_m[tid];
            float al = 1.f;
            if (tmax > m_old + kLazy) {  // also the first finite maximum (m_old = -inf)
                al = (m_old == -INFINITY) ? 0.f : exp2f(m_old - tmax);
                resc = m_old != -INFINITY;
                s_m[tid] = tmax;
            }
            s_al[tid] = al;
        }
        resc = __syncthreads_or(resc);
        const float* al = s_al + 16 * cg;  // this warp's heads (shared-memory broadcasts)
        const float* mh = s_m + 16 * cg;
        if (resc) {
            // every O^T MMA so far has completed (the S^T commit tracks them): scale in place
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                uint32_t v[16];
                const uint32_t addr = tb + lane_base + kOCol + 64 * mt + 16 * cg;
                tmem_ld16(addr, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * al[i]);
                tmem_st16(addr, v);
            }
            tmem_st_wait();
        }
        // a valid key makes every head's maximum finite, so p needs no test of m for -inf
        uint32_t ph[8];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const float p0 = valid ? ex2(fmaf(lg[i], scale2, -mh[i])) : 0.f;
            const float p1 = valid ? ex2(fmaf(lg[i + 1], scale2, -mh[i + 1])) : 0.f;
            lsum[i] = fmaf(lsum[i], al[i], p0);
            lsum[i + 1] = fmaf(lsum[i + 1], al[i + 1], p1);
            ph[i >> 1] = pack_h2(p0, p1);
        }
        // P [key][head]: heads 16 cg .. +7 -> chunk 2 cg, 16 cg + 8 .. -> chunk 2 cg + 1
        *reinterpret_cast<uint4*>(Ps + sw(key, 2 * cg)) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
        *reinterpret_cast<uint4*>(Ps + sw(key, 2 * cg + 1)) = make_uint4(ph[4], ph[5], ph[6], ph[7]);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // A = L^T: channels 128 mt .. (blocks 2 mt, 2 mt + 1, kBlk apart), keys 16 kk ..
                    const uint64_t ad = sw128_desc_mn(smem_u32(Lt) + (uint32_t)(2 * mt * kBlk + 2048 * kk), kBlk);
                    // B = P: heads 0..63 (one 64-element group), keys 16 kk ..
                    const uint64_t bd = sw128_desc_mn(smem_u32(Ps) + (uint32_t)(2048 * kk), 0);
                    mma_f16(tb + kOCol + 64 * mt, ad, bd, kIdescO, j > 0 || kk > 0);
                }
                if (mt == 1) mma_commit(&bars[kBarO0]);  // channel half 0 of L is free again
            }
            mma_commit(&bars[kBarO1]);
        }
        __syncwarp();
    }
    if (nt > 0) {
        wait_bar(kBarO1, (uint32_t)(nt - 1) & 1u);  // the last MMAs (in issue order)
        tc_fence_after();
    }

    // ---- epilogue: l per head, then out = O / l (warp: channels 128 mt + 32 quad + lane, heads 16 cg ..) ----
    {
        const float r = warp_sum16(lsum, lane);
        if (lane < 16) red[quad * 64 + 16 * cg + lane] = r;
    }
    __syncthreads();
    if (tid < 64) {
        const float l = (red[tid] + red[64 + tid]) + (red[128 + tid] + red[192 + tid]);
        s_l[tid] = l;
        const bool em = (nt == 0) || (s_m[tid] == -INFINITY) || !(l > 0.f);
        s_al[tid] = em ? 0.f : 1.f / l;  // 1 / l per head (0 for a row with no key: O is 0 there)
    }
    __syncthreads();
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
        uint32_t v[16] = {};
        if (nt > 0) {
            tmem_ld16(tb + lane_base + kOCol + 64 * mt + 16 * cg, v);
            tmem_ld_wait();
        }
        const int d = 128 * mt + 32 * quad + lane;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float x = __uint_as_float(v[i]) * s_al[16 * cg + i];
            const size_t ob = ((size_t)row * kLatHQ + 16 * cg + i) * kLatD + d;
            a.out[ob] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
            if (a.out_f32) a.out_f32[ob] = x;
        }
    }
    if (a.lse && tid < 64) {
        const bool e = (nt == 0) || (s_m[tid] == -INFINITY) || !(s_l[tid] > 0.f);
        a.lse[(size_t)row * kLatHQ + tid] = e ? -INFINITY : (s_m[tid] * 0.6931471805599453f + logf(s_l[tid]));
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tb, kCols);
}

}  // namespace

size_t latent_attend_smem_bytes() { return kSmem; }

cudaError_t launch_latent_attend(const LatentAttendArgs& a, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(latent_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    if (a.rows == 0) return cudaSuccess;
    return launch_after_prior(latent_attend_kernel, dim3((unsigned)a.rows), dim3(kT), kSmem, s, a);
}

}  // namespace csa2
