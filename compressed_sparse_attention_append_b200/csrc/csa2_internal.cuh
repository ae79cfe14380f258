// csa2_internal.cuh -- device helpers and the workspace plan shared by libcsa2's kernels.
//
// Sources (tags as in include/csa2.h):
//   [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token",
//       sec. XI "FP4 Main KV Cache": E2M1 elements, one E4M3 scale per 16 channels, no global
//       scale; SWA KV at FP8.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_fp4.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

// ---- fixed shapes of this library -------------------------------------------------------------
constexpr int kHQ = 16;       // query heads
constexpr int kD = 128;       // head dim (K and V)
constexpr int kKVBytes = 128; // packed E2M1 bytes of one main K||V row (256 channels)
constexpr int kKVScales = 16; // E4M3 scale bytes of one main row
constexpr int kHI = 4;        // indexer query heads
constexpr int kDI = 64;       // indexer head dim
constexpr int kHK = 4;        // indexer key heads
constexpr int kIKBytes = kHK * kDI / 2;   // 128
constexpr int kIKScales = kHK * kDI / 16; // 16
constexpr int kBS = 8;        // positions per pool block
constexpr int kSWABytes = 256;
constexpr int kMaxK = 2048;   // largest Top-k / pool size
constexpr int kPartStride = kD + 4;  // floats per (split, head) partial: O[128], m, l, 2 pad (16-byte rows)
constexpr int kKeyBins = 2048;  // score histogram bins of a decode row (sign, exponent, 4 mantissa bits)
constexpr int kSubBins = 1024;  // second-level bins (the next 10 bits) of a decode row's cut bin

// ---- device status word (first 4 bytes of the workspace) --------------------------------------
__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bit) {
    if (status) atomicOr(status, bit);
}

// ---- codec helpers -----------------------------------------------------------------------------
// Two E2M1 codes (one byte: low nibble = first element) -> half2 (low half = first element).
// Hardware conversion cvt.rn.f16x2.e2m1x2 (sm_100a); exact, every E2M1 value is an fp16 value.
__device__ __forceinline__ void e2m1x8_to_h2x4(uint32_t w, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

// Two E4M3 bytes (16-bit: low byte first) -> half2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint16_t v) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
    return r;
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t b) {
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3);
    return __half2float(__half(h));
}

__device__ __forceinline__ float2 h2_to_f2(uint32_t h) {
    __half2 v = *reinterpret_cast<__half2*>(&h);
    return __half22float2(v);
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float(((uint32_t)b) << 16);
}

// Orderable 64-bit key of an exact score: larger score <-> larger key; -0 and +0 map to the same
// key (the score is canonicalised by adding +0).
__device__ __forceinline__ uint64_t score_key(double s) {
    s = s + 0.0;
    uint64_t u = (uint64_t)__double_as_longlong(s);
    return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

// ---- codec: quantise one 16-channel block (the rule of include/csa2.h) -----------------------
// Two fp32 -> one byte of two E2M1 codes (first argument -> low nibble), RNE, saturating.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
    uint16_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
        "mov.b16 %0, {t, 0};\n\t}"
        : "=h"(r)
        : "f"(lo), "f"(hi));
    return r & 0xFF;
}

// Two fp32 -> two E4M3 bytes (first argument -> low byte), RNE, saturating to +-448.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void load16_bf16(const uint16_t* p, float (&x)[16]) {
    uint4 a = *reinterpret_cast<const uint4*>(p);
    uint4 b = *reinterpret_cast<const uint4*>(p + 8);
    uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// One 16-channel block: 8 code bytes + 1 scale byte.
__device__ __forceinline__ void quantize_block(const float (&x)[16], uint2& codes, uint8_t& scale) {
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    float s32 = __fdiv_rn(amax, 6.0f);
    uint32_t sc = f32x2_to_e4m3x2(s32, 0.f) & 0xFF;
    float s = e4m3_to_f32((uint8_t)sc);
    uint32_t b[8];
    if (s == 0.f) {
#pragma unroll
        for (int j = 0; j < 8; ++j) b[j] = 0;
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) b[j] = f32x2_to_e2m1x2(__fdiv_rn(x[2 * j], s), __fdiv_rn(x[2 * j + 1], s));
    }
    codes.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    codes.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
    scale = (uint8_t)sc;
}

// ---- score keys and their histogram bins ----------------------------------------------------------
// Histogram bin of an orderable score key (0 = no key): the score rounded to fp32 (round to
// nearest, so a larger score never rounds lower), then its sign, exponent and the top 4 mantissa
// bits. A larger key never has a smaller bin. Nonzero scores (|score| < 2^51) have exponents
// 127..178, so the positive bins are 1024 + 16..847 and the negative ones mirror them below 1024.
__device__ __forceinline__ int key_bin(unsigned long long key) {
    const unsigned int b = __float_as_uint(__ll2float_rn((long long)(key ^ 0x8000000000000000ull)));
    const int em = (int)((b >> 19) & 0xFFFu);  // exponent * 16 + top 4 mantissa bits
    const int f = em ? em - (126 << 4) : 0;
    return (b >> 31) ? kKeyBins / 2 - 1 - f : kKeyBins / 2 + f;
}

// Second-level bin of a key inside its key_bin: the next 10 mantissa bits of the same fp32 value,
// ordered like the keys within the bin.
__device__ __forceinline__ int sub_bin(unsigned long long key) {
    const unsigned int b = __float_as_uint(__ll2float_rn((long long)(key ^ 0x8000000000000000ull)));
    const int sb = (int)((b >> 9) & (unsigned int)(kSubBins - 1));
    return (b >> 31) ? kSubBins - 1 - sb : sb;
}

// ---- programmatic dependent launch -----------------------------------------------------------------
// Kernels that read an earlier kernel's output are launched with programmatic stream serialisation,
// so that their launch overlaps the end of the kernel before them; each one waits here before its
// first access to data an earlier kernel wrote (a no-op when launched without the attribute).
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_after_prior(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---- cp.async helpers ----------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N)); }

// ---- workspace plan (host and device agree on it) --------------------------------------------------
struct RowCtr {            // per query row of the index step
    unsigned int ticket;   // chunk items finished
    unsigned int ncand;    // candidates emitted
    unsigned long long tau;// max over finished chunks of their local k-th key (lower bound)
};

// Several query rows per sequence on the tensor cores (index_mma.cu): block-scaled FP4 MMA scores
// of 128-position key tiles against tiles of `nq` query rows; a sampled pass sets each row's
// admission threshold, a full pass collects the positions above it, exact integer rescoring picks
// the Top-k among them (index.cu).
constexpr int kMmaTile = 128;     // key positions per tile
constexpr int kMmaCap = 4096;     // candidates a row may rank (and positions it may rescore exactly)
constexpr int kMmaTarget = 1536;  // candidates per row the sampled threshold aims at
constexpr int64_t kMmaMinCtx = 8192;  // smaller contexts take the exact scan alone

struct MmaPlan {
    int on;            // 1: this plan runs the tensor-core filter (when the call allows it)
    int nq;            // query columns per tile: 16 or 256
    int nseq, nqt;     // sequences, query tiles per sequence
    int nt;            // key tiles per sequence covering max_ctx
    int st, ns;        // sampled key tiles: about every st-th tile, ns of them per sequence
    int kc, nchunks;   // key tiles per filter work item, work items per (sequence, query tile)
    int sc, nschunks;  // sampled tiles per sampling work item, items per (sequence, query tile)
    int subcap;        // candidate slots of one row in one filter work item
};

// Key tile of sample s: one tile out of each run of st, at an offset that varies with s.
__host__ __device__ inline int mma_sample_tile(int st, int s) { return s * st + (int)(((long long)s * 7) % st); }

struct IndexPlan {
    int rows;          // batch * tq
    int k;
    int units_max;     // 8-position units scanned per row (upper bound)
    int chunk_units;   // units per work item (several-row plans)
    int chunks;        // work items per row (several-row plans)
    int pool_blocks;   // 0 = no pool
    size_t cand_cap;   // candidate slots per row (decode rows: one key per position)
    int decode;        // 1: one query row per sequence, scored by score_kernel then select_kernel
    MmaPlan mma;
};

struct AttendPlan {
    int rows;
    int tiles;         // key tiles of a row: ceil(k / 16) tiles of selected entries, then ceil(win / 8) of the window
    int tps;           // tiles per split
    int splits;
    int warps;         // warps per CTA: 16 (one CTA per SM) or 8 (two CTAs per SM)
    int stages;        // gather ring depth per warp (3 with 16 warps, 5 with 8)
};

// Workspace: a fixed counter area first (its offsets never depend on the call, so counters
// left at zero by one call are zero for the next), then per-call data regions.
//   [0, 256)            header: u32 status, u32 pad, u32 index_next, u32 index_done
//   [256, +16*kMaxRows) RowCtr per index row
//   [.., +4*kMaxRows)   attention ticket per row
//   data: candidates, block maxima, attention partials (contents are scratch)
constexpr int kMaxRows = 65536;
constexpr int kSelCand = 4096;  // candidates of a decode row ranked by its last select CTA
// per decode row: key histogram, block-maximum histogram, and the two second-level histograms
constexpr int kRowHist = 2 * (kKeyBins + kSubBins);
constexpr size_t kHdrStatus = 0, kHdrIndexNext = 8, kHdrIndexDone = 12;

struct WsLayout {
    size_t row_ctr;    // RowCtr[kMaxRows]
    size_t att_ticket; // u32[kMaxRows]
    size_t cand_key;   // u64[rows * cand_cap]
    size_t cand_pos;   // i32[rows * cand_cap]
    size_t bmax;       // u64[rows * units_max] (pool)
    size_t key_hist;   // u32[rows][kRowHist] (decode plans: score histograms)
    size_t sel_key;    // u64[rows][2][kSelCand] (decode plans: candidate keys, then block maxima)
    size_t sel_pos;    // u64[rows][2][kSelCand] (element index << 32 | position, of each candidate)
    size_t att_part;   // f32[rows * splits * hq * kPartStride]
    // tensor-core filter (several-row plans with mma.on); the first four are one zeroed range
    size_t mma_zero, mma_zero_bytes;
    size_t mma_smax;   // u32[nseq][16]: largest key scale byte of each 16-channel block
    size_t mma_tend;   // u32[nseq * nqt]: key tiles visible to the rows of a query tile
    size_t mma_fail_n; // u32: rows left to the exact scan
    size_t mma_tm;     // u32[rows][ns]: orderable sampled tile maxima
    size_t mma_cnt;    // u32[rows][nchunks]: candidates of a row found by each filter item
    size_t mma_qc;     // u8[rows][128]: quantised query codes
    size_t mma_qs;     // u8[rows][16]: their scales
    size_t mma_row;    // float4[rows]: threshold estimate, error bound, admission threshold
    size_t mma_cpos;   // i32[rows][nchunks][subcap]: candidate positions
    size_t mma_cval;   // f32[rows][nchunks][subcap]: their approximate scores
    size_t mma_fail;   // i32[rows]
    size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// RowCtr index stride of the decode index path: row r uses RowCtr[r * stride], a 128-byte line of
// its own when the rows allow it (atomics of different rows then never share a line).
__host__ __device__ inline int ctr_stride(int rows) { return rows <= kMaxRows / 8 ? 8 : 1; }

inline IndexPlan make_index_plan(int rows, int tq, int k, int64_t max_scan, int pool_blocks) {
    IndexPlan p{};
    p.rows = rows;
    p.k = k;
    p.pool_blocks = pool_blocks;
    p.units_max = (int)((max_scan + kBS - 1) / kBS);
    if (p.units_max < 1) p.units_max = 1;
    if (tq == 1) {
        // decode rows: one orderable key per position (8 bytes against 144 bytes of indexer entry),
        // plus the select kernel's histograms and candidate lists (make_layout)
        p.decode = 1;
        p.cand_cap = (size_t)p.units_max * kBS;
        return p;
    }
    const int items_target = 148 * 4;
    int chunks_target = (items_target + rows - 1) / rows;
    if (chunks_target < 1) chunks_target = 1;
    int cu = (p.units_max + chunks_target - 1) / chunks_target;
    cu = (cu + 31) / 32 * 32;
    if (cu < 32) cu = 32;
    if (cu > 2048) cu = 2048;
    p.chunk_units = cu;
    p.chunks = (p.units_max + cu - 1) / cu;
    p.cand_cap = (size_t)p.chunks * (size_t)k;
    if (max_scan >= kMmaMinCtx && k <= 1024 && pool_blocks == 0) {
        MmaPlan& m = p.mma;
        m.on = 1;
        m.nq = tq <= 16 ? 16 : 256;
        m.nseq = rows / tq;
        m.nqt = (tq + m.nq - 1) / m.nq;
        m.nt = (int)((max_scan + kMmaTile - 1) / kMmaTile);
        int ns = m.nt / 16;
        ns = ns < 64 ? 64 : (ns > 256 ? 256 : ns);
        if (ns > m.nt) ns = m.nt;
        m.st = (m.nt + ns - 1) / ns;
        m.ns = (m.nt + m.st - 1) / m.st;
        const long long pairs = (long long)m.nseq * m.nqt;
        long long kc = (pairs * m.nt + 887) / 888;  // about six filter items per SM
        m.kc = (int)(kc < 8 ? 8 : (kc > 64 ? 64 : kc));
        m.nchunks = (m.nt + m.kc - 1) / m.kc;
        // about three times the candidates a row expects from one item, plus headroom
        const long long e = ((long long)kMmaTarget * m.kc + m.nt - 1) / m.nt;
        m.subcap = (int)((3 * e + 16 + 15) / 16 * 16);
        long long sc = (pairs * m.ns + 887) / 888;
        m.sc = (int)(sc < 1 ? 1 : (sc > 16 ? 16 : sc));
        m.nschunks = (m.ns + m.sc - 1) / m.sc;
    }
    return p;
}

inline AttendPlan make_attend_plan(int rows, int k, int win) {
    // A row's key tiles (16 selected entries, or 8 window rows, each) are split over the warps of one
    // CTA; 16 warps run on every SM (one CTA of 16 warps, or two of 8 when there are more CTAs than
    // SMs). Large batches take one CTA per row; small ones split a row's tiles over several CTAs (at
    // least one tile per warp each) so that about one CTA runs per SM, and merge the splits through
    // the workspace.
    AttendPlan a{};
    a.rows = rows;
    a.tiles = (k + 15) / 16 + (win + 7) / 8;
    int max_splits = a.tiles / 16 > 1 ? a.tiles / 16 : 1;
    int splits = rows >= 74 ? 1 : 148 / (rows > 0 ? rows : 1);
    if (splits < 1) splits = 1;
    if (splits > max_splits) splits = max_splits;
    a.tps = (a.tiles + splits - 1) / splits;
    a.splits = (a.tiles + a.tps - 1) / a.tps;
    const bool two_per_sm = (long long)rows * a.splits > 148;
    a.warps = two_per_sm ? 8 : 16;
    a.stages = two_per_sm ? 5 : 3;
    return a;
}

inline WsLayout make_layout(const IndexPlan* ip, const AttendPlan* ap) {
    WsLayout L{};
    size_t off = 256;
    L.row_ctr = off; off = align256(off + sizeof(RowCtr) * (size_t)kMaxRows);
    L.att_ticket = off; off = align256(off + 4 * (size_t)kMaxRows);
    int rows_i = ip ? ip->rows : 0;
    size_t cc = ip ? ip->cand_cap : 0;
    L.cand_key = off; off = align256(off + 8 * (size_t)rows_i * cc);
    L.cand_pos = off; off = align256(off + ((ip && ip->decode) ? 0 : 4 * (size_t)rows_i * cc));
    // rows of the decode path start on 16-byte boundaries (an even number of u64 per row)
    size_t bm = (ip && ip->pool_blocks > 0) ? (size_t)rows_i * (size_t)((ip->units_max + 1) & ~1) : 0;
    L.bmax = off; off = align256(off + 8 * bm);
    const size_t drows = (ip && ip->decode) ? (size_t)rows_i : 0;
    L.key_hist = off; off = align256(off + drows * kRowHist * 4);
    L.sel_key = off; off = align256(off + drows * 2 * kSelCand * 8);
    L.sel_pos = off; off = align256(off + drows * 2 * kSelCand * 8);
    size_t part = ap ? (size_t)ap->rows * (size_t)ap->splits * kHQ * kPartStride : 0;
    L.att_part = off; off = align256(off + 4 * part);
    const bool mma = ip && ip->mma.on;
    const size_t mrows = mma ? (size_t)rows_i : 0;
    L.mma_zero = off;
    L.mma_smax = off; off = align256(off + (mma ? 64 * (size_t)ip->mma.nseq : 0));
    L.mma_tend = off; off = align256(off + (mma ? 4 * (size_t)ip->mma.nseq * ip->mma.nqt : 0));
    L.mma_fail_n = off; off = align256(off + (mma ? 16 : 0));
    L.mma_tm = off; off = align256(off + (mma ? 4 * mrows * ip->mma.ns : 0));
    L.mma_zero_bytes = off - L.mma_zero;
    const size_t nch = mma ? (size_t)ip->mma.nchunks : 0, sub = mma ? (size_t)ip->mma.subcap : 0;
    L.mma_cnt = off; off = align256(off + 4 * mrows * nch);
    L.mma_qc = off; off = align256(off + 128 * mrows);
    L.mma_qs = off; off = align256(off + 16 * mrows);
    L.mma_row = off; off = align256(off + 16 * mrows);
    L.mma_cpos = off; off = align256(off + 4 * mrows * nch * sub);
    L.mma_cval = off; off = align256(off + 4 * mrows * nch * sub);
    L.mma_fail = off; off = align256(off + 4 * mrows);
    L.total = off;
    return L;
}

// ---- kernel launchers (defined in append.cu, index.cu, index_decode.cu, attend.cu) -----------------------------------
struct AppendArgs {
    csa2_cache c;
    int batch, t;
    const int64_t* pos;  // [batch], or NULL: every sequence starts at pos_host
    int64_t pos_host;
    const uint16_t* kv;
    const uint16_t* idx_k;
    const uint16_t* swa_kv;
    uint32_t* status;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t s);
cudaError_t launch_mxfp4(const uint16_t* x, long long rows, int channels, uint8_t* data, uint8_t* scale,
                         cudaStream_t s);  // append.cu: MXFP4 rows

struct IndexArgs {
    csa2_cache c;
    int rows;            // batch * tq
    int tq;
    const int64_t* qpos; // [rows], or NULL: row r sits at qpos_base + r % tq
    int64_t qpos_base;
    const uint16_t* idx_q;
    int reindex;         // 0 = Full, 1 = Reindex
    const int32_t* pool; // Reindex: [batch][pool_stride]
    const int32_t* pool_n;
    int pool_stride;
    int64_t max_ctx;     // Full: bound on the visible entries
    int ratio;           // tokens per cache entry (1 or 2): a row at token q sees (q + 1) / ratio entries
    int32_t* out_idx;
    int32_t* out_pool;
    int32_t* out_pool_n;
    uint32_t flags;
    IndexPlan plan;
    unsigned char* ws;
    WsLayout L;
    const int32_t* row_list;   // index_kernel: when set, only the rows listed (count *row_n) are scanned
    const uint32_t* row_n;
};
cudaError_t launch_index(const IndexArgs& a, cudaStream_t s);         // index.cu: any tq
cudaError_t launch_index_decode(const IndexArgs& a, cudaStream_t s);  // index_decode.cu: plan.decode
// index_mma.cu: the tensor-core filter up to the candidate lists (the final selection is index.cu's)
cudaError_t launch_index_mma(const IndexArgs& a, cudaStream_t s);

// Last visible cache entry of query row `row` of an index call: -1 when none is visible yet, -2 for
// a row whose token position is invalid (negative, or its entry at or past the capacity or max_ctx).
__device__ __forceinline__ int64_t index_row_last(const IndexArgs& a, int row) {
    const int64_t tok = a.qpos ? a.qpos[row] : a.qpos_base + row % a.tq;
    if (tok < 0) return -2;
    const int64_t q = (tok + 1) / a.ratio - 1;
    if (q >= a.c.cap || q >= a.max_ctx) return -2;
    return q;
}

// Orderable 32-bit image of a float (larger float <-> larger unsigned; 0 is below every image).
__device__ __forceinline__ uint32_t f32_order(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float f32_unorder(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

struct AttendArgs {
    csa2_cache c;
    int rows, tq, k, win;
    int ratio;            // tokens per cache entry: selected entries must be < (qpos + 1) / ratio
    const int64_t* qpos;  // or NULL: qpos_base + r % tq
    int64_t qpos_base;
    int64_t swa_begin_host;  // used when swa_begin is NULL
    const uint16_t* q;
    const int32_t* idx;
    const int64_t* swa_begin;
    float sm_scale;
    uint16_t* out;
    float* out_f32;
    float* lse;
    AttendPlan plan;
    unsigned char* ws;
    WsLayout L;
};
cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s);

// ---- the pages' own shape: the 512-channel latent (append.cu, latent.cu) ----------------------------
constexpr int kLatD = 512;       // latent channels (K = V)
constexpr int kLatHQ = 64;       // query heads
constexpr int kLatBytes = 256;   // E2M1 bytes of one latent entry
constexpr int kLatScales = 32;   // E4M3 scale bytes of one latent entry
constexpr int kLatKBytes = 64;   // MXFP4 codes of the 128-channel indexer key
constexpr int kLatKScales = 4;   // its E8M0 scales
constexpr int kLatSwa = 512;     // E4M3 bytes of one window row

struct LatentAppendArgs {
    csa2_latent_cache c;
    int batch, t;
    const int64_t* pos;  // [batch]
    const uint16_t* latent;
    const uint16_t* idx_k;
    const uint16_t* swa;
    uint32_t* status;
};
cudaError_t launch_latent_append(const LatentAppendArgs& a, cudaStream_t s);

struct LatentAttendArgs {
    csa2_latent_cache c;
    int rows, tq, k, win, ratio;
    const int64_t* qpos;       // [rows]
    const int64_t* swa_begin;  // [rows / tq] or NULL
    const uint16_t* q;
    const int32_t* idx;
    float sm_scale;
    uint16_t* out;
    float* out_f32;
    float* lse;
    uint32_t* status;
};
size_t latent_attend_smem_bytes();
cudaError_t launch_latent_attend(const LatentAttendArgs& a, cudaStream_t s);

constexpr int kLatMaxHI = 64;    // indexer query heads the latent indexer takes
struct LatIndexArgs {
    csa2_latent_cache c;
    int rows, tq, hi, k, ratio;
    int64_t max_ctx;              // bound on a row's visible entries (the key buffer's row length)
    const int64_t* qpos;          // [rows]
    uint32_t flags;
    const uint8_t* qcodes;        // workspace: the rows' quantised queries [rows][hi][64]
    const uint8_t* qscales;       // [rows][hi][4]
    unsigned long long* keys;     // [rows][max_ctx] orderable score keys
    int64_t key_stride;
    int32_t* out_idx;
    uint32_t* status;
};
size_t latent_index_ws_bytes(int rows, int hi, int64_t max_ctx);
cudaError_t launch_latent_index(LatIndexArgs a, const uint16_t* idx_q, unsigned char* ws, cudaStream_t s);

}  // namespace csa2
