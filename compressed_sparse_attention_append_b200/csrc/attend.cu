// attend.cu -- fused gather / dequantise / sparse softmax attention.
//
// [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token":
//   sec. VI "What one layer looks like": the layer's own query attends to the selected entries of
//   the shared main KV plus its own recent window;
//   sec. XI: cached values are dequantised before attention (E2M1 x E4M3 products are exact in
//   fp16, and FP8 window values are exact in fp16, so the dequantised keys and values are exact);
//   sec. XII: a query at position i sees window keys [max(s, i - win + 1), i].
// Reading taken here: one softmax over selected and window keys together, 16 query heads
// sharing one K/V head, default scale 1/sqrt(128).
//
// Work decomposition. A row's keys come in tiles: tile j < ceil(k / 16) holds the selected entries
// idx[16j .. 16j + 15] (entries that are -1 or invalid are zero-filled and masked), and the tiles
// after them hold 8 window rows each. One CTA of W warps takes a split of a row's tiles (one split
// per row for large batches); warp w takes the split's tiles w, w + W, ... and gathers each with
// cp.async into its own ring of S 2304-byte slots. With 16 warps of 3 slots (one CTA per SM) or 8
// warps of 5 slots (two per SM), a whole row of 512 selected entries and its window is requested
// at once, before any compute waits on memory, and 16 warps per SM hide each other's latencies.
// There is no compaction prologue: each warp reads the 16 indices of its own tile.
//
// Per tile, the raw rows are dequantised straight into mma.sync m16n8k16 fragments (fp16 in, fp32
// accumulate), the 16 heads being the M dimension:
//   S = Q K^T: the contraction order of the 128 dims is permuted so that thread (g, t) of a warp
//     takes k-step kk's operands from bytes 2kk, 2kk+1 of its own 16-byte slice [16t, 16t+16) of
//     the key's K codes (dims 32t..32t+31): one 16-byte load per key; Q is permuted alike.
//   O += P V: output dims are permuted so that thread (g, t) covers dims 16g..16g+15 (one scale
//     block) of four keys: one 8-byte load per key, pairs of keys interleaved with prmt.
// FP4 tiles and window tiles are never mixed, so every branch on the key kind is warp-uniform.
// The warps' (m, l, O) are merged in shared memory (with 16 warps, warps 8..15 first fold into
// warps 0..7); with several splits per row the partial results go to the workspace and the CTA that
// finishes a row's last split combines them.
//
// Precision: Q is converted bf16 -> fp16 (exact for |q| >= 2^-14; smaller magnitudes round to fp16
// subnormals, an absolute error below 2^-25); P is rounded to fp16 (relative 2^-11); all sums are
// fp32.
#include "csa2_internal.cuh"

namespace csa2 {

namespace {

constexpr int kTile = 16;                                  // selected entries per FP4 tile
constexpr int kWinTile = 8;                                // window rows per window tile
constexpr int kFp4Row = kKVBytes + kKVScales;              // 144: K codes 64, V codes 64, scales 16
constexpr int kSlot = kTile * kFp4Row;                     // 2304 (a window tile uses 8 x 256 = 2048)
constexpr int kQBytes = kHQ * kD * 2;                      // fp16 Q, 16-byte chunks XOR-swizzled by head

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t scale_h2(uint8_t s) { return e4m3x2_to_h2((uint16_t)(s | (s << 8))); }

// byte I of w (two E2M1 codes) -> half2, exact
template <int I>
__device__ __forceinline__ uint32_t e2m1x2_byte(uint32_t w) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b%2;\n\t}"
        : "=r"(r) : "r"(w), "n"(I));
    return r;
}

__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool on) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(on ? 16 : 0));
}

template <int W, int S>
__global__ void __launch_bounds__(W * 32, (W == 8 ? 2 : 1)) attend_kernel(AttendArgs a) {
    constexpr int kAThreads = W * 32, kAWarps = W;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int s_last;
    __shared__ unsigned int s_mask[kAWarps][S];  // valid keys of each ring slot (FP4 tiles)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int row = blockIdx.x, split = blockIdx.y;
    const int K = a.k;
    wait_prior_grid();  // indices, cache and queries come from earlier work on the stream
    uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + kHdrStatus);
    unsigned char* qs = smem + kAWarps * S * kSlot;

    const int b = row / a.tq;
    const int64_t qpos = a.qpos ? a.qpos[row] : a.qpos_base + row % a.tq;
    const int64_t qlast = qpos < 0 ? -1 : (qpos + 1) / a.ratio - 1;  // the last visible entry
    const bool row_ok = qpos >= 0 && qlast < a.c.cap;
    int64_t lo = qpos - a.win + 1;
    {
        const int64_t sb = a.swa_begin ? a.swa_begin[b] : a.swa_begin_host;
        if (lo < sb) lo = sb;
        if (lo < 0) lo = 0;
    }
    const int nwin = (row_ok && qpos >= lo) ? (int)(qpos - lo + 1) : 0;
    const int ft = (K + kTile - 1) / kTile;                    // FP4 tiles
    const int nt = row_ok ? ft + (nwin + kWinTile - 1) / kWinTile : 0;
    // this CTA's tiles [t_begin, t_end); this warp's: t_begin + warp + 8 i
    const int t_begin = split * a.plan.tps;
    const int t_end = min(t_begin + a.plan.tps, nt);
    const int my_first = t_begin + warp;
    const int ntiles = my_first < t_end ? (t_end - my_first + kAWarps - 1) / kAWarps : 0;

    // ---- Q -> fp16 in shared memory (thread: head tid>>4, dims 8*(tid&15) .. +7) ----
    if (tid < 256) {
        const int h = tid >> 4, c = tid & 15;
        const uint4 x0 = *reinterpret_cast<const uint4*>(a.q + (size_t)row * (kHQ * kD) + h * kD + 8 * c);
        const uint32_t w[4] = {x0.x, x0.y, x0.z, x0.w};
        uint32_t hv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) hv[i] = pack_h2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
        *reinterpret_cast<uint4*>(qs + h * 256 + ((c ^ (h & 7)) << 4)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    }

    unsigned char* wbase = smem + warp * (S * kSlot);
    const int32_t* idx = a.idx + (size_t)row * K;
    const size_t seq_row0 = (size_t)b * a.c.cap;
    const size_t swa_row0 = (size_t)b * a.c.swa_cap;
    const uint8_t* kv_base = a.c.kv_data + seq_row0 * kKVBytes;
    const uint8_t* sc_base = a.c.kv_scale + seq_row0 * kKVScales;
    // gather of tile `tj` into ring slot `st`:
    //   FP4 tile: 16 entries x (8 code chunks + 1 scale chunk) = 144 copies, lane l: l, l + 32, ...
    //   window tile: 8 rows x 16 chunks = 128 copies
    // index of entry (lane & 15) of tile tj (lanes 0..15; -1 past k or for a window tile); loaded
    // ahead of its issue so that the load latency overlaps other work
    auto load_idx = [&](int tj) -> int {
        const int i = tj * kTile + (lane & 15);
        return (tj < ft && lane < 16 && i < K) ? __ldg(idx + i) : -1;
    };
    auto issue = [&](int tj, int slot, int v) {
        unsigned char* st = wbase + slot * kSlot;
        if (tj < ft) {
            // codes: copy r, lane l -> chunk l & 7 of entry 4 r + l / 8 (four whole 128-byte rows per
            // copy instruction); scales: lanes 0..15, one 16-byte chunk each
            const int i = tj * kTile + (lane & 15);
            const bool ok = row_ok && v >= 0 && (int64_t)v <= qlast && (int64_t)v < a.c.cap;
            if (lane < 16 && i < K && !ok && v != -1) set_status(status, CSA2_DEV_BAD_INDEX);
            const unsigned int m = __ballot_sync(0xffffffffu, ok) & 0xFFFFu;
            if (lane == 0) s_mask[warp][slot] = m;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int kj = 4 * r + (lane >> 3), ch = lane & 7;
                const int e = __shfl_sync(0xffffffffu, v, kj);
                const bool on = (m >> kj) & 1u;
                cp_async16_zfill(st + kj * kFp4Row + 16 * ch, kv_base + (on ? (size_t)e : 0) * kKVBytes + 16 * ch, on);
            }
            {
                const int kj = lane & 15;
                const bool on = lane < 16 && ((m >> kj) & 1u);
                if (lane < 16) cp_async16_zfill(st + kj * kFp4Row + kKVBytes, sc_base + (on ? (size_t)v : 0) * kKVScales, on);
            }
        } else {
            // copy r, lane l -> chunk l & 15 of window row 2 r + l / 16 (two whole rows per copy)
            const int w0 = (tj - ft) * kWinTile;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int kj = 2 * r + (lane >> 4), ch = lane & 15;
                const bool on = w0 + kj < nwin;
                const int64_t p = lo + w0 + kj;
                const uint8_t* src = a.c.swa + (swa_row0 + (size_t)(on ? (p & (a.c.swa_cap - 1)) : 0)) * kSWABytes + 16 * ch;
                cp_async16_zfill(st + kj * kSWABytes + 16 * ch, src, on);
            }
        }
        cp_async_commit();
    };

    int vpre[S];
#pragma unroll
    for (int i = 0; i < S; ++i) vpre[i] = i < ntiles ? load_idx(my_first + i * kAWarps) : -1;
#pragma unroll
    for (int i = 0; i < S - 1; ++i) {
        if (i < ntiles) issue(my_first + i * kAWarps, i, vpre[i]);
        else cp_async_commit();
    }
    int vnext = vpre[S - 1];  // indices of the next tile to issue (tile S - 1, then one ahead)
    __syncthreads();  // Q in shared memory
    const float scale2 = a.sm_scale * 1.4426950408889634f;  // logits in log2 units

    // ---- Q fragments (read from shared memory at each use), permuted dims: k-step kk, thread t ->
    //      dims 32t + 4kk .. +3 of heads g (a0, a2) and g + 8 (a1, a3) ----
    auto q_frag = [&](int kk, uint32_t (&qa)[4]) {
        const int chunk = 4 * t + (kk >> 1), off = 8 * (kk & 1);
        const uint2 lo2 = *reinterpret_cast<const uint2*>(qs + g * 256 + ((chunk ^ g) << 4) + off);
        const uint2 hi2 = *reinterpret_cast<const uint2*>(qs + (g + 8) * 256 + ((chunk ^ g) << 4) + off);
        qa[0] = lo2.x;
        qa[1] = hi2.x;
        qa[2] = lo2.y;
        qa[3] = hi2.y;
    };

    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int it = 0; it < ntiles; ++it) {
        const int pf = it + S - 1;
        if (pf < ntiles) {
            issue(my_first + pf * kAWarps, pf % S, vnext);
            vnext = pf + 1 < ntiles ? load_idx(my_first + (pf + 1) * kAWarps) : -1;
        } else {
            cp_async_commit();
        }
        cp_async_wait<S - 1>();
        __syncwarp();
        const int slot = it % S;
        const unsigned char* st = wbase + slot * kSlot;
        const int tj = my_first + it * kAWarps;
        const bool fp4 = tj < ft;  // warp-uniform
        // valid keys of the tile: bit j = key j (FP4: 16 keys, window: 8 keys)
        const unsigned int vmask = fp4 ? s_mask[warp][slot]
                                       : ((nwin - (tj - ft) * kWinTile) >= kWinTile ? 0xFFu
                                          : ((1u << (nwin - (tj - ft) * kWinTile)) - 1u));
        // ---- S = Q K^T : n-tile nn holds keys 8nn .. 8nn+7, this thread's key 8nn + g ----
        float sc[2][4];
#pragma unroll
        for (int nn = 0; nn < 2; ++nn) sc[nn][0] = sc[nn][1] = sc[nn][2] = sc[nn][3] = 0.f;
        if (fp4) {
            //   FP4 row: k-step kk uses bytes 2kk, 2kk+1 of the 16-byte slice at 16t (dims 32t..32t+31);
            //   the two keys' MMA chains are interleaved
            uint32_t wa[2][4], sA[2], sB[2];
#pragma unroll
            for (int nn = 0; nn < 2; ++nn) {
                const unsigned char* sl = st + (8 * nn + g) * kFp4Row;
                const uint4 wv = *reinterpret_cast<const uint4*>(sl + 16 * t);
                const uint16_t s2 = *reinterpret_cast<const uint16_t*>(sl + 128 + 2 * t);
                wa[nn][0] = wv.x; wa[nn][1] = wv.y; wa[nn][2] = wv.z; wa[nn][3] = wv.w;
                sA[nn] = scale_h2((uint8_t)(s2 & 0xFF));
                sB[nn] = scale_h2((uint8_t)(s2 >> 8));
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t qa[4];
                q_frag(kk, qa);
#pragma unroll
                for (int nn = 0; nn < 2; ++nn) {
                    const uint32_t w = wa[nn][kk >> 1], sq = kk < 4 ? sA[nn] : sB[nn];
                    const uint32_t b0 = hmul2((kk & 1) ? e2m1x2_byte<2>(w) : e2m1x2_byte<0>(w), sq);
                    const uint32_t b1 = hmul2((kk & 1) ? e2m1x2_byte<3>(w) : e2m1x2_byte<1>(w), sq);
                    mma16816(sc[nn], qa, b0, b1);
                }
            }
        } else {
            //   FP8 row (a window tile has 8 keys): k-step kk uses bytes 4kk .. 4kk+3 of the 32-byte slice at 32t
            const unsigned char* sl = st + g * kSWABytes;
            const uint4 wA = *reinterpret_cast<const uint4*>(sl + 32 * t);
            const uint4 wB = *reinterpret_cast<const uint4*>(sl + 32 * t + 16);
            const uint32_t wa[8] = {wA.x, wA.y, wA.z, wA.w, wB.x, wB.y, wB.z, wB.w};
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t b0 = e4m3x2_to_h2((uint16_t)(wa[kk] & 0xFFFF));
                const uint32_t b1 = e4m3x2_to_h2((uint16_t)(wa[kk] >> 16));
                uint32_t qa[4];
                q_frag(kk, qa);
                mma16816(sc[0], qa, b0, b1);
            }
        }
        // ---- online softmax (rows g and g+8); masked keys get -inf ----
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nn = 0; nn < 2; ++nn) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const bool v = (vmask >> (nn * 8 + 2 * t + c)) & 1u;
                sc[nn][c] = v ? sc[nn][c] * scale2 : -INFINITY;
                sc[nn][2 + c] = v ? sc[nn][2 + c] * scale2 : -INFINITY;
                mx0 = fmaxf(mx0, sc[nn][c]);
                mx1 = fmaxf(mx1, sc[nn][2 + c]);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = (mn0 == -INFINITY) ? 1.f : exp2f(m0 - mn0);
        const float al1 = (mn1 == -INFINITY) ? 1.f : exp2f(m1 - mn1);
        float ps0 = 0.f, ps1 = 0.f;
        uint32_t pa[4];
#pragma unroll
        for (int nn = 0; nn < 2; ++nn) {
            const float p0 = (mn0 == -INFINITY) ? 0.f : exp2f(sc[nn][0] - mn0);
            const float p1 = (mn0 == -INFINITY) ? 0.f : exp2f(sc[nn][1] - mn0);
            const float p2 = (mn1 == -INFINITY) ? 0.f : exp2f(sc[nn][2] - mn1);
            const float p3 = (mn1 == -INFINITY) ? 0.f : exp2f(sc[nn][3] - mn1);
            ps0 += p0 + p1;
            ps1 += p2 + p3;
            pa[2 * nn] = pack_h2(p0, p1);
            pa[2 * nn + 1] = pack_h2(p2, p3);
        }
        l0 = l0 * al0 + ps0;
        l1 = l1 * al1 + ps1;
        m0 = mn0;
        m1 = mn1;
        if (!__all_sync(0xffffffffu, al0 == 1.f && al1 == 1.f)) {
#pragma unroll
            for (int i = 0; i < 16; ++i) { o[i][0] *= al0; o[i][1] *= al0; o[i][2] *= al1; o[i][3] *= al1; }
        }
        // ---- O += P V : keys 2t, 2t+1 (b0) and 2t+8, 2t+9 (b1); dims 16g + nd ----
        if (fp4) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {  // nd = 8hf .. 8hf+7
                uint32_t vw[4], vs[4];
#pragma unroll
                for (int kq = 0; kq < 4; ++kq) {
                    const int kj = (kq & 1) + 2 * t + ((kq & 2) ? 8 : 0);
                    const unsigned char* sl = st + kj * kFp4Row;
                    vw[kq] = *reinterpret_cast<const uint32_t*>(sl + 64 + 8 * g + 4 * hf);
                    vs[kq] = scale_h2(sl[128 + 8 + g]);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    // dims 16g + 8hf + 2i, +1 of the four keys
                    uint32_t hv[4];
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq) {
                        const uint32_t c = i == 0 ? e2m1x2_byte<0>(vw[kq]) : i == 1 ? e2m1x2_byte<1>(vw[kq])
                                         : i == 2 ? e2m1x2_byte<2>(vw[kq]) : e2m1x2_byte<3>(vw[kq]);
                        hv[kq] = hmul2(c, vs[kq]);
                    }
                    // n-tile nd = 8hf + 2i (low halves) and 8hf + 2i + 1 (high halves)
                    mma16816(o[8 * hf + 2 * i], pa, prmt(hv[0], hv[1], 0x5410), prmt(hv[2], hv[3], 0x5410));
                    mma16816(o[8 * hf + 2 * i + 1], pa, prmt(hv[0], hv[1], 0x7632), prmt(hv[2], hv[3], 0x7632));
                }
            }
        } else {
            // window tile: keys 2t, 2t+1 only (keys 8..15 of the mma are zero, their P is zero)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint2 vw[2];
#pragma unroll
                for (int kq = 0; kq < 2; ++kq)
                    vw[kq] = *reinterpret_cast<const uint2*>(st + (2 * t + kq) * kSWABytes + 128 + 16 * g + 8 * hf);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t hv[2];
#pragma unroll
                    for (int kq = 0; kq < 2; ++kq) {
                        const uint32_t w = (i >> 1) ? vw[kq].y : vw[kq].x;
                        hv[kq] = e4m3x2_to_h2((uint16_t)((i & 1) ? (w >> 16) : (w & 0xFFFF)));
                    }
                    mma16816(o[8 * hf + 2 * i], pa, prmt(hv[0], hv[1], 0x5410), 0u);
                    mma16816(o[8 * hf + 2 * i + 1], pa, prmt(hv[0], hv[1], 0x7632), 0u);
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    // ---- combine the warps (and splits) ----
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    __syncthreads();
    // O staging of 8 warps: head h, dim d = 32 c + j at h * kCoRow + 33 c + j (conflict-free for
    // both patterns)
    constexpr int kCoRow = 132;
    float* cm = reinterpret_cast<float*>(smem);              // [8][16] m
    float* cl = cm + 8 * kHQ;                                // [8][16] l
    float* co = cl + 8 * kHQ;                                // [8][16][kCoRow] O
    auto stage_out = [&](int slot8) {
        if (t == 0) {
            cm[slot8 * kHQ + g] = m0; cm[slot8 * kHQ + g + 8] = m1;
            cl[slot8 * kHQ + g] = l0; cl[slot8 * kHQ + g + 8] = l1;
        }
        // o[nd][0..1] -> head g, dims 32t + nd and 32t + 16 + nd; o[nd][2..3] -> head g + 8
        float* ow = co + slot8 * kHQ * kCoRow;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
            ow[g * kCoRow + 33 * t + nd] = o[nd][0];
            ow[g * kCoRow + 33 * t + 16 + nd] = o[nd][1];
            ow[(g + 8) * kCoRow + 33 * t + nd] = o[nd][2];
            ow[(g + 8) * kCoRow + 33 * t + 16 + nd] = o[nd][3];
        }
    };
    if (W == 16) {
        // first merge step: warps 8..15 stage, warps 0..7 fold their partner's (m, l, O) into their own
        if (warp >= 8) stage_out(warp - 8);
        __syncthreads();
        if (warp < 8) {
            const float pm0 = cm[warp * kHQ + g], pm1 = cm[warp * kHQ + g + 8];
            const float pl0 = cl[warp * kHQ + g], pl1 = cl[warp * kHQ + g + 8];
            const float n0 = fmaxf(m0, pm0), n1 = fmaxf(m1, pm1);
            const float fa0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - n0), fb0 = (pm0 == -INFINITY) ? 0.f : exp2f(pm0 - n0);
            const float fa1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - n1), fb1 = (pm1 == -INFINITY) ? 0.f : exp2f(pm1 - n1);
            const float* ow = co + warp * kHQ * kCoRow;
#pragma unroll
            for (int nd = 0; nd < 16; ++nd) {
                o[nd][0] = fa0 * o[nd][0] + fb0 * ow[g * kCoRow + 33 * t + nd];
                o[nd][1] = fa0 * o[nd][1] + fb0 * ow[g * kCoRow + 33 * t + 16 + nd];
                o[nd][2] = fa1 * o[nd][2] + fb1 * ow[(g + 8) * kCoRow + 33 * t + nd];
                o[nd][3] = fa1 * o[nd][3] + fb1 * ow[(g + 8) * kCoRow + 33 * t + 16 + nd];
            }
            l0 = fa0 * l0 + fb0 * pl0;
            l1 = fa1 * l1 + fb1 * pl1;
            m0 = n0;
            m1 = n1;
        }
        __syncthreads();
    }
    if (warp < 8) stage_out(warp);
    __syncthreads();
    const int splits = a.plan.splits;
    float* part = reinterpret_cast<float*>(a.ws + a.L.att_part) + ((size_t)row * splits) * kHQ * kPartStride;
    // 256 threads combine and write the output: thread -> (head h, 8 dims); with 16 warps the
    // others only take part in the barriers
    const bool wr = tid < 256;
    const int h = (tid & 255) >> 4, d0 = (tid & 15) * 8;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) M = fmaxf(M, cm[w * kHQ + h]);
    float Lsum = 0.f, acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const float mw = cm[w * kHQ + h];
        const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        Lsum += f * cl[w * kHQ + h];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += f * co[(w * kHQ + h) * kCoRow + 33 * (d0 >> 5) + (d0 & 31) + j];
    }
    if (splits > 1) {
        float* pp = part + ((size_t)split * kHQ + h) * kPartStride;
        if (wr) {
#pragma unroll
            for (int j = 0; j < 8; ++j) pp[d0 + j] = acc[j];
            if ((tid & 15) == 0) { pp[kD] = M; pp[kD + 1] = Lsum; }
        }
        __threadfence();
        __syncthreads();
        unsigned int* tk = reinterpret_cast<unsigned int*>(a.ws + a.L.att_ticket) + row;
        if (tid == 0) s_last = (atomicAdd(tk, 1u) == (unsigned)splits - 1);
        __syncthreads();
        if (!s_last || !wr) return;
        __threadfence();
        // the other splits' partials, read from L2 (they were written by other CTAs); this split's
        // own partial is still in registers. The splits are folded in index order, whichever CTA
        // finished last, so that the result does not depend on the order the splits finished in.
        const float M_own = M, L_own = Lsum;
        float acc_own[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) { acc_own[j] = acc[j]; acc[j] = 0.f; }
        M = M_own;
        for (int sp = 0; sp < splits; ++sp)
            if (sp != split) M = fmaxf(M, __ldcg(part + ((size_t)sp * kHQ + h) * kPartStride + kD));
        Lsum = 0.f;
        for (int sp = 0; sp < splits; ++sp) {
            float mw, lw, v[8];
            if (sp == split) {
                mw = M_own;
                lw = L_own;
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = acc_own[j];
            } else {
                const float* q = part + ((size_t)sp * kHQ + h) * kPartStride;
                const float4 v0 = __ldcg(reinterpret_cast<const float4*>(q + d0));
                const float4 v1 = __ldcg(reinterpret_cast<const float4*>(q + d0 + 4));
                mw = __ldcg(q + kD);
                lw = __ldcg(q + kD + 1);
                v[0] = v0.x; v[1] = v0.y; v[2] = v0.z; v[3] = v0.w;
                v[4] = v1.x; v[5] = v1.y; v[6] = v1.z; v[7] = v1.w;
            }
            const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
            Lsum += f * lw;
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] += f * v[j];
        }
        if (tid == 0) *tk = 0;
    }
    if (!wr) return;
    const bool empty = (M == -INFINITY) || !(Lsum > 0.f);
    const float inv = empty ? 0.f : 1.f / Lsum;
    const size_t ob = ((size_t)row * kHQ + h) * kD + d0;
    uint32_t pk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float x0 = acc[2 * j] * inv, x1 = acc[2 * j + 1] * inv;
        __nv_bfloat162 bb = __floats2bfloat162_rn(x0, x1);
        pk[j] = *reinterpret_cast<uint32_t*>(&bb);
        if (a.out_f32) *reinterpret_cast<float2*>(a.out_f32 + ob + 2 * j) = make_float2(x0, x1);
    }
    *reinterpret_cast<uint4*>(a.out + ob) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    if (a.lse && (tid & 15) == 0)
        a.lse[(size_t)row * kHQ + h] = empty ? -INFINITY : (M * 0.6931471805599453f + logf(Lsum));
}

}  // namespace

size_t attend_smem_bytes(int warps, int stages) { return (size_t)warps * stages * kSlot + kQBytes; }

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s) {
    const int W = a.plan.warps, S = a.plan.stages;
    const size_t smem = attend_smem_bytes(W, S);
    void (*kern)(AttendArgs) = W == 16 ? attend_kernel<16, 3> : attend_kernel<8, 5>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (a.rows == 0) return cudaSuccess;
    dim3 grid(a.rows, a.plan.splits);
    return launch_after_prior(kern, grid, dim3(W == 16 ? 512 : 256), smem, s, a);
}

}  // namespace csa2
