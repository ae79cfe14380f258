// attend.cu -- fused gather / dequantise / sparse softmax attention with split-K.
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
// Per CTA: one query row and one split of its key list (valid selected entries in index order,
// then the window). Eight warps each own 16-key tiles. Raw rows (FP4 codes + scales, or FP8
// window entries) are gathered with cp.async into a warp-private 3-stage ring and dequantised
// straight into mma.sync m16n8k16 fragments (fp16 in, fp32 accumulate), the 16 heads being the M
// dimension:
//   S = Q K^T: the contraction order of the 128 dims is permuted so that thread (g, t) of a warp
//     takes k-step kk's operands from bytes 2kk, 2kk+1 of its own 16-byte slice [16t, 16t+16) of
//     the key's K codes (dims 32t..32t+31): one 16-byte load per key; Q is permuted alike.
//   O += P V: output dims are permuted so that thread (g, t) covers dims 16g..16g+15 (one scale
//     block) of four keys: one 8-byte load per key, pairs of keys interleaved with prmt.
// The eight warps' (m, l, O) are merged in shared memory; with several splits per row the partial
// results go to the workspace and the CTA that finishes a row's last split combines them.
//
// Precision: Q is converted bf16 -> fp16 (exact for |q| >= 2^-14; smaller magnitudes round to fp16
// subnormals, an absolute error below 2^-25); P is rounded to fp16 (relative 2^-11); all sums are
// fp32.
#include "csa2_internal.cuh"

namespace csa2 {

namespace {

constexpr int kAThreads = 256;
constexpr int kAWarps = 8;
constexpr int kTile = 16;        // keys per warp step
constexpr int kStages = 3;
// stage layout: one 272-byte slot per key. An FP4 row keeps the cache layout (K codes at 0, V codes
// at 64, scales at 128); a window row holds its FP8 K at 0 and V at 128.
constexpr int kSlot = 272;
constexpr int kStageBytes = kTile * kSlot;                 // 4352
constexpr int kWarpSmem = kStages * kStageBytes;           // 13056
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

struct RowKeys {
    int nsel, nwin, nk;
    int64_t lo, qpos;
    int b;
};

__global__ void __launch_bounds__(kAThreads, 2) attend_kernel(AttendArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int s_cnt[64];
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int row = blockIdx.x, split = blockIdx.y;
    const int K = a.k;
    wait_prior_grid();  // indices, cache and queries come from earlier work on the stream
    uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + kHdrStatus);
    unsigned char* qs = smem + kAWarps * kWarpSmem;
    int* list = reinterpret_cast<int*>(qs + kQBytes);

    RowKeys R;
    R.b = row / a.tq;
    R.qpos = a.qpos ? a.qpos[row] : a.qpos_base + row % a.tq;
    const int64_t qlast = R.qpos < 0 ? -1 : (R.qpos + 1) / a.ratio - 1;  // the last visible entry
    const bool row_ok = R.qpos >= 0 && qlast < a.c.cap;
    // ---- Q -> fp16 in shared memory (thread: head tid>>4, dims 8*(tid&15) .. +7) ----
    {
        const int h = tid >> 4, c = tid & 15;
        const uint4 x0 = *reinterpret_cast<const uint4*>(a.q + (size_t)row * (kHQ * kD) + h * kD + 8 * c);
        const uint32_t w[4] = {x0.x, x0.y, x0.z, x0.w};
        uint32_t hv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) hv[i] = pack_h2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
        *reinterpret_cast<uint4*>(qs + h * 256 + ((c ^ (h & 7)) << 4)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    }
    // ---- valid selected indices, compacted in index order (coalesced, two passes) ----
    const int32_t* idx = a.idx + (size_t)row * K;
    const int rounds = (K + kAThreads - 1) / kAThreads;
    for (int r = 0; r < rounds; ++r) {
        const int i = r * kAThreads + tid;
        const int v = i < K ? idx[i] : -1;
        const bool ok = row_ok && v >= 0 && v <= qlast && (int64_t)v < a.c.cap;
        if (!ok && v != -1 && split == 0) set_status(status, CSA2_DEV_BAD_INDEX);
        const unsigned int bal = __ballot_sync(0xffffffffu, ok);
        if (lane == 0) s_cnt[r * kAWarps + warp] = __popc(bal);
    }
    __syncthreads();
    if (warp == 0) {
        const int n = rounds * kAWarps;  // <= 64 (k <= 2048)
        const int c0 = lane < n ? s_cnt[lane] : 0, c1 = lane + 32 < n ? s_cnt[lane + 32] : 0;
        int inc0 = c0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc0, o);
            if (lane >= o) inc0 += v;
        }
        const int tot0 = __shfl_sync(0xffffffffu, inc0, 31);
        int inc1 = c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc1, o);
            if (lane >= o) inc1 += v;
        }
        if (lane < n) s_cnt[lane] = inc0 - c0;
        if (lane + 32 < n) s_cnt[lane + 32] = tot0 + inc1 - c1;
        if (lane == 31) s_last = tot0 + inc1;
    }
    __syncthreads();
    for (int r = 0; r < rounds; ++r) {
        const int i = r * kAThreads + tid;
        const int v = i < K ? idx[i] : -1;
        const bool ok = row_ok && v >= 0 && v <= qlast && (int64_t)v < a.c.cap;
        const unsigned int bal = __ballot_sync(0xffffffffu, ok);
        if (ok) list[s_cnt[r * kAWarps + warp] + __popc(bal & ((1u << lane) - 1))] = v;
    }
    R.nsel = s_last;
    {
        int64_t lo = R.qpos - a.win + 1;
        const int64_t sb = a.swa_begin ? a.swa_begin[R.b] : a.swa_begin_host;
        if (lo < sb) lo = sb;
        if (lo < 0) lo = 0;
        R.lo = lo;
        R.nwin = (row_ok && R.qpos >= lo) ? (int)(R.qpos - lo + 1) : 0;
        R.nk = R.nsel + R.nwin;
    }
    __syncthreads();

    const int k_begin = split * a.plan.kps;
    const int k_end = min(k_begin + a.plan.kps, R.nk);
    const float scale2 = a.sm_scale * 1.4426950408889634f;  // logits in log2 units

    // ---- Q fragments (read from shared memory at each use), permuted dims: k-step kk, thread t ->
    //      dims 32t + 4kk .. +3 of heads g (a0, a2) and g + 8 (a1, a3) ----
    auto q_frag = [&](int kk, uint32_t (&qa)[4]) {
        const int chunk = 4 * t + (kk >> 1), off = 8 * (kk & 1);
        const uint2 lo = *reinterpret_cast<const uint2*>(qs + g * 256 + ((chunk ^ g) << 4) + off);
        const uint2 hi = *reinterpret_cast<const uint2*>(qs + (g + 8) * 256 + ((chunk ^ g) << 4) + off);
        qa[0] = lo.x;
        qa[1] = hi.x;
        qa[2] = lo.y;
        qa[3] = hi.y;
    };

    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    unsigned char* wbase = smem + warp * kWarpSmem;
    const size_t seq_row0 = (size_t)R.b * a.c.cap;
    const size_t swa_row0 = (size_t)R.b * a.c.swa_cap;
    // gather of tile `ts` (16 keys): FP4 rows -> 4 K chunks, 4 V chunks, 1 scale chunk;
    // window rows -> 8 K chunks, 8 V chunks
    auto issue = [&](int ts, unsigned char* st) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int slot = lane + 32 * i;
            const int kj = slot >> 4, ch = slot & 15;
            const int gk = ts + kj;
            if (gk >= k_end) continue;
            unsigned char* dst = st + kj * kSlot + 16 * ch;
            if (gk < R.nsel) {
                const size_t r = seq_row0 + (size_t)list[gk];
                if (ch < 8) cp_async16(dst, a.c.kv_data + r * kKVBytes + 16 * ch);
                else if (ch == 8) cp_async16(dst, a.c.kv_scale + r * kKVScales);
            } else {
                const int64_t p = R.lo + (gk - R.nsel);
                cp_async16(dst, a.c.swa + (swa_row0 + (size_t)(p & (a.c.swa_cap - 1))) * kSWABytes + 16 * ch);
            }
        }
        cp_async_commit();
    };

    const int step = kAWarps * kTile;
    const int first = k_begin + warp * kTile;
    const int ntiles = first < k_end ? (k_end - first + step - 1) / step : 0;
#pragma unroll
    for (int i = 0; i < kStages - 1; ++i) {
        if (i < ntiles) issue(first + i * step, wbase + i * kStageBytes);
        else cp_async_commit();
    }
    for (int it = 0; it < ntiles; ++it) {
        const int pf = it + kStages - 1;
        if (pf < ntiles) issue(first + pf * step, wbase + (pf % kStages) * kStageBytes);
        else cp_async_commit();
        cp_async_wait<kStages - 1>();
        __syncwarp();
        const unsigned char* st = wbase + (it % kStages) * kStageBytes;
        const int ts = first + it * step;
        // ---- S = Q K^T : n-tile nt holds keys 8nt .. 8nt+7, this thread's key 8nt + g ----
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
            const int kj = 8 * nt + g;
            const unsigned char* slot = st + kj * kSlot;
            // A tile may hold FP4 rows and FP8 window rows side by side, so each thread builds its
            // operands for its own key and the warp-wide mma.sync is issued outside any branch.
            //   FP4 row: k-step kk uses bytes 2kk, 2kk+1 of the 16-byte slice at 16t (dims 32t..32t+31)
            //   FP8 row: k-step kk uses bytes 4kk .. 4kk+3 of the 32-byte slice at 32t
            const bool fp4 = ts + kj < R.nsel;
            const uint4 wA = *reinterpret_cast<const uint4*>(slot + (fp4 ? 16 * t : 32 * t));
            const uint4 wB = *reinterpret_cast<const uint4*>(slot + 32 * t + 16);
            const uint16_t s2 = *reinterpret_cast<const uint16_t*>(slot + 128 + 2 * t);
            const uint32_t sA = scale_h2((uint8_t)(s2 & 0xFF)), sB = scale_h2((uint8_t)(s2 >> 8));
            const uint32_t wa[4] = {wA.x, wA.y, wA.z, wA.w}, wb[4] = {wB.x, wB.y, wB.z, wB.w};
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t b0, b1;
                if (fp4) {
                    const uint32_t w = wa[kk >> 1], sq = kk < 4 ? sA : sB;
                    b0 = hmul2((kk & 1) ? e2m1x2_byte<2>(w) : e2m1x2_byte<0>(w), sq);
                    b1 = hmul2((kk & 1) ? e2m1x2_byte<3>(w) : e2m1x2_byte<1>(w), sq);
                } else {
                    const uint32_t w = kk < 4 ? wa[kk] : wb[kk - 4];
                    b0 = e4m3x2_to_h2((uint16_t)(w & 0xFFFF));
                    b1 = e4m3x2_to_h2((uint16_t)(w >> 16));
                }
                uint32_t qa[4];
                q_frag(kk, qa);
                mma16816(sc[nt], qa, b0, b1);
            }
        }
        // ---- online softmax (rows g and g+8); keys past k_end are masked ----
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const bool v = ts + nt * 8 + 2 * t + c < k_end;
                sc[nt][c] = v ? sc[nt][c] * scale2 : -INFINITY;
                sc[nt][2 + c] = v ? sc[nt][2 + c] * scale2 : -INFINITY;
                mx0 = fmaxf(mx0, sc[nt][c]);
                mx1 = fmaxf(mx1, sc[nt][2 + c]);
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
        for (int nt = 0; nt < 2; ++nt) {
            const float p0 = (mn0 == -INFINITY) ? 0.f : exp2f(sc[nt][0] - mn0);
            const float p1 = (mn0 == -INFINITY) ? 0.f : exp2f(sc[nt][1] - mn0);
            const float p2 = (mn1 == -INFINITY) ? 0.f : exp2f(sc[nt][2] - mn1);
            const float p3 = (mn1 == -INFINITY) ? 0.f : exp2f(sc[nt][3] - mn1);
            ps0 += p0 + p1;
            ps1 += p2 + p3;
            pa[2 * nt] = pack_h2(p0, p1);
            pa[2 * nt + 1] = pack_h2(p2, p3);
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
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {  // nd = 8hf .. 8hf+7
            uint32_t vw[4][2], vs[4];
            int kind[4];                  // 0: FP4 row, 1: FP8 window row, 2: past the split
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                const int kj = (kq & 1) + 2 * t + ((kq & 2) ? 8 : 0);
                const int gk = ts + kj;
                const unsigned char* slot = st + kj * kSlot;
                vw[kq][0] = vw[kq][1] = 0u;
                vs[kq] = 0u;
                if (gk < R.nsel) {
                    kind[kq] = 0;
                    vw[kq][0] = *reinterpret_cast<const uint32_t*>(slot + 64 + 8 * g + 4 * hf);
                    vs[kq] = scale_h2(slot[128 + 8 + g]);
                } else if (gk < k_end) {
                    kind[kq] = 1;
                    const uint2 w = *reinterpret_cast<const uint2*>(slot + 128 + 16 * g + 8 * hf);
                    vw[kq][0] = w.x;
                    vw[kq][1] = w.y;
                } else {
                    kind[kq] = 2;
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // dims 16g + 8hf + 2i, +1 of the four keys
                uint32_t hv[4];
#pragma unroll
                for (int kq = 0; kq < 4; ++kq) {
                    uint32_t x;
                    if (kind[kq] == 0) {
                        const uint32_t c = i == 0 ? e2m1x2_byte<0>(vw[kq][0]) : i == 1 ? e2m1x2_byte<1>(vw[kq][0])
                                         : i == 2 ? e2m1x2_byte<2>(vw[kq][0]) : e2m1x2_byte<3>(vw[kq][0]);
                        x = hmul2(c, vs[kq]);
                    } else if (kind[kq] == 1) {
                        const uint32_t w = vw[kq][i >> 1];
                        x = e4m3x2_to_h2((uint16_t)((i & 1) ? (w >> 16) : (w & 0xFFFF)));
                    } else {
                        x = 0u;
                    }
                    hv[kq] = x;
                }
                // n-tile nd = 8hf + 2i (low halves) and 8hf + 2i + 1 (high halves)
                mma16816(o[8 * hf + 2 * i], pa, prmt(hv[0], hv[1], 0x5410), prmt(hv[2], hv[3], 0x5410));
                mma16816(o[8 * hf + 2 * i + 1], pa, prmt(hv[0], hv[1], 0x7632), prmt(hv[2], hv[3], 0x7632));
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    // ---- combine the 4 warps (and splits) ----
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    __syncthreads();
    // O staging: head h, dim d = 32 c + j at h * kCoRow + 33 c + j (conflict-free for both patterns)
    constexpr int kCoRow = 132;
    float* cm = reinterpret_cast<float*>(smem);              // [4][16] m
    float* cl = cm + kAWarps * kHQ;                          // [4][16] l
    float* co = cl + kAWarps * kHQ;                          // [4][16][kCoRow] O
    {
        if (t == 0) {
            cm[warp * kHQ + g] = m0; cm[warp * kHQ + g + 8] = m1;
            cl[warp * kHQ + g] = l0; cl[warp * kHQ + g + 8] = l1;
        }
        // o[nd][0..1] -> head g, dims 32t + nd and 32t + 16 + nd; o[nd][2..3] -> head g + 8
        float* ow = co + warp * kHQ * kCoRow;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
            ow[g * kCoRow + 33 * t + nd] = o[nd][0];
            ow[g * kCoRow + 33 * t + 16 + nd] = o[nd][1];
            ow[(g + 8) * kCoRow + 33 * t + nd] = o[nd][2];
            ow[(g + 8) * kCoRow + 33 * t + 16 + nd] = o[nd][3];
        }
    }
    __syncthreads();
    const int splits = a.plan.splits;
    float* part = reinterpret_cast<float*>(a.ws + a.L.att_part) + ((size_t)row * splits) * kHQ * kPartStride;
    // thread -> (head h, 8 dims)
    const int h = tid >> 4, d0 = (tid & 15) * 8;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w) M = fmaxf(M, cm[w * kHQ + h]);
    float Lsum = 0.f, acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w) {
        const float mw = cm[w * kHQ + h];
        const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        Lsum += f * cl[w * kHQ + h];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += f * co[(w * kHQ + h) * kCoRow + 33 * (d0 >> 5) + (d0 & 31) + j];
    }
    if (splits > 1) {
        float* pp = part + ((size_t)split * kHQ + h) * kPartStride;
#pragma unroll
        for (int j = 0; j < 8; ++j) pp[d0 + j] = acc[j];
        if ((tid & 15) == 0) { pp[kD] = M; pp[kD + 1] = Lsum; }
        __threadfence();
        __syncthreads();
        unsigned int* tk = reinterpret_cast<unsigned int*>(a.ws + a.L.att_ticket) + row;
        if (tid == 0) s_last = (atomicAdd(tk, 1u) == (unsigned)splits - 1);
        __syncthreads();
        if (!s_last) return;
        __threadfence();
        // the other splits' partials, read from L2 (they were written by other CTAs); this split's
        // own partial is still in registers
        const float M_own = M, L_own = Lsum;
        float acc_own[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) { acc_own[j] = acc[j]; acc[j] = 0.f; }
        M = M_own;
        for (int sp = 0; sp < splits; ++sp)
            if (sp != split) M = fmaxf(M, __ldcg(part + ((size_t)sp * kHQ + h) * kPartStride + kD));
        {
            const float f = (M_own == -INFINITY) ? 0.f : exp2f(M_own - M);
            Lsum = f * L_own;
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = f * acc_own[j];
        }
        for (int sp = 0; sp < splits; ++sp) {
            if (sp == split) continue;
            const float* q = part + ((size_t)sp * kHQ + h) * kPartStride;
            const float4 v0 = __ldcg(reinterpret_cast<const float4*>(q + d0));
            const float4 v1 = __ldcg(reinterpret_cast<const float4*>(q + d0 + 4));
            const float mw = __ldcg(q + kD), lw = __ldcg(q + kD + 1);
            const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
            Lsum += f * lw;
            acc[0] += f * v0.x; acc[1] += f * v0.y; acc[2] += f * v0.z; acc[3] += f * v0.w;
            acc[4] += f * v1.x; acc[5] += f * v1.y; acc[6] += f * v1.z; acc[7] += f * v1.w;
        }
        if (tid == 0) *tk = 0;
    }
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

size_t attend_smem_bytes(int k) { return (size_t)kAWarps * kWarpSmem + kQBytes + 4 * (size_t)k; }

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s) {
    const size_t smem = attend_smem_bytes(a.k);
    cudaError_t e = cudaFuncSetAttribute(attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (a.rows == 0) return cudaSuccess;
    dim3 grid(a.rows, a.plan.splits);
    return launch_after_prior(attend_kernel, grid, dim3(kAThreads), smem, s, a);
}

}  // namespace csa2
