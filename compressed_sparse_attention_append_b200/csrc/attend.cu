// attend.cu -- fused gather / dequantise / sparse softmax attention with split-K.
//
// [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token":
//   sec. VI "What one layer looks like": the layer's own query attends to the selected entries of
//   the shared main KV plus its own recent window;
//   sec. XI: cached values are dequantised before attention (E2M1 x E4M3 products are exact in
//   fp16, and FP8 window values are exact in fp16, so the dequantised keys and values are exact);
//   sec. XII: a query at position i sees window keys [max(s, i - win + 1), i].
// This build's reading: one softmax over selected and window keys together, 16 query heads
// sharing one K/V head, default scale 1/sqrt(128).
//
// Per CTA: one query row and one split of its key list (selected entries in index order, then the
// window). Four warps each own 16-key tiles: rows are gathered with cp.async into a warp-private
// double-buffered stage, dequantised to fp16 in shared memory (16-byte chunks XOR-swizzled for
// conflict-free ldmatrix), and multiplied on the tensor cores with mma.sync m16n8k16 (fp16 in, fp32
// accumulate): S = Q K^T with the 16 heads as the M dimension, then O += P V with P rounded to fp16.
// The four warps' (m, l, O) are merged in shared memory; with several splits per row the partial
// results go to the workspace and the CTA that finishes a row's last split combines them.
//
// Precision: Q is converted bf16 -> fp16 (exact for |q| >= 2^-14; smaller magnitudes round to fp16
// subnormals, an absolute error below 2^-25); P is rounded to fp16 (relative 2^-11); all sums are
// fp32.
#include "csa2_internal.cuh"

namespace csa2 {

namespace {

constexpr int kAThreads = 128;
constexpr int kAWarps = 4;
constexpr int kTile = 16;                    // keys per warp step
constexpr int kStageBytes = kTile * 256;     // raw rows (main 144 B or window 256 B, 256 B slots)
constexpr int kWarpSmem = 2 * kStageBytes + 2 * kTile * 256;  // 2 stages + fp16 K and V tiles

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

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(p);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(s));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(p);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(s));
}

// fp16 tile [16 keys][128 dims], row = 256 B = 16 chunks of 16 B, chunk c stored at c ^ (key & 7)
__device__ __forceinline__ int swz(int key, int chunk) { return key * 256 + ((chunk ^ (key & 7)) << 4); }

struct RowKeys {
    int nsel, nwin, nk;
    int64_t lo, qpos;
    int b;
};

__global__ void __launch_bounds__(kAThreads) attend_kernel(AttendArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int s_cnt[kAThreads];
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = blockIdx.x, split = blockIdx.y;
    const int K = a.k;
    uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + kHdrStatus);
    int* list = reinterpret_cast<int*>(smem + kAWarps * kWarpSmem);

    RowKeys R;
    R.b = row / a.tq;
    R.qpos = a.qpos ? a.qpos[row] : a.qpos_base + row % a.tq;
    const bool row_ok = R.qpos >= 0 && R.qpos < a.c.cap;
    // ---- deterministic compaction of the valid selected indices (index order) ----
    {
        const int32_t* idx = a.idx + (size_t)row * K;
        const int per = (K + kAThreads - 1) / kAThreads;
        const int i0 = tid * per, i1 = min(i0 + per, K);
        int c = 0;
        for (int i = i0; i < i1; ++i) {
            const int v = idx[i];
            const bool ok = v >= 0 && v <= R.qpos && (int64_t)v < a.c.cap && row_ok;
            if (!ok && v != -1 && split == 0) set_status(status, CSA2_DEV_BAD_INDEX);
            c += ok;
        }
        s_cnt[tid] = c;
        __syncthreads();
        // exclusive scan over 128 counts (warp 0)
        if (warp == 0) {
            int v[4], sum = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) { v[j] = s_cnt[lane * 4 + j]; sum += v[j]; }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            int run = incl - sum;
#pragma unroll
            for (int j = 0; j < 4; ++j) { const int t = v[j]; s_cnt[lane * 4 + j] = run; run += t; }
            if (lane == 31) s_last = incl;
        }
        __syncthreads();
        int o = s_cnt[tid];
        for (int i = i0; i < i1; ++i) {
            const int v = idx[i];
            if (v >= 0 && v <= R.qpos && (int64_t)v < a.c.cap && row_ok) list[o++] = v;
        }
        R.nsel = s_last;
    }
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

    // ---- Q fragments (fp16), A operand of m16n8k16: rows = heads ----
    uint32_t qa[8][4];
    {
        const uint16_t* q = a.q + (size_t)row * (kHQ * kD);
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int h = g + ((r & 1) ? 8 : 0);
                const int d = kk * 16 + 2 * t + ((r & 2) ? 8 : 0);
                const uint32_t w = *reinterpret_cast<const uint32_t*>(q + h * kD + d);
                qa[kk][r] = pack_h2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
            }
        }
    }

    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    unsigned char* wbase = smem + warp * kWarpSmem;
    unsigned char* stage[2] = {wbase, wbase + kStageBytes};
    unsigned char* kt = wbase + 2 * kStageBytes;
    unsigned char* vt = kt + kTile * 256;

    const size_t seq_row0 = (size_t)R.b * a.c.cap;
    const size_t swa_row0 = (size_t)R.b * a.c.swa_cap;
    auto issue = [&](int tile_start, unsigned char* st) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int slot = lane + 32 * i;
            const int kj = slot >> 4, ch = slot & 15;
            const int gk = tile_start + kj;
            if (gk >= k_end) continue;
            unsigned char* dst = st + kj * 256 + ch * 16;
            if (gk < R.nsel) {
                const size_t r = seq_row0 + (size_t)list[gk];
                if (ch < 8) cp_async16(dst, a.c.kv_data + r * kKVBytes + ch * 16);
                else if (ch == 8) cp_async16(dst, a.c.kv_scale + r * kKVScales);
            } else {
                const int64_t p = R.lo + (gk - R.nsel);
                const size_t r = swa_row0 + (size_t)(p & (a.c.swa_cap - 1));
                cp_async16(dst, a.c.swa + r * kSWABytes + ch * 16);
            }
        }
        cp_async_commit();
    };

    const int first = k_begin + warp * kTile;
    if (first < k_end) issue(first, stage[0]);
    int it = 0;
    for (int ts = first; ts < k_end; ts += kAWarps * kTile, ++it) {
        const int nts = ts + kAWarps * kTile;
        if (nts < k_end) {
            issue(nts, stage[(it + 1) & 1]);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
        // ---- dequantise: lane -> key lane>>1, half lane&1 (0 = K dims, 1 = V dims) ----
        {
            const unsigned char* st = stage[it & 1];
            const int kj = lane >> 1, half = lane & 1;
            const int gk = ts + kj;
            unsigned char* dstt = half ? vt : kt;
            if (gk < k_end && gk < R.nsel) {
                const unsigned char* src = st + kj * 256;
                const uint2 scl = *reinterpret_cast<const uint2*>(src + 128 + 8 * half);
                const uint32_t sw[2] = {scl.x, scl.y};
#pragma unroll
                for (int blk = 0; blk < 8; ++blk) {
                    const uint2 c = *reinterpret_cast<const uint2*>(src + 64 * half + 8 * blk);
                    const uint8_t sb = (uint8_t)(sw[blk >> 2] >> (8 * (blk & 3)));
                    const uint32_t s2 = e4m3x2_to_h2((uint16_t)(sb | (sb << 8)));
                    uint32_t h0[4], h1[4];
                    e2m1x8_to_h2x4(c.x, h0);
                    e2m1x8_to_h2x4(c.y, h1);
                    uint4 v0 = make_uint4(hmul2(h0[0], s2), hmul2(h0[1], s2), hmul2(h0[2], s2), hmul2(h0[3], s2));
                    uint4 v1 = make_uint4(hmul2(h1[0], s2), hmul2(h1[1], s2), hmul2(h1[2], s2), hmul2(h1[3], s2));
                    *reinterpret_cast<uint4*>(dstt + swz(kj, 2 * blk)) = v0;
                    *reinterpret_cast<uint4*>(dstt + swz(kj, 2 * blk + 1)) = v1;
                }
            } else if (gk < k_end) {
                const unsigned char* src = st + kj * 256 + 128 * half;
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {
                    const uint4 raw = *reinterpret_cast<const uint4*>(src + 16 * c16);
                    const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
                    uint32_t hv[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        hv[2 * j] = e4m3x2_to_h2((uint16_t)(rw[j] & 0xFFFF));
                        hv[2 * j + 1] = e4m3x2_to_h2((uint16_t)(rw[j] >> 16));
                    }
                    *reinterpret_cast<uint4*>(dstt + swz(kj, 2 * c16)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                    *reinterpret_cast<uint4*>(dstt + swz(kj, 2 * c16 + 1)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
                }
            } else {
                const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4*>(dstt + swz(kj, c)) = z;
            }
        }
        __syncwarp();
        // ---- S = Q K^T : 2 n-tiles of 8 keys ----
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
            for (int kp = 0; kp < 4; ++kp) {
                uint32_t b[4];
                const int key = nt * 8 + (lane & 7);
                const int chunk = 4 * kp + (lane >> 3);
                ldsm_x4(b, kt + swz(key, chunk));
                mma16816(sc[nt], qa[2 * kp], b[0], b[1]);
                mma16816(sc[nt], qa[2 * kp + 1], b[2], b[3]);
            }
        }
        // ---- online softmax (rows g and g+8) ----
        const int t = lane & 3;
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int gk = ts + nt * 8 + 2 * t + c;
                const bool v = gk < k_end;
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
#pragma unroll
        for (int i = 0; i < 16; ++i) { o[i][0] *= al0; o[i][1] *= al0; o[i][2] *= al1; o[i][3] *= al1; }
        // ---- O += P V : 16 n-tiles of 8 dims ----
#pragma unroll
        for (int np = 0; np < 8; ++np) {
            uint32_t b[4];
            const int mi = lane >> 3;
            const int key = (mi & 1) * 8 + (lane & 7);
            const int chunk = 2 * np + (mi >> 1);
            ldsm_x4_t(b, vt + swz(key, chunk));
            mma16816(o[2 * np], pa, b[0], b[1]);
            mma16816(o[2 * np + 1], pa, b[2], b[3]);
        }
        __syncwarp();
    }
    // ---- combine the 4 warps (and splits) ----
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    __syncthreads();
    float* cm = reinterpret_cast<float*>(smem);              // [4][16] m
    float* cl = cm + kAWarps * kHQ;                          // [4][16] l
    float* co = cl + kAWarps * kHQ;                          // [4][16][128] O
    {
        const int g = lane >> 2, t = lane & 3;
        if (t == 0) {
            cm[warp * kHQ + g] = m0; cm[warp * kHQ + g + 8] = m1;
            cl[warp * kHQ + g] = l0; cl[warp * kHQ + g + 8] = l1;
        }
        float* ow = co + warp * kHQ * kD;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
            const int d = nd * 8 + 2 * t;
            *reinterpret_cast<float2*>(ow + g * kD + d) = make_float2(o[nd][0], o[nd][1]);
            *reinterpret_cast<float2*>(ow + (g + 8) * kD + d) = make_float2(o[nd][2], o[nd][3]);
        }
    }
    __syncthreads();
    const int splits = a.plan.splits;
    float* part = reinterpret_cast<float*>(a.ws + a.L.att_part) + ((size_t)row * splits) * kHQ * (kD + 2);
    // thread -> (head h, 16 dims)
    const int h = tid >> 3, d0 = (tid & 7) * 16;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w) M = fmaxf(M, cm[w * kHQ + h]);
    float Lsum = 0.f, acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w) {
        const float mw = cm[w * kHQ + h];
        const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        Lsum += f * cl[w * kHQ + h];
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] += f * co[(w * kHQ + h) * kD + d0 + j];
    }
    if (splits > 1) {
        float* pp = part + ((size_t)split * kHQ + h) * (kD + 2);
#pragma unroll
        for (int j = 0; j < 16; ++j) pp[d0 + j] = acc[j];
        if ((tid & 7) == 0) { pp[kD] = M; pp[kD + 1] = Lsum; }
        __threadfence();
        __syncthreads();
        unsigned int* tk = reinterpret_cast<unsigned int*>(a.ws + a.L.att_ticket) + row;
        if (tid == 0) s_last = (atomicAdd(tk, 1u) == (unsigned)splits - 1);
        __syncthreads();
        if (!s_last) return;
        __threadfence();
        M = -INFINITY;
        for (int sp = 0; sp < splits; ++sp) M = fmaxf(M, ((volatile float*)part)[((size_t)sp * kHQ + h) * (kD + 2) + kD]);
        Lsum = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] = 0.f;
        for (int sp = 0; sp < splits; ++sp) {
            const volatile float* q = part + ((size_t)sp * kHQ + h) * (kD + 2);
            const float mw = q[kD];
            const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
            Lsum += f * q[kD + 1];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] += f * q[d0 + j];
        }
        if (tid == 0) *tk = 0;
    }
    const bool empty = (M == -INFINITY) || !(Lsum > 0.f);
    const float inv = empty ? 0.f : 1.f / Lsum;
    const size_t ob = ((size_t)row * kHQ + h) * kD + d0;
    uint32_t pk[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float x0 = acc[2 * j] * inv, x1 = acc[2 * j + 1] * inv;
        __nv_bfloat162 bb = __floats2bfloat162_rn(x0, x1);
        pk[j] = *reinterpret_cast<uint32_t*>(&bb);
        if (a.out_f32) *reinterpret_cast<float2*>(a.out_f32 + ob + 2 * j) = make_float2(x0, x1);
    }
    *reinterpret_cast<uint4*>(a.out + ob) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    *reinterpret_cast<uint4*>(a.out + ob + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    if (a.lse && (tid & 7) == 0)
        a.lse[(size_t)row * kHQ + h] = empty ? -INFINITY : (M * 0.6931471805599453f + logf(Lsum));
}

}  // namespace

size_t attend_smem_bytes(int k) { return (size_t)kAWarps * kWarpSmem + 4 * (size_t)k + 64; }

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s) {
    const size_t smem = attend_smem_bytes(a.k);
    cudaError_t e = cudaFuncSetAttribute(attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (a.rows == 0) return cudaSuccess;
    dim3 grid(a.rows, a.plan.splits);
    attend_kernel<<<grid, kAThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace csa2
