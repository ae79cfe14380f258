// latent_index.cu -- the indexer of the pages' own shape: hi query heads x 128 channels over ONE
// shared 128-channel MXFP4 key per entry, exact scores and Top-k.
//
// [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token", sec. VII: the
// indexer key is MXFP4 (E2M1 elements, one E8M0 scale per 32 channels, 68 B per entry); the
// configuration list: 32 indexer query heads of dimension 128. [B] "DeepSeek Cuts KV Cache
// Footprint Fourfold", "Technical Approach", and [C] sec. VI: a query keeps the Top-k of the entries
// visible to it by index score.
// Reading taken here: score(p) = sum over heads h of q_h . k_p (the ReLU variant sums
// max(0, q_h . k_p)), the query quantised with the key's MXFP4 rule; ranking by score descending,
// ties to the lower position; the selection emitted in ascending position order, padded with -1.
//
// Exactness. Twice an E2M1 value is an integer of magnitude at most 12, so the dot of a query
// head and a key over one 32-channel block is an exact integer I (|I| <= 4608; dp4a over int8)
// times the product of the two blocks' scales, a power of two. A head's dot is the sum of its 4
// such terms in fp64, and the score the sum of the heads' dots in fp64: every term is exact, and
// so is every sum as long as the exponents within a row's sums span fewer than about 38 bits. That
// holds for any query and keys whose 32-channel block maxima lie within 2^38 of each other, which
// covers the workloads by a wide margin. The scores then are the exact rational scores (times 4),
// and so is the ranking.
//
// lat_index_score_kernel: one thread per (row, visible position); the row's quantised query sits
//   in shared memory as int8 words and fp64 block scales; the position's 64 code bytes become 32
//   int8 words in registers. Writes the orderable 64-bit key of each score.
// lat_index_select_kernel: one CTA per row; an exact radix select (eight 8-bit digits, most
//   significant first, warp-aggregated shared-memory counts) finds the k-th largest key T and how
//   many keys equal to T are taken; an ordered compaction (block prefix sums over the positions in
//   ascending order) then writes the positions with a key above T and the lowest positions with a
//   key equal to T.
#include "csa2_internal.cuh"

namespace csa2 {

namespace {

constexpr int kSThr = 256;   // score kernel
constexpr int kQThr = 1024;  // select kernel

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// four E2M1 codes (the low 16 bits: code j in nibble j) -> four int8 of twice their values
__device__ __forceinline__ uint32_t e2m1x4_to_i8x4(uint32_t codes) {
    uint32_t r = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t c = (codes >> (4 * j)) & 0xFu;
        // twice the magnitudes of the E2M1 codes 0..7 are 0, 1, 2, 3, 4, 6, 8, 12
        const uint32_t mag = prmt(0x03020100u, 0x0C080604u, c & 7u) & 0xFFu;
        r |= ((c & 8u) ? ((0u - mag) & 0xFFu) : mag) << (8 * j);
    }
    return r;
}

// entries visible to a row at token qpos (0 for qpos < 0; -1 when the last one is past the cache
// or the workspace's bound)
__device__ __forceinline__ int64_t lat_visible(const LatIndexArgs& a, int row) {
    const int64_t qpos = a.qpos[row];
    if (qpos < 0) return 0;
    const int64_t n = (qpos + 1) / a.ratio;
    if (n > a.c.cap || n > a.max_ctx) return -1;
    return n;
}

__global__ void __launch_bounds__(kSThr) lat_index_score_kernel(LatIndexArgs a) {
    __shared__ uint32_t qw[kLatMaxHI][32];  // twice the quantised query, int8 x 4 per word
    __shared__ double qs[kLatMaxHI][4];     // its block scales
    const int row = blockIdx.y, tid = threadIdx.x;
    wait_prior_grid();  // the quantised query comes from the kernel before
    const int64_t n = lat_visible(a, row);
    if (n < 0) {
        if (blockIdx.x == 0 && tid == 0) set_status(a.status, CSA2_DEV_BAD_POS);
        return;
    }
    if ((int64_t)blockIdx.x * kSThr >= n) return;
    const int hi = a.hi;
    const uint8_t* qc = a.qcodes + (size_t)row * hi * kLatKBytes;
    const uint8_t* qsb = a.qscales + (size_t)row * hi * kLatKScales;
    for (int i = tid; i < hi * 32; i += kSThr) {
        const int h = i >> 5, w = i & 31;  // word w: channels 4w .. 4w + 3, code bytes 2w, 2w + 1
        const uint32_t codes = (uint32_t)qc[h * kLatKBytes + 2 * w] | ((uint32_t)qc[h * kLatKBytes + 2 * w + 1] << 8);
        qw[h][w] = e2m1x4_to_i8x4(codes);
    }
    for (int i = tid; i < hi * 4; i += kSThr) qs[i >> 2][i & 3] = ldexp(1.0, (int)qsb[i] - 127);
    __syncthreads();
    const int64_t p = (int64_t)blockIdx.x * kSThr + tid;
    if (p >= n) return;
    const int b = row / a.tq;
    const size_t e = (size_t)b * a.c.cap + (size_t)p;
    uint32_t kw[32];
    {
        const uint4* src = reinterpret_cast<const uint4*>(a.c.k_data + e * kLatKBytes);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = __ldg(src + i);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                kw[8 * i + 2 * j] = e2m1x4_to_i8x4(w4[j] & 0xFFFFu);
                kw[8 * i + 2 * j + 1] = e2m1x4_to_i8x4(w4[j] >> 16);
            }
        }
    }
    const uint32_t ksw = __ldg(reinterpret_cast<const uint32_t*>(a.c.k_scale + e * kLatKScales));
    double ks[4];
#pragma unroll
    for (int bk = 0; bk < 4; ++bk) ks[bk] = ldexp(1.0, (int)((ksw >> (8 * bk)) & 0xFFu) - 127);
    const bool relu = (a.flags & CSA2_SCORE_RELU) != 0;
    double total = 0.0;
    for (int h = 0; h < hi; ++h) {
        double dot = 0.0;
#pragma unroll
        for (int bk = 0; bk < 4; ++bk) {
            int I = 0;
#pragma unroll
            for (int w = 0; w < 8; ++w) I = __dp4a((int)qw[h][8 * bk + w], (int)kw[8 * bk + w], I);
            dot += (double)I * (qs[h][bk] * ks[bk]);  // exact: a 13-bit integer times a power of two
        }
        total += (relu && dot < 0.0) ? 0.0 : dot;
    }
    a.keys[(size_t)row * a.key_stride + p] = score_key(total);
}

// exclusive prefix sum of a 0/1 flag over the CTA in thread order; *total receives the sum
__device__ __forceinline__ int block_scan(bool f, int* wsum, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned int bal = __ballot_sync(0xffffffffu, f);
    const int in_warp = __popc(bal & ((1u << lane) - 1u));
    __syncthreads();
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
        const int v = wsum[lane];
        int s = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, s, d);
            if (lane >= d) s += t;
        }
        wsum[lane] = s - v;  // exclusive
        if (lane == 31) wsum[32] = s;
    }
    __syncthreads();
    *total = wsum[32];
    return wsum[warp] + in_warp;
}

__global__ void __launch_bounds__(kQThr) lat_index_select_kernel(LatIndexArgs a) {
    __shared__ unsigned int hist[256];
    __shared__ int wsum[33];
    __shared__ int s_digit, s_rem;
    const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    wait_prior_grid();  // the keys come from the score kernel
    const int K = a.k;
    int32_t* out = a.out_idx + (size_t)row * K;
    const int64_t n = lat_visible(a, row);
    if (n <= (int64_t)K) {  // every visible entry (none for an invalid row), then -1
        for (int i = tid; i < K; i += kQThr) out[i] = (int64_t)i < n ? i : -1;
        return;
    }
    const unsigned long long* keys = a.keys + (size_t)row * a.key_stride;
    unsigned long long prefix = 0ull, mask = 0ull;
    int rem = K;  // keys still to take among those matching the prefix
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kQThr) hist[i] = 0u;
        __syncthreads();
        for (int64_t p0 = 0; p0 < n; p0 += kQThr) {
            const int64_t p = p0 + tid;
            int d = -1;
            if (p < n) {
                const unsigned long long key = keys[p];
                if ((key & mask) == prefix) d = (int)((key >> shift) & 0xFFull);
            }
            // one shared-memory add per distinct digit of the warp
            const unsigned int peers = __match_any_sync(0xffffffffu, d);
            if (d >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (unsigned)__popc(peers));
        }
        __syncthreads();
        if (tid == 0) {
            int acc = 0, d = 255;
            while (d > 0 && acc + (int)hist[d] < rem) acc += (int)hist[d--];
            s_digit = d;
            s_rem = rem - acc;
        }
        __syncthreads();
        prefix |= (unsigned long long)s_digit << shift;
        mask |= 0xFFull << shift;
        rem = s_rem;
        __syncthreads();  // s_digit / s_rem are rewritten by the next digit
    }
    // prefix is the k-th largest key T; rem keys equal to T are taken, the lowest positions first
    const unsigned long long T = prefix;
    int written = 0, eq_seen = 0;
    for (int64_t p0 = 0; p0 < n; p0 += kQThr) {
        const int64_t p = p0 + tid;
        const unsigned long long key = p < n ? keys[p] : 0ull;
        const bool eq = p < n && key == T;
        int eq_total;
        const int eq_rank = eq_seen + block_scan(eq, wsum, &eq_total);
        const bool sel = p < n && (key > T || (eq && eq_rank < rem));
        int sel_total;
        const int r = written + block_scan(sel, wsum, &sel_total);
        if (sel) out[r] = (int32_t)p;
        written += sel_total;
        eq_seen += eq_total;
    }
}

}  // namespace

size_t latent_index_ws_bytes(int rows, int hi, int64_t max_ctx) {
    size_t off = 256;                                                   // status word
    off += align256((size_t)rows * hi * kLatKBytes);                    // quantised query codes
    off += align256((size_t)rows * hi * kLatKScales);                   // their E8M0 scales
    off += align256((size_t)rows * (size_t)max_ctx * sizeof(uint64_t));  // keys
    return off;
}

cudaError_t launch_latent_index(LatIndexArgs a, const uint16_t* idx_q, unsigned char* ws, cudaStream_t s) {
    size_t off = 256;
    a.status = reinterpret_cast<uint32_t*>(ws);
    uint8_t* qcodes = ws + off;
    off += align256((size_t)a.rows * a.hi * kLatKBytes);
    uint8_t* qscales = ws + off;
    off += align256((size_t)a.rows * a.hi * kLatKScales);
    a.qcodes = qcodes;
    a.qscales = qscales;
    a.keys = reinterpret_cast<unsigned long long*>(ws + off);
    a.key_stride = a.max_ctx;
    if (a.rows == 0) return cudaSuccess;
    cudaError_t e = launch_mxfp4(idx_q, (long long)a.rows * a.hi, 128, qcodes, qscales, s);
    if (e != cudaSuccess) return e;
    const long long bx = (a.max_ctx + kSThr - 1) / kSThr;
    e = launch_after_prior(lat_index_score_kernel, dim3((unsigned)bx, (unsigned)a.rows), dim3(kSThr), 0, s, a);
    if (e != cudaSuccess) return e;
    return launch_after_prior(lat_index_select_kernel, dim3((unsigned)a.rows), dim3(kQThr), 0, s, a);
}

}  // namespace csa2
