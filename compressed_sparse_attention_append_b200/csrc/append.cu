// append.cu -- quantise-append of new tokens into the FP4 cache planes and the FP8 window ring.
//
// [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token", sec. XI:
// E2M1 elements with one E4M3 scale per 16 channels and no scale for the whole tensor on top,
// quantised after RoPE; the sliding-window KV stays at FP8. [B] "DeepSeek Cuts KV Cache Footprint
// Fourfold", "Technical Approach": only Full mode writes main KV and indexer keys; every mode
// writes its own sliding-window KV.
//
// Rounding (the reading taken here of a rule the pages leave open): s = E4M3_RNE_satfinite(amax / 6) in fp32,
// all-zero codes when s == 0, code = E2M1_RNE_satfinite(x / s) with the sign of x kept.
// The quotients are IEEE fp32 divisions; because x has 8 significant bits and s has 4, an fp32
// quotient can never fall between a rounding boundary and the exact quotient, so these
// decisions equal those taken on exact rationals.
//
// Work split: one thread per 16-channel block. A token has 16 main blocks, hk*4 = 16 indexer
// blocks and 16 window groups of 16 channels; 48 threads per token. The latent cache of the pages'
// own shape (latent_append_kernel) takes 68 threads per token, and the MXFP4 codec one thread per
// 32-channel block.
#include "csa2_internal.cuh"

namespace csa2 {

namespace {

__global__ void __launch_bounds__(192) append_kernel(AppendArgs a) {
    // the slots written here may still be read by the previous step's attention (the window ring)
    wait_prior_grid();
    const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long ntok = (long long)a.batch * a.t;
    if (id >= ntok * 48) return;
    const long long tok = id / 48;
    const int task = (int)(id % 48);
    const int b = (int)(tok / a.t);
    const int i = (int)(tok % a.t);
    const int64_t p0 = a.pos ? a.pos[b] : a.pos_host;
    const int64_t p = p0 + i;
    if (task < 32) {
        if (p0 < 0 || p0 + a.t > a.c.cap) {
            if (task == 0 && i == 0) set_status(a.status, CSA2_DEV_BAD_POS);
            return;
        }
        const bool main = task < 16;
        const uint16_t* src = main ? a.kv : a.idx_k;
        if (!src) return;
        const int blk = main ? task : task - 16;
        float x[16];
        load16_bf16(src + tok * 256 + blk * 16, x);
        uint2 codes;
        uint8_t sc;
        quantize_block(x, codes, sc);
        const size_t row = (size_t)b * a.c.cap + p;
        uint8_t* dst = main ? a.c.kv_data : a.c.ik_data;
        uint8_t* sdst = main ? a.c.kv_scale : a.c.ik_scale;
        *reinterpret_cast<uint2*>(dst + row * 128 + blk * 8) = codes;
        sdst[row * 16 + blk] = sc;
    } else {
        if (!a.swa_kv) return;
        if (p0 < 0) {
            if (task == 32 && i == 0) set_status(a.status, CSA2_DEV_BAD_POS);
            return;
        }
        // the ring keeps the latest swa_cap positions: older tokens of this call would share a
        // slot with a newer one, so they are not written
        if ((int64_t)i < (int64_t)a.t - a.c.swa_cap) return;
        const int g = task - 32;
        float x[16];
        load16_bf16(a.swa_kv + tok * 256 + g * 16, x);
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            w[j] = f32x2_to_e4m3x2(x[4 * j], x[4 * j + 1]) | (f32x2_to_e4m3x2(x[4 * j + 2], x[4 * j + 3]) << 16);
        const size_t slot = (size_t)b * a.c.swa_cap + (size_t)(p & (a.c.swa_cap - 1));
        *reinterpret_cast<uint4*>(a.c.swa + slot * 256 + g * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// One MXFP4 block ([C] sec. VII): 32 bf16 channels -> 16 code bytes and the E8M0 byte.
// X = 2^(floor(log2 amax) - 2), byte log2 X + 127 clamped to 0..254; x / X is exact (a power-of-two
// scale), so the hardware E2M1 conversion of the fp32 quotient decides each code as an exact
// rational would.
__device__ __forceinline__ void mx_block(const uint16_t* x, uint4& codes, uint8_t& sbyte) {
    const uint4* src = reinterpret_cast<const uint4*>(x);
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 v = __ldg(src + i);
        w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
        amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
    }
    int sb = 0;
    if (amax > 0.f) {
        sb = ilogbf(amax) - 2 + 127;  // floor(log2 amax), subnormals included
        sb = sb < 0 ? 0 : (sb > 254 ? 254 : sb);
    }
    uint32_t c[4] = {0u, 0u, 0u, 0u};
    if (amax > 0.f) {
        const float X = ldexpf(1.0f, sb - 127);  // 2^-127 .. 2^127, exact in fp32
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float lo = __fdiv_rn(__uint_as_float(w[i] << 16), X);
            const float hi = __fdiv_rn(__uint_as_float(w[i] & 0xFFFF0000u), X);
            c[i >> 2] |= f32x2_to_e2m1x2(lo, hi) << (8 * (i & 3));
        }
    }
    codes = make_uint4(c[0], c[1], c[2], c[3]);
    sbyte = (uint8_t)sb;
}

// MXFP4 rows: one thread per 32-channel block.
__global__ void __launch_bounds__(256) mxfp4_kernel(const uint16_t* x, long long blocks, int nb, uint8_t* data,
                                                    uint8_t* scale) {
    const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= blocks) return;
    uint4 codes;
    uint8_t sb;
    mx_block(x + id * 32, codes, sb);
    *reinterpret_cast<uint4*>(data + id * 16) = codes;
    scale[id] = sb;
}

// Append into the latent cache of the pages' own shape ([C] sec. VII, XI). Per token: 32 tasks of
// one 16-channel latent block (E2M1 + E4M3 scale, the rule of quantize_block), 4 tasks of one
// 32-channel MXFP4 block of the indexer key, and 32 tasks of 16 window channels (E4M3).
constexpr int kLatTasks = 32 + 4 + 32;

__global__ void __launch_bounds__(256) latent_append_kernel(LatentAppendArgs a) {
    wait_prior_grid();  // the window slots may still be read by earlier attention on the stream
    const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long ntok = (long long)a.batch * a.t;
    if (id >= ntok * kLatTasks) return;
    const long long tok = id / kLatTasks;
    const int task = (int)(id % kLatTasks);
    const int b = (int)(tok / a.t);
    const int i = (int)(tok % a.t);
    const int64_t p0 = a.pos[b];
    const int64_t p = p0 + i;
    if (task < 36) {
        if (p0 < 0 || p0 + a.t > a.c.cap) {
            if (task == 0 && i == 0 && (a.latent || a.idx_k)) set_status(a.status, CSA2_DEV_BAD_POS);
            return;
        }
        const size_t row = (size_t)b * a.c.cap + p;
        if (task < 32) {
            if (!a.latent) return;
            float x[16];
            load16_bf16(a.latent + tok * kLatD + task * 16, x);
            uint2 codes;
            uint8_t sc;
            quantize_block(x, codes, sc);
            *reinterpret_cast<uint2*>(a.c.l_data + row * kLatBytes + task * 8) = codes;
            a.c.l_scale[row * kLatScales + task] = sc;
        } else {
            if (!a.idx_k) return;
            const int blk = task - 32;
            uint4 codes;
            uint8_t sb;
            mx_block(a.idx_k + tok * 128 + blk * 32, codes, sb);
            *reinterpret_cast<uint4*>(a.c.k_data + row * kLatKBytes + blk * 16) = codes;
            a.c.k_scale[row * kLatKScales + blk] = sb;
        }
    } else {
        if (!a.swa) return;
        if (p0 < 0) {
            if (task == 36 && i == 0) set_status(a.status, CSA2_DEV_BAD_POS);
            return;
        }
        // older tokens of this call that would share a ring slot with a newer one are not written
        if ((int64_t)i < (int64_t)a.t - a.c.swa_cap) return;
        const int g = task - 36;
        float x[16];
        load16_bf16(a.swa + tok * kLatD + g * 16, x);
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            w[j] = f32x2_to_e4m3x2(x[4 * j], x[4 * j + 1]) | (f32x2_to_e4m3x2(x[4 * j + 2], x[4 * j + 3]) << 16);
        const size_t slot = (size_t)b * a.c.swa_cap + (size_t)(p & (a.c.swa_cap - 1));
        *reinterpret_cast<uint4*>(a.c.swa + slot * kLatSwa + g * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace

cudaError_t launch_mxfp4(const uint16_t* x, long long rows, int channels, uint8_t* data, uint8_t* scale,
                         cudaStream_t s) {
    const long long blocks = rows * (channels / 32);
    if (blocks == 0) return cudaSuccess;
    mxfp4_kernel<<<(unsigned)((blocks + 255) / 256), 256, 0, s>>>(x, blocks, channels / 32, data, scale);
    return cudaGetLastError();
}

cudaError_t launch_latent_append(const LatentAppendArgs& a, cudaStream_t s) {
    const long long threads = (long long)a.batch * a.t * kLatTasks;
    if (threads == 0) return cudaSuccess;
    return launch_after_prior(latent_append_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, s, a);
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s) {
    const long long threads = (long long)a.batch * a.t * 48;
    if (threads == 0) return cudaSuccess;
    const int blk = 192;
    const long long grid = (threads + blk - 1) / blk;
    return launch_after_prior(append_kernel, dim3((unsigned)grid), dim3(blk), 0, s, a);
}

}  // namespace csa2
