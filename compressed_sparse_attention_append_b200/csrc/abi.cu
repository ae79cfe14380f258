// abi.cu -- the extern "C" entry points of libcsa2 (declared and documented in include/csa2.h):
// argument validation, workspace planning, kernel launches, status codes. Nothing here computes
// any part of the layer step; every step runs in the kernels of append.cu, index.cu, index_decode.cu,
// index_mma.cu, attend.cu, noalloc.cu, latent.cu and latent_index.cu.
#include <math.h>

#include "csa2_internal.cuh"

using namespace csa2;

namespace {

bool al16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

csa2_status check_shape(const csa2_shape* s) {
    if (!s) return CSA2_ERR_INVALID_ARG;
    if (s->hq != kHQ || s->d != kD || s->hi != kHI || s->di != kDI || s->hk != kHK || s->bs != kBS ||
        s->win < 0 || s->win > 128 || (s->ratio != 1 && s->ratio != 2))
        return CSA2_ERR_UNSUPPORTED_SHAPE;
    return CSA2_OK;
}

// planes: 1 = main, 2 = indexer, 4 = window
csa2_status check_cache(const csa2_cache* c, int planes) {
    if (!c || c->cap <= 0 || c->swa_cap <= 0 || (c->swa_cap & (c->swa_cap - 1))) return CSA2_ERR_INVALID_ARG;
    if (c->cap > ((int64_t)1 << 30)) return CSA2_ERR_CAPACITY;  // positions travel as int32 with headroom
    if (planes & 1) {
        if (!c->kv_data || !c->kv_scale || !al16(c->kv_data) || !al16(c->kv_scale)) return CSA2_ERR_INVALID_ARG;
    }
    if (planes & 2) {
        if (!c->ik_data || !c->ik_scale || !al16(c->ik_data) || !al16(c->ik_scale)) return CSA2_ERR_INVALID_ARG;
    }
    if (planes & 4) {
        if (!c->swa || !al16(c->swa)) return CSA2_ERR_INVALID_ARG;
    }
    return CSA2_OK;
}

csa2_status from_cuda(cudaError_t e) { return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

size_t index_bytes(const IndexPlan& ip) { return make_layout(&ip, nullptr).total; }
size_t attend_bytes(const AttendPlan& ap) { return make_layout(nullptr, &ap).total; }

#define CSA2_TRY(x)                          \
    do {                                     \
        csa2_status _s = (x);                \
        if (_s != CSA2_OK) return _s;        \
    } while (0)

csa2_status do_append(const csa2_shape* shape, const csa2_cache* cache, int batch, int t, const int64_t* pos,
                      int64_t pos_host, const uint16_t* kv, const uint16_t* idx_k, const uint16_t* swa_kv, void* ws,
                      size_t ws_bytes, void* stream) {
    CSA2_TRY(check_shape(shape));
    if (batch < 0 || t < 0) return CSA2_ERR_INVALID_ARG;
    const int planes = (kv ? 1 : 0) | (idx_k ? 2 : 0) | (swa_kv ? 4 : 0);
    CSA2_TRY(check_cache(cache, planes));
    if (batch == 0 || t == 0 || planes == 0) return CSA2_OK;
    if ((kv && !al16(kv)) || (idx_k && !al16(idx_k)) || (swa_kv && !al16(swa_kv))) return CSA2_ERR_INVALID_ARG;
    if ((kv || idx_k) && t > cache->cap) return CSA2_ERR_CAPACITY;
    if (ws && ws_bytes < 256) return CSA2_ERR_WORKSPACE;
    if (!pos && pos_host < 0) return CSA2_ERR_INVALID_ARG;
    if (!pos && (kv || idx_k) && pos_host + t > cache->cap) return CSA2_ERR_CAPACITY;
    AppendArgs a{};
    a.c = *cache;
    a.batch = batch;
    a.t = t;
    a.pos = pos;
    a.pos_host = pos_host;
    a.kv = kv;
    a.idx_k = idx_k;
    a.swa_kv = swa_kv;
    a.status = ws ? reinterpret_cast<uint32_t*>(ws) : nullptr;
    return from_cuda(launch_append(a, (cudaStream_t)stream));
}

csa2_status do_index(const csa2_shape* shape, const csa2_cache* cache, int batch, int tq, const int64_t* qpos,
                     int64_t qpos_base, const uint16_t* idx_q, int k, int32_t* out_idx, int pool_blocks,
                     int32_t* out_pool, int32_t* out_pool_n, int64_t max_ctx, int reindex, const int32_t* pool,
                     const int32_t* pool_n, int pool_stride, uint32_t flags, void* ws, size_t ws_bytes, void* stream) {
    CSA2_TRY(check_shape(shape));
    CSA2_TRY(check_cache(cache, 2));
    if (batch < 0 || tq < 1 || k < 1 || k > kMaxK || !idx_q || !out_idx || !al16(idx_q)) return CSA2_ERR_INVALID_ARG;
    if ((long long)batch * tq > kMaxRows) return CSA2_ERR_INVALID_ARG;
    if (flags & ~CSA2_SCORE_RELU) return CSA2_ERR_INVALID_ARG;
    if (!ws) return CSA2_ERR_WORKSPACE;
    if (reindex) {
        if (!pool || !pool_n || pool_stride < 0) return CSA2_ERR_INVALID_ARG;
        pool_blocks = 0;
    } else {
        if (pool_blocks < 0 || pool_blocks > kMaxK) return CSA2_ERR_INVALID_ARG;
        if (pool_blocks > 0 && (tq != 1 || !out_pool || !out_pool_n)) return CSA2_ERR_INVALID_ARG;
        if (max_ctx < 1) return CSA2_ERR_INVALID_ARG;
        if (max_ctx > cache->cap) return CSA2_ERR_CAPACITY;
    }
    if (batch == 0) return CSA2_OK;
    const int64_t max_scan = reindex ? (int64_t)pool_stride * kBS : max_ctx;
    IndexPlan ip = make_index_plan(batch * tq, tq, k, max_scan, pool_blocks);
    WsLayout L = make_layout(&ip, nullptr);
    if (ws_bytes < L.total) return CSA2_ERR_WORKSPACE;
    IndexArgs a{};
    a.c = *cache;
    a.rows = batch * tq;
    a.tq = tq;
    a.qpos = qpos;
    a.qpos_base = qpos_base;
    a.idx_q = idx_q;
    a.reindex = reindex;
    a.pool = pool;
    a.pool_n = pool_n;
    a.pool_stride = pool_stride;
    a.max_ctx = reindex ? cache->cap : max_ctx;
    a.ratio = shape->ratio;
    a.out_idx = out_idx;
    a.out_pool = out_pool;
    a.out_pool_n = out_pool_n;
    a.flags = flags;
    a.plan = ip;
    a.ws = reinterpret_cast<unsigned char*>(ws);
    a.L = L;
    return from_cuda(ip.decode ? launch_index_decode(a, (cudaStream_t)stream) : launch_index(a, (cudaStream_t)stream));
}

csa2_status do_attend(const csa2_shape* shape, const csa2_cache* cache, int batch, int tq, const int64_t* qpos,
                      int64_t qpos_base, const uint16_t* q, const int32_t* idx, int k, const int64_t* swa_begin,
                      int64_t swa_begin_host, float sm_scale, uint16_t* out, float* out_f32, float* lse, void* ws,
                      size_t ws_bytes, void* stream) {
    CSA2_TRY(check_shape(shape));
    CSA2_TRY(check_cache(cache, 1 | 4));
    if (batch < 0 || tq < 1 || k < 1 || k > kMaxK || !q || !idx || !out || !al16(q) || !al16(out))
        return CSA2_ERR_INVALID_ARG;
    if (out_f32 && !al16(out_f32)) return CSA2_ERR_INVALID_ARG;
    if ((long long)batch * tq > kMaxRows) return CSA2_ERR_INVALID_ARG;
    if (!(sm_scale >= 0.f) || isinf(sm_scale)) return CSA2_ERR_INVALID_ARG;
    if (!ws) return CSA2_ERR_WORKSPACE;
    if (batch == 0) return CSA2_OK;
    AttendPlan ap = make_attend_plan(batch * tq, k, shape->win);
    WsLayout L = make_layout(nullptr, &ap);
    if (ws_bytes < L.total) return CSA2_ERR_WORKSPACE;
    AttendArgs a{};
    a.c = *cache;
    a.rows = batch * tq;
    a.tq = tq;
    a.k = k;
    a.win = shape->win;
    a.ratio = shape->ratio;
    a.qpos = qpos;
    a.qpos_base = qpos_base;
    a.swa_begin_host = swa_begin_host;
    a.q = q;
    a.idx = idx;
    a.swa_begin = swa_begin;
    a.sm_scale = sm_scale == 0.f ? 1.0f / sqrtf((float)kD) : sm_scale;
    a.out = out;
    a.out_f32 = out_f32;
    a.lse = lse;
    a.plan = ap;
    a.ws = reinterpret_cast<unsigned char*>(ws);
    a.L = L;
    return from_cuda(launch_attend(a, (cudaStream_t)stream));
}

}  // namespace

extern "C" {

size_t csa2_entry_bytes(int channels) {
    if (channels <= 0 || channels % 16) return 0;
    return (size_t)channels / 2 + (size_t)channels / 16;
}

size_t csa2_mx_entry_bytes(int channels) {
    if (channels <= 0 || channels % 32) return 0;
    return (size_t)channels / 2 + (size_t)channels / 32;
}

csa2_status csa2_mxfp4_quantize(const uint16_t* x, int64_t rows, int channels, uint8_t* data, uint8_t* scale,
                                void* stream) {
    if (rows < 0 || channels <= 0 || channels % 32 || !x || !data || !scale || !al16(x) || !al16(data))
        return CSA2_ERR_INVALID_ARG;
    if (rows == 0) return CSA2_OK;
    return from_cuda(launch_mxfp4(x, (long long)rows, channels, data, scale, (cudaStream_t)stream));
}

csa2_status csa2_latent_append(const csa2_latent_cache* cache, int batch, int t, const int64_t* pos,
                               const uint16_t* latent, const uint16_t* idx_k, const uint16_t* swa, void* ws,
                               size_t ws_bytes, void* stream) {
    if (!cache || !pos || batch < 0 || t < 0) return CSA2_ERR_INVALID_ARG;
    if (cache->cap <= 0 || cache->swa_cap <= 0 || (cache->swa_cap & (cache->swa_cap - 1))) return CSA2_ERR_INVALID_ARG;
    if (cache->cap > ((int64_t)1 << 30)) return CSA2_ERR_CAPACITY;
    if (latent && (!al16(latent) || !cache->l_data || !cache->l_scale || !al16(cache->l_data) || !al16(cache->l_scale)))
        return CSA2_ERR_INVALID_ARG;
    if (idx_k && (!al16(idx_k) || !cache->k_data || !cache->k_scale || !al16(cache->k_data) || !al16(cache->k_scale)))
        return CSA2_ERR_INVALID_ARG;
    if (swa && (!al16(swa) || !cache->swa || !al16(cache->swa))) return CSA2_ERR_INVALID_ARG;
    if (ws && ws_bytes < 256) return CSA2_ERR_WORKSPACE;
    if (batch == 0 || t == 0 || (!latent && !idx_k && !swa)) return CSA2_OK;
    if ((latent || idx_k) && t > cache->cap) return CSA2_ERR_CAPACITY;
    LatentAppendArgs a{};
    a.c = *cache;
    a.batch = batch;
    a.t = t;
    a.pos = pos;
    a.latent = latent;
    a.idx_k = idx_k;
    a.swa = swa;
    a.status = ws ? reinterpret_cast<uint32_t*>(ws) : nullptr;
    return from_cuda(launch_latent_append(a, (cudaStream_t)stream));
}

csa2_status csa2_latent_attend(const csa2_latent_cache* cache, int batch, int tq, const int64_t* qpos,
                               const uint16_t* q, const int32_t* idx, int k, const int64_t* swa_begin, int win,
                               int ratio, float sm_scale, uint16_t* out, float* out_f32, float* lse, void* ws,
                               size_t ws_bytes, void* stream) {
    if (!cache || !qpos || !q || !out || batch < 0 || tq < 1 || k < 0 || k > kMaxK) return CSA2_ERR_INVALID_ARG;
    if (win < 0 || win > 128 || (ratio != 1 && ratio != 2)) return CSA2_ERR_UNSUPPORTED_SHAPE;
    if (cache->cap <= 0 || cache->swa_cap <= 0 || (cache->swa_cap & (cache->swa_cap - 1))) return CSA2_ERR_INVALID_ARG;
    if (cache->cap > ((int64_t)1 << 30)) return CSA2_ERR_CAPACITY;
    if (win > 0 && cache->swa_cap < win) return CSA2_ERR_CAPACITY;  // the ring must hold the window
    if (k > 0 && (!idx || !cache->l_data || !cache->l_scale || !al16(cache->l_data) || !al16(cache->l_scale)))
        return CSA2_ERR_INVALID_ARG;
    if (win > 0 && (!cache->swa || !al16(cache->swa))) return CSA2_ERR_INVALID_ARG;
    if (!al16(q) || !al16(out) || (out_f32 && !al16(out_f32))) return CSA2_ERR_INVALID_ARG;
    if (ws && ws_bytes < 256) return CSA2_ERR_WORKSPACE;
    if ((long long)batch * tq > (1ll << 31) - 1) return CSA2_ERR_INVALID_ARG;
    if (batch == 0) return CSA2_OK;
    LatentAttendArgs a{};
    a.c = *cache;
    a.rows = batch * tq;
    a.tq = tq;
    a.k = k;
    a.win = win;
    a.ratio = ratio;
    a.qpos = qpos;
    a.swa_begin = swa_begin;
    a.q = q;
    a.idx = idx;
    a.sm_scale = sm_scale == 0.f ? 1.0f / sqrtf((float)kLatD) : sm_scale;
    a.out = out;
    a.out_f32 = out_f32;
    a.lse = lse;
    a.status = ws ? reinterpret_cast<uint32_t*>(ws) : nullptr;
    return from_cuda(launch_latent_attend(a, (cudaStream_t)stream));
}

csa2_status csa2_latent_index_workspace_size(int rows, int hi, int64_t max_ctx, size_t* bytes) {
    if (!bytes || rows < 0 || rows > 65535 || hi < 1 || hi > kLatMaxHI || max_ctx < 1) return CSA2_ERR_INVALID_ARG;
    *bytes = latent_index_ws_bytes(rows, hi, max_ctx);
    return CSA2_OK;
}

csa2_status csa2_latent_index_topk(const csa2_latent_cache* cache, int batch, int tq, const int64_t* qpos,
                                   const uint16_t* idx_q, int hi, int k, int ratio, int64_t max_ctx, uint32_t flags,
                                   int32_t* out_idx, void* ws, size_t ws_bytes, void* stream) {
    if (!cache || !qpos || !idx_q || !out_idx || !ws || batch < 0 || tq < 1) return CSA2_ERR_INVALID_ARG;
    if (hi < 1 || hi > kLatMaxHI || k < 1 || k > kMaxK || max_ctx < 1) return CSA2_ERR_INVALID_ARG;
    if (ratio != 1 && ratio != 2) return CSA2_ERR_UNSUPPORTED_SHAPE;
    if ((long long)batch * tq > 65535) return CSA2_ERR_INVALID_ARG;
    if (cache->cap <= 0 || cache->cap > ((int64_t)1 << 30)) return CSA2_ERR_INVALID_ARG;
    if (!cache->k_data || !cache->k_scale || !al16(cache->k_data) || !al16(cache->k_scale)) return CSA2_ERR_INVALID_ARG;
    if (!al16(idx_q) || ((uintptr_t)ws & 255u)) return CSA2_ERR_INVALID_ARG;
    const int rows = batch * tq;
    if (ws_bytes < latent_index_ws_bytes(rows, hi, max_ctx)) return CSA2_ERR_WORKSPACE;
    if (rows == 0) return CSA2_OK;
    LatIndexArgs a{};
    a.c = *cache;
    a.rows = rows;
    a.tq = tq;
    a.hi = hi;
    a.k = k;
    a.ratio = ratio;
    a.max_ctx = max_ctx;
    a.qpos = qpos;
    a.flags = flags;
    a.out_idx = out_idx;
    return from_cuda(launch_latent_index(a, idx_q, reinterpret_cast<unsigned char*>(ws), (cudaStream_t)stream));
}

const char* csa2_status_string(csa2_status s) {
    switch (s) {
        case CSA2_OK: return "ok";
        case CSA2_ERR_INVALID_ARG: return "invalid argument";
        case CSA2_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case CSA2_ERR_CAPACITY: return "capacity exceeded";
        case CSA2_ERR_WORKSPACE: return "workspace missing or too small";
        case CSA2_ERR_CUDA: return "CUDA launch failed";
        case CSA2_ERR_DEVICE: return "device-side error bits set";
    }
    return "unknown status";
}

int csa2_version(void) { return 200; }

csa2_status csa2_workspace_size(const csa2_shape* shape, int batch, int tq, int k, int64_t max_scan, int pool_blocks,
                                size_t* bytes) {
    CSA2_TRY(check_shape(shape));
    if (!bytes || batch < 0 || tq < 1 || k < 1 || k > kMaxK || max_scan < 0 || pool_blocks < 0 || pool_blocks > kMaxK)
        return CSA2_ERR_INVALID_ARG;
    if ((long long)batch * tq > kMaxRows) return CSA2_ERR_INVALID_ARG;
    const int rows = batch * tq;
    IndexPlan ip = make_index_plan(rows, tq, k, max_scan > 0 ? max_scan : 1, pool_blocks);
    AttendPlan ap = make_attend_plan(rows, k, shape->win);
    const size_t a = index_bytes(ip), b = attend_bytes(ap);
    *bytes = a > b ? a : b;
    return CSA2_OK;
}

csa2_status csa2_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (!ws || ws_bytes < 256 || ((uintptr_t)ws & 255u)) return CSA2_ERR_INVALID_ARG;
    return from_cuda(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
}

csa2_status csa2_quantize_append(const csa2_shape* shape, const csa2_cache* cache, int batch, int t, const int64_t* pos,
                                 const uint16_t* kv, const uint16_t* idx_k, const uint16_t* swa_kv, void* ws,
                                 size_t ws_bytes, void* stream) {
    if (!pos) return CSA2_ERR_INVALID_ARG;
    return do_append(shape, cache, batch, t, pos, 0, kv, idx_k, swa_kv, ws, ws_bytes, stream);
}

csa2_status csa2_index_topk_full(const csa2_shape* shape, const csa2_cache* cache, int batch, int tq,
                                 const int64_t* qpos, const uint16_t* idx_q, int k, int32_t* out_idx, int pool_blocks,
                                 int32_t* out_pool, int32_t* out_pool_n, int64_t max_ctx, uint32_t flags, void* ws,
                                 size_t ws_bytes, void* stream) {
    if (!qpos) return CSA2_ERR_INVALID_ARG;
    return do_index(shape, cache, batch, tq, qpos, 0, idx_q, k, out_idx, pool_blocks, out_pool, out_pool_n, max_ctx, 0,
                    nullptr, nullptr, 0, flags, ws, ws_bytes, stream);
}

csa2_status csa2_index_topk_reindex(const csa2_shape* shape, const csa2_cache* cache, int batch, const int64_t* qpos,
                                    const uint16_t* idx_q, const int32_t* pool, const int32_t* pool_n, int pool_stride,
                                    int k, int32_t* out_idx, uint32_t flags, void* ws, size_t ws_bytes, void* stream) {
    if (!qpos) return CSA2_ERR_INVALID_ARG;
    return do_index(shape, cache, batch, 1, qpos, 0, idx_q, k, out_idx, 0, nullptr, nullptr, 0, 1, pool, pool_n,
                    pool_stride, flags, ws, ws_bytes, stream);
}

csa2_status csa2_sparse_attend(const csa2_shape* shape, const csa2_cache* cache, int batch, int tq, const int64_t* qpos,
                               const uint16_t* q, const int32_t* idx, int k, const int64_t* swa_begin, float sm_scale,
                               uint16_t* out, float* out_f32, float* lse, void* ws, size_t ws_bytes, void* stream) {
    if (!qpos) return CSA2_ERR_INVALID_ARG;
    return do_attend(shape, cache, batch, tq, qpos, 0, q, idx, k, swa_begin, 0, sm_scale, out, out_f32, lse, ws,
                     ws_bytes, stream);
}

csa2_status csa2_decode_full(const csa2_shape* shape, const csa2_cache* cache, int batch, const int64_t* qpos,
                             const uint16_t* kv, const uint16_t* idx_k, const uint16_t* swa_kv, const uint16_t* idx_q,
                             const uint16_t* q, int k, int32_t* out_idx, int pool_blocks, int32_t* out_pool,
                             int32_t* out_pool_n, int64_t max_ctx, const int64_t* swa_begin, float sm_scale,
                             uint16_t* out, float* out_f32, float* lse, uint32_t flags, void* ws, size_t ws_bytes,
                             void* stream) {
    if (!qpos || !kv || !idx_k || !swa_kv) return CSA2_ERR_INVALID_ARG;
    CSA2_TRY(check_shape(shape));
    if (shape->ratio != 1) return CSA2_ERR_UNSUPPORTED_SHAPE;  // an entry per token only
    CSA2_TRY(do_append(shape, cache, batch, 1, qpos, 0, kv, idx_k, swa_kv, ws, ws_bytes, stream));
    CSA2_TRY(do_index(shape, cache, batch, 1, qpos, 0, idx_q, k, out_idx, pool_blocks, out_pool, out_pool_n, max_ctx, 0,
                      nullptr, nullptr, 0, flags, ws, ws_bytes, stream));
    return do_attend(shape, cache, batch, 1, qpos, 0, q, out_idx, k, swa_begin, 0, sm_scale, out, out_f32, lse, ws,
                     ws_bytes, stream);
}

csa2_status csa2_decode_reindex(const csa2_shape* shape, const csa2_cache* cache, int batch, const int64_t* qpos,
                                const uint16_t* swa_kv, const uint16_t* idx_q, const uint16_t* q, const int32_t* pool,
                                const int32_t* pool_n, int pool_stride, int k, int32_t* out_idx,
                                const int64_t* swa_begin, float sm_scale, uint16_t* out, float* out_f32, float* lse,
                                uint32_t flags, void* ws, size_t ws_bytes, void* stream) {
    if (!qpos || !swa_kv) return CSA2_ERR_INVALID_ARG;
    CSA2_TRY(do_append(shape, cache, batch, 1, qpos, 0, nullptr, nullptr, swa_kv, ws, ws_bytes, stream));
    CSA2_TRY(do_index(shape, cache, batch, 1, qpos, 0, idx_q, k, out_idx, 0, nullptr, nullptr, 0, 1, pool, pool_n,
                      pool_stride, flags, ws, ws_bytes, stream));
    return do_attend(shape, cache, batch, 1, qpos, 0, q, out_idx, k, swa_begin, 0, sm_scale, out, out_f32, lse, ws,
                     ws_bytes, stream);
}

csa2_status csa2_decode_minimal(const csa2_shape* shape, const csa2_cache* cache, int batch, const int64_t* qpos,
                                const uint16_t* swa_kv, const uint16_t* q, const int32_t* idx, int k,
                                const int64_t* swa_begin, float sm_scale, uint16_t* out, float* out_f32, float* lse,
                                void* ws, size_t ws_bytes, void* stream) {
    if (!qpos || !swa_kv) return CSA2_ERR_INVALID_ARG;
    CSA2_TRY(do_append(shape, cache, batch, 1, qpos, 0, nullptr, nullptr, swa_kv, ws, ws_bytes, stream));
    return do_attend(shape, cache, batch, 1, qpos, 0, q, idx, k, swa_begin, 0, sm_scale, out, out_f32, lse, ws,
                     ws_bytes, stream);
}

csa2_status csa2_prefill_chunk(const csa2_shape* shape, const csa2_cache* cache, int64_t pos0, int t,
                               const uint16_t* kv, const uint16_t* idx_k, const uint16_t* swa_kv,
                               const uint16_t* idx_q, const uint16_t* q, int k, int32_t* out_idx, int64_t swa_begin,
                               float sm_scale, uint16_t* out, float* out_f32, float* lse, uint32_t flags, void* ws,
                               size_t ws_bytes, void* stream) {
    if (!shape || !cache || !kv || !idx_k || !swa_kv || t < 1 || pos0 < 0) return CSA2_ERR_INVALID_ARG;
    CSA2_TRY(check_shape(shape));
    if (shape->ratio != 1) return CSA2_ERR_UNSUPPORTED_SHAPE;  // an entry per token only
    if (pos0 + t > cache->cap) return CSA2_ERR_CAPACITY;
    if (cache->swa_cap < (int64_t)t + (shape ? shape->win : 0)) return CSA2_ERR_CAPACITY;
    CSA2_TRY(do_append(shape, cache, 1, t, nullptr, pos0, kv, idx_k, swa_kv, ws, ws_bytes, stream));
    CSA2_TRY(do_index(shape, cache, 1, t, nullptr, pos0, idx_q, k, out_idx, 0, nullptr, nullptr, pos0 + t, 0, nullptr,
                      nullptr, 0, flags, ws, ws_bytes, stream));
    return do_attend(shape, cache, 1, t, nullptr, pos0, q, out_idx, k, nullptr, swa_begin, sm_scale, out, out_f32, lse,
                     ws, ws_bytes, stream);
}

csa2_status csa2_get_device_status(void* ws, void* stream, int32_t* host_status) {
    if (!ws || !host_status) return CSA2_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, 4, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    *host_status = (int32_t)v;
    return v ? CSA2_ERR_DEVICE : CSA2_OK;
}

}  // extern "C"
