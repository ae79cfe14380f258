// noalloc.cu -- csa2_sparse_attend_noalloc: sparse attention without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run attention: a host
// application that owns every byte of device memory through its own allocator, or a serving loop
// that must not allocate after start-up because an allocation can synchronise the device. This
// entry point runs the same attention kernel as csa2_sparse_attend, but its scratch (the
// split-combine tickets, the partial results and the device status word) lives in one file-scope
// device array that every GPU loading the library holds until the process exits.
//
// Scratch layout (fixed, so that tickets left at zero by one call are zero for the next):
//   [0, 256)                         status word (never reported by this entry point)
//   [256, 256 + 4*kNoAllocMaxRows)   one ticket per query row
//   [align256(..), kNoAllocBytes)    partial (m, l, O) of each split, used only when a row is split
#include <mutex>

#include "csa2_internal.cuh"

using namespace csa2;

namespace {

constexpr int kNoAllocMaxRows = 1024;                       // batch * tq
constexpr size_t kNoAllocBytes = (size_t)4 << 20;           // 4 MiB per device
constexpr size_t kNoAllocTickets = 256;
constexpr size_t kNoAllocParts = (kNoAllocTickets + 4 * (size_t)kNoAllocMaxRows + 255) & ~size_t(255);

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of the array on each device, taken once with that device current. A host-side
// reference to g_noalloc_scratch names a host stand-in, never the device memory itself.
// The array needs no clearing: a __device__ array without an initialiser is zero when the module
// is loaded on a device, and every call leaves the tickets it used at zero again. (Clearing it here
// with a memset would need ordering against the caller's stream, which may be a non-blocking one.)
// The cached address belongs to the device's primary context: after cudaDeviceReset the module is
// loaded afresh at another address, so this entry point must not be used after a device reset.
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[256] = {};

csa2_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return CSA2_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CSA2_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return CSA2_OK;
}

bool al16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" CSA2_API csa2_status csa2_sparse_attend_noalloc(const csa2_shape* shape, const csa2_cache* cache, int batch,
                                                           int tq, const int64_t* qpos, const uint16_t* q,
                                                           const int32_t* idx, int k, const int64_t* swa_begin,
                                                           float sm_scale, uint16_t* out, float* out_f32, float* lse,
                                                           void* stream) {
    if (!shape || !cache) return CSA2_ERR_INVALID_ARG;
    if (shape->hq != kHQ || shape->d != kD || shape->hi != kHI || shape->di != kDI || shape->hk != kHK ||
        shape->bs != kBS || shape->win < 0 || shape->win > 128 || (shape->ratio != 1 && shape->ratio != 2))
        return CSA2_ERR_UNSUPPORTED_SHAPE;
    if (cache->cap <= 0 || cache->swa_cap <= 0 || (cache->swa_cap & (cache->swa_cap - 1)) || !cache->kv_data ||
        !cache->kv_scale || !cache->swa || !al16(cache->kv_data) || !al16(cache->kv_scale) || !al16(cache->swa))
        return CSA2_ERR_INVALID_ARG;
    if (cache->cap > ((int64_t)1 << 30)) return CSA2_ERR_CAPACITY;
    if (batch < 0 || tq < 1 || k < 1 || k > kMaxK || !qpos || !q || !idx || !out || !al16(q) || !al16(out))
        return CSA2_ERR_INVALID_ARG;
    if (out_f32 && !al16(out_f32)) return CSA2_ERR_INVALID_ARG;
    if (!(sm_scale >= 0.f) || isinf(sm_scale)) return CSA2_ERR_INVALID_ARG;
    if ((long long)batch * tq > kNoAllocMaxRows) return CSA2_ERR_CAPACITY;
    if (batch == 0) return CSA2_OK;
    AttendPlan ap = make_attend_plan(batch * tq, k, shape->win);
    WsLayout L{};
    L.att_ticket = kNoAllocTickets;
    L.att_part = kNoAllocParts;
    const size_t part = ap.splits > 1 ? (size_t)ap.rows * ap.splits * kHQ * kPartStride * 4 : 0;
    if (kNoAllocParts + part > kNoAllocBytes) return CSA2_ERR_CAPACITY;
    void* scratch = nullptr;
    csa2_status st = noalloc_scratch(&scratch);
    if (st != CSA2_OK) return st;
    AttendArgs a{};
    a.c = *cache;
    a.rows = batch * tq;
    a.tq = tq;
    a.k = k;
    a.win = shape->win;
    a.ratio = shape->ratio;
    a.qpos = qpos;
    a.q = q;
    a.idx = idx;
    a.swa_begin = swa_begin;
    a.sm_scale = sm_scale == 0.f ? 1.0f / sqrtf((float)kD) : sm_scale;
    a.out = out;
    a.out_f32 = out_f32;
    a.lse = lse;
    a.plan = ap;
    a.ws = reinterpret_cast<unsigned char*>(scratch);
    a.L = L;
    return launch_attend(a, (cudaStream_t)stream) == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}
