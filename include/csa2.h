/*
 * csa2.h -- C ABI of libcsa2: one CSA2 (Compressed Sparse Attention 2) layer step over an FP4
 * KV cache, on one NVIDIA B200 (sm_100a).
 *
 * Sources (tags used in the comments below):
 *   [A] "DeepSeek-V4.1-Flash: Shrinking KV Cache at 552B Scale" (visualisation captions page)
 *   [B] "DeepSeek Cuts KV Cache Footprint Fourfold" (paper summary), "Technical Approach"
 *   [C] "DeepSeek-V4.1-Flash: Pushing KV Cache Compression to 890 Bytes per Token"
 *       (engineering article), sections VI, VII, IX, XI, XII
 *
 * The pages define the operations but no API, no cache layout, no index-score formula, no
 * softmax scale and no rounding rule. Where this header fixes one of those, it says so.
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless marked "host". bf16 tensors are passed as their raw
 *     16-bit patterns (uint16_t). All tensors are dense, row-major, in the shapes stated.
 *   - Ownership: the caller owns every buffer (cache planes, inputs, outputs, workspace).
 *     libcsa2 allocates nothing, keeps no mutable global state and never frees.
 *   - Streams: `stream` is a cudaStream_t passed as void*. Every call only enqueues work on it
 *     and returns without synchronising (except csa2_get_device_status). Calls on one stream
 *     run in order; calls that share one workspace must not run concurrently.
 *   - Errors: host-checkable argument errors return a status before anything is enqueued.
 *     Errors found on the device (an inherited index out of range, an append past the cache
 *     capacity, a pool block id out of range) set bits of a status word inside the workspace
 *     and the offending item is skipped; read it with csa2_get_device_status. No call traps,
 *     asserts or spins on the device.
 *   - Fixed shapes of this library: hq = 16 query heads, d = 128 (K and V each), one shared KV
 *     head, hi = 4 indexer query heads, di = 64, hk = 4 indexer key heads, bs = 8 positions
 *     per pool block, win <= 128. Other values return CSA2_ERR_UNSUPPORTED_SHAPE.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1,      /* null pointer, negative size, misaligned pointer        */
    CSA2_ERR_UNSUPPORTED_SHAPE = 2,/* shape outside what this library implements             */
    CSA2_ERR_CAPACITY = 3,         /* a bound that the host can see exceeds the cache        */
    CSA2_ERR_WORKSPACE = 4,        /* workspace pointer null or smaller than required        */
    CSA2_ERR_CUDA = 5,             /* a kernel launch failed (cudaGetLastError)              */
    CSA2_ERR_DEVICE = 6            /* csa2_get_device_status found device-side error bits    */
} csa2_status;

/* Device status bits (csa2_get_device_status). */
#define CSA2_DEV_BAD_INDEX   0x1   /* selected / inherited index < -1, > qpos or >= cap       */
#define CSA2_DEV_BAD_POS     0x2   /* append position outside [0, cap) or qpos >= bound       */
#define CSA2_DEV_BAD_POOL    0x4   /* pool block id outside [0, cap / bs)                     */
#define CSA2_DEV_TIMEOUT     0x8   /* a tensor-core pipeline wait ran out (no output written)  */

/* Flags for the index entry points. */
#define CSA2_SCORE_RELU      0x1u  /* score = sum_h max(0, q_h . k_h) instead of sum_h q_h . k_h */

typedef struct {
    int hq;   /* query heads (16)                                 */
    int d;    /* head dim of K and of V (128)                     */
    int hi;   /* indexer query heads (4)                          */
    int di;   /* indexer head dim (64)                            */
    int hk;   /* indexer key heads (4)                            */
    int win;  /* sliding-window length (128; [C] config list)     */
    int bs;   /* positions per pool block (8; [C] sec. IX)        */
    int ratio; /* tokens per main / indexer cache entry: 1, or 2 for the encoder layers of
                  [C] sec. VIII (one entry per 2 tokens). Entry e summarises tokens
                  ratio*e .. ratio*e + ratio - 1; a query at token i may use entries
                  0 .. floor((i + 1) / ratio) - 1. Window slots stay per token. */
} csa2_shape;

/*
 * Cache of `batch` sequences (layout fixed by this library; the pages give none). Per sequence b
 * and position p (0 <= p < cap):
 *   kv_data  + (b*cap + p)*128      : main K||V, 256 channels (K = 0..127, V = 128..255) as E2M1
 *                                     codes, channel 2j in the low nibble of byte j
 *   kv_scale + (b*cap + p)*16       : one E4M3 scale byte per 16 channels (block b <-> byte b)
 *   ik_data  + (b*cap + p)*hk*32    : indexer key, hk heads x 64 channels, E2M1 as above
 *   ik_scale + (b*cap + p)*hk*4     : its E4M3 scales
 *   swa      + (b*swa_cap + (p & (swa_cap-1)))*256 : sliding-window K||V as E4M3 bytes (no
 *                                     scale), a ring of swa_cap slots (power of two)
 * Every plane base must be 16-byte aligned. Entry bytes: 144 (main) + 144 (indexer) per
 * position; csa2_entry_bytes gives the rule.
 */
typedef struct {
    uint8_t* kv_data;
    uint8_t* kv_scale;
    uint8_t* ik_data;
    uint8_t* ik_scale;
    uint8_t* swa;
    int64_t cap;      /* positions per sequence in the main and indexer planes (<= 2^30) */
    int64_t swa_cap;  /* ring slots per sequence, power of two, >= win (decode) */
} csa2_cache;

/* [C] sec. VII (byte budget): an entry of `channels` E2M1 values with one 1-byte E4M3 scale per
 * 16 channels occupies channels/2 + channels/16 bytes. Returns 0 if channels is not a positive
 * multiple of 16. Host only. */
CSA2_API size_t csa2_entry_bytes(int channels);

/* [C] sec. VII: an MXFP4 entry of `channels` E2M1 values with one 1-byte E8M0 scale per 32
 * channels (the pages' indexer-key format) occupies channels/2 + channels/32 bytes. Returns 0 if
 * channels is not a positive multiple of 32. Host only. */
CSA2_API size_t csa2_mx_entry_bytes(int channels);

/* Text of a status code. Host only; never NULL. */
CSA2_API const char* csa2_status_string(csa2_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. Host only. */
CSA2_API int csa2_version(void);

/*
 * Workspace bytes needed by any entry point below when called with at most `batch` sequences,
 * `tq` query rows per sequence, top-k `k` (<= 2048), at most `max_scan` positions scanned by
 * the indexer per query row (Full: the largest qpos+1; Reindex: pool entries * bs) and
 * `pool_blocks` pool blocks (0 if no pool is built). Host only. The workspace must be 256-byte
 * aligned and, once after allocation, cleared with csa2_workspace_init; every call leaves its
 * counters cleared again.
 */
CSA2_API csa2_status csa2_workspace_size(const csa2_shape* shape, int batch, int tq, int k, int64_t max_scan,
                                int pool_blocks, size_t* bytes /* host */);

/* Zeroes the workspace (one cudaMemsetAsync on `stream`). */
CSA2_API csa2_status csa2_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Quantise-append. [C] sec. XI: cached values are E2M1 with one E4M3 scale per 16 channels and
 * no scale for the whole tensor on top, quantised after RoPE; the sliding-window KV stays at FP8.
 * [B] "Technical Approach": Full mode writes main KV and indexer keys, Reindex and Minimal
 * write only their own sliding-window KV (pass NULL for the planes a mode does not write).
 *   pos    [batch] int64 : first new position of each sequence; tokens go to pos..pos+t-1
 *   kv     [batch][t][256] bf16 or NULL  -> kv_data / kv_scale
 *   idx_k  [batch][t][hk*64] bf16 or NULL -> ik_data / ik_scale
 *   swa_kv [batch][t][256] bf16 or NULL  -> swa ring slots (pos+i) & (swa_cap-1)
 * Rounding (the reading taken here): per 16-channel block s = E4M3_RNE_satfinite(amax/6);
 * s == 0 gives all-zero codes; code_i = E2M1_RNE_satfinite(x_i / s) keeping the sign of x_i;
 * SWA bytes = E4M3_RNE_satfinite(x). A sequence whose range leaves [0, cap) sets
 * CSA2_DEV_BAD_POS and is skipped (needs `ws`; pass NULL to skip the device check).
 */
CSA2_API csa2_status csa2_quantize_append(const csa2_shape* shape, const csa2_cache* cache, int batch, int t,
                                 const int64_t* pos, const uint16_t* kv, const uint16_t* idx_k,
                                 const uint16_t* swa_kv, void* ws, size_t ws_bytes, void* stream);

/*
 * Full-mode index step. [B] "Technical Approach": Full mode computes the Top-K indices;
 * [C] sec. VI "Shortlist-of-a-shortlist" and sec. IX Figure 4: the decoder's first Full layer
 * scores every causally visible position, and collects the blocks with the highest maximum
 * score (up to 2,048 blocks of 8 positions) into a shared candidate pool.
 *   qpos     [batch*tq] int64 : query token of each row; entries 0 .. floor((qpos+1)/ratio)-1 are
 *              visible (with ratio 1: positions 0..qpos)
 *   idx_q    [batch][tq][hi][di] bf16 : indexer query, quantised in-kernel with the codec above
 *   k        : Top-k (<= 2048)
 *   out_idx  [batch][tq][k] int32 : selected positions, ascending, padded with -1
 *   pool_blocks : 0, or the pool size P (decode only: tq == 1)
 *   out_pool [batch][P] int32 : pool block ids, ascending, padded with -1 (NULL if P == 0)
 *   out_pool_n [batch] int32 : min(P, ceil(visible entries / bs))  (NULL if P == 0)
 *   max_ctx  : host upper bound on the visible entries over all rows (<= cap)
 * Score (the reading taken here): score(p) = sum_h q_h . k_{p,h} on dequantised values, exact;
 * ranking by score descending, ties to the lower position (lower block id for the pool).
 */
CSA2_API csa2_status csa2_index_topk_full(const csa2_shape* shape, const csa2_cache* cache, int batch, int tq,
                                 const int64_t* qpos, const uint16_t* idx_q, int k, int32_t* out_idx,
                                 int pool_blocks, int32_t* out_pool, int32_t* out_pool_n, int64_t max_ctx,
                                 uint32_t flags, void* ws, size_t ws_bytes, void* stream);

/*
 * Reindex-mode index step (decode, one query row per sequence). [B] "Technical Approach" and
 * [C] sec. VI: a fresh indexer query chooses its Top-k only inside the shared candidate pool.
 *   qpos   [batch] int64, idx_q [batch][hi][di] bf16
 *   pool   [batch][pool_stride] int32 : block ids (each covers positions bs*id .. bs*id+bs-1)
 *   pool_n [batch] int32 : entries used in each row (<= pool_stride)
 *   out_idx [batch][k] int32 : ascending, padded with -1; entries that are not visible at qpos
 *              (see ratio) are never chosen
 */
CSA2_API csa2_status csa2_index_topk_reindex(const csa2_shape* shape, const csa2_cache* cache, int batch,
                                    const int64_t* qpos, const uint16_t* idx_q, const int32_t* pool,
                                    const int32_t* pool_n, int pool_stride, int k, int32_t* out_idx,
                                    uint32_t flags, void* ws, size_t ws_bytes, void* stream);

/*
 * Sparse attention. [C] sec. VI "What one layer looks like": the layer's own query attends to
 * the selected entries of the shared main KV plus its own recent window; [C] sec. XI: cached
 * values are dequantised before attention; [C] sec. XII: with a replay start s, a query at i
 * sees window keys [max(s, i-win+1), i].
 *   qpos [batch*tq] int64 (query token), q [batch][tq][hq][d] bf16
 *   idx  [batch][tq][k] int32 : main-KV entries, -1 = skip, any order
 *   swa_begin [batch] int64 or NULL (= 0)
 *   sm_scale : softmax scale, 0 gives 1/sqrt(d)
 *   out [batch][tq][hq][d] bf16; out_f32 (same shape, fp32) and lse [batch][tq][hq] fp32 (natural
 *   log) may be NULL.
 * Reading taken here: ONE softmax over selected rows and window rows together; a position may
 * appear in both (its FP4 main entry and its FP8 window entry are different vectors). An index
 * < -1, not visible at qpos (see ratio) or >= cap sets CSA2_DEV_BAD_INDEX and is skipped. A row
 * with no key gives out = 0 and lse = -inf.
 */
CSA2_API csa2_status csa2_sparse_attend(const csa2_shape* shape, const csa2_cache* cache, int batch, int tq,
                               const int64_t* qpos, const uint16_t* q, const int32_t* idx, int k,
                               const int64_t* swa_begin, float sm_scale, uint16_t* out, float* out_f32,
                               float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * One decode step per mode ([B] "Technical Approach": Full computes main KV, indexer keys and
 * Top-K; Reindex reuses main KV and indexer keys and recomputes the selection; Minimal reuses
 * all three and computes only its own query and sliding-window KV). Each is the composition
 * quantise-append -> index step -> sparse attention on `stream`, with the arguments above;
 * the new token sits at qpos[b] (appended before scoring, so it is visible).
 *   decode_full    : appends kv, idx_k, swa_kv; Full index step (pool optional); attention
 *                    (ratio 1 only: with ratio 2 an entry is appended every second token, so the
 *                    caller appends it and calls the index step and attention itself)
 *   decode_reindex : appends swa_kv; Reindex index step; attention
 *   decode_minimal : appends swa_kv; attention with the inherited idx
 * Multi-token decode (t draft tokens per sequence verified together) has no composed call: it is
 * csa2_quantize_append with t tokens at pos[b], csa2_index_topk_full with tq = t (row i of
 * sequence b at qpos[b*t + i] = pos[b] + i, no pool) and csa2_sparse_attend with tq = t; the
 * window ring then needs swa_cap >= win + t.
 */
CSA2_API csa2_status csa2_decode_full(const csa2_shape* shape, const csa2_cache* cache, int batch, const int64_t* qpos,
                             const uint16_t* kv, const uint16_t* idx_k, const uint16_t* swa_kv,
                             const uint16_t* idx_q, const uint16_t* q, int k, int32_t* out_idx,
                             int pool_blocks, int32_t* out_pool, int32_t* out_pool_n, int64_t max_ctx,
                             const int64_t* swa_begin, float sm_scale, uint16_t* out, float* out_f32,
                             float* lse, uint32_t flags, void* ws, size_t ws_bytes, void* stream);

CSA2_API csa2_status csa2_decode_reindex(const csa2_shape* shape, const csa2_cache* cache, int batch,
                                const int64_t* qpos, const uint16_t* swa_kv, const uint16_t* idx_q,
                                const uint16_t* q, const int32_t* pool, const int32_t* pool_n,
                                int pool_stride, int k, int32_t* out_idx, const int64_t* swa_begin,
                                float sm_scale, uint16_t* out, float* out_f32, float* lse, uint32_t flags,
                                void* ws, size_t ws_bytes, void* stream);

CSA2_API csa2_status csa2_decode_minimal(const csa2_shape* shape, const csa2_cache* cache, int batch,
                                const int64_t* qpos, const uint16_t* swa_kv, const uint16_t* q,
                                const int32_t* idx, int k, const int64_t* swa_begin, float sm_scale,
                                uint16_t* out, float* out_f32, float* lse, void* ws, size_t ws_bytes,
                                void* stream);

/*
 * Prefill chunk of t tokens at positions pos0..pos0+t-1 of one sequence (batch 1). [C] sec. X
 * and XI: the chunk's K/V and indexer keys are quantised and appended; every new token then
 * selects its Top-k among positions <= its own and attends to them plus its window.
 *   kv [t][256], idx_k [t][hk*64], swa_kv [t][256], idx_q [t][hi][di], q [t][hq][d] (bf16)
 *   out_idx [t][k] int32, out [t][hq][d] bf16; swa_cap must be >= t + win. ratio 1 only.
 */
CSA2_API csa2_status csa2_prefill_chunk(const csa2_shape* shape, const csa2_cache* cache, int64_t pos0, int t,
                               const uint16_t* kv, const uint16_t* idx_k, const uint16_t* swa_kv,
                               const uint16_t* idx_q, const uint16_t* q, int k, int32_t* out_idx,
                               int64_t swa_begin, float sm_scale, uint16_t* out, float* out_f32, float* lse,
                               uint32_t flags, void* ws, size_t ws_bytes, void* stream);

/*
 * Sparse attention that allocates nothing and takes no workspace (the pages have no counterpart:
 * this is a deployment convenience). Same arguments, outputs and semantics as
 * csa2_sparse_attend, minus `ws` / `ws_bytes`. For callers that cannot allocate device memory
 * where they run attention: a host application whose own allocator owns all device memory, or a
 * serving loop that must not allocate after start-up because an allocation can synchronise the
 * device.
 *   - Scratch: a 4 MiB file-scope device array per GPU, held until the process exits.
 *   - Limit: batch * tq <= 1024; larger calls return CSA2_ERR_CAPACITY.
 *   - The array is zero when the library's module is loaded on a device, and every call leaves
 *     its split tickets at zero again, so no clearing is needed. The first call on a device takes
 *     the array's device address (cudaGetSymbolAddress) and keeps it; make that first call before
 *     any stream capture, and do not call this entry point after cudaDeviceReset on that device.
 *   - Every call shares the one array: calls whose kernels overlap on the GPU (other streams,
 *     other threads) race and must be serialised by the caller.
 *   - Device-side status bits (bad indices) are not reported; bad indices are still skipped.
 */
CSA2_API csa2_status csa2_sparse_attend_noalloc(const csa2_shape* shape, const csa2_cache* cache, int batch, int tq,
                                                const int64_t* qpos, const uint16_t* q, const int32_t* idx, int k,
                                                const int64_t* swa_begin, float sm_scale, uint16_t* out,
                                                float* out_f32, float* lse, void* stream);

/*
 * MXFP4 row codec: the indexer-key format of the pages' own shape ([C] sec. VII names MXFP4: E2M1
 * elements with one E8M0 scale per 32 channels). Rows of `channels` bf16 values (a positive
 * multiple of 32) are quantised independently:
 *   x     [rows][channels] bf16 (device, 16-byte aligned)
 *   data  [rows][channels/2] E2M1 codes, channel 2j in the low nibble of byte j (device, 16-byte
 *         aligned, caller-owned; a cache plane of such rows is data + position * channels/2)
 *   scale [rows][channels/32] E8M0 bytes (device, caller-owned)
 * Rule (the reading taken here; the pages name the format only): per 32-channel block with
 * amax = max |x| > 0, the scale is X = 2^(floor(log2 amax) - 2) (6 = 1.5 * 2^2 is E2M1's largest
 * value), stored as the byte log2 X + 127 clamped to 0..254; code_i = E2M1_RNE_satfinite(x_i / X)
 * keeping the sign of x_i. amax == 0 gives scale byte 0 and all codes +0.
 * Returns CSA2_ERR_INVALID_ARG for a null or misaligned pointer, rows < 0 or a bad `channels`.
 */
CSA2_API csa2_status csa2_mxfp4_quantize(const uint16_t* x, int64_t rows, int channels, uint8_t* data, uint8_t* scale,
                                         void* stream);

/*
 * The pages' own attention shape ([C] sec. VII: the main KV is ONE 512-channel latent per entry,
 * 288 B in E2M1 with an E4M3 scale per 16 channels; the configuration list of [C]'s closing
 * section: 64 query heads of dimension 512, an indexer of 32 heads x 128 over one 128-channel
 * MXFP4 key per entry). The latent is both K and V. Cache of `batch` sequences, per sequence b
 * and position p (0 <= p < cap); every plane base 16-byte aligned; the caller owns every plane:
 *   l_data  + (b*cap + p)*256     : the latent's 512 channels as E2M1 codes (channel 2j in the
 *                                    low nibble of byte j)
 *   l_scale + (b*cap + p)*32      : one E4M3 scale per 16 channels (the codec of this header)
 *   k_data  + (b*cap + p)*64      : the 128-channel indexer key as MXFP4 codes
 *   k_scale + (b*cap + p)*4       : its E8M0 scales (one per 32 channels; see csa2_mxfp4_quantize)
 *   swa     + (b*swa_cap + (p & (swa_cap-1)))*512 : window rows, 512 E4M3 bytes, no scale
 */
typedef struct {
    uint8_t* l_data;
    uint8_t* l_scale;
    uint8_t* k_data;
    uint8_t* k_scale;
    uint8_t* swa;
    int64_t cap;      /* positions per sequence (<= 2^30) */
    int64_t swa_cap;  /* ring slots per sequence, power of two */
} csa2_latent_cache;

/*
 * Quantise-append of t tokens per sequence into the latent cache, at positions pos[b] .. pos[b]
 * + t - 1 ([C] sec. XI: quantised as they are written; the window stays FP8):
 *   latent [batch][t][512], idx_k [batch][t][128], swa [batch][t][512] (bf16, 16-byte aligned;
 *   any may be NULL, and its plane is then neither read nor written). The latent takes the
 *   E2M1/E4M3 codec of csa2_quantize_append, the key the MXFP4 rule of csa2_mxfp4_quantize,
 *   window rows E4M3 (RNE, saturating). A position outside [0, cap) sets CSA2_DEV_BAD_POS in
 *   `ws` (which may be NULL: the bit is then not recorded) and that sequence is skipped.
 * Returns CSA2_ERR_INVALID_ARG for null / misaligned pointers or negative sizes.
 */
CSA2_API csa2_status csa2_latent_append(const csa2_latent_cache* cache, int batch, int t, const int64_t* pos,
                                        const uint16_t* latent, const uint16_t* idx_k, const uint16_t* swa, void* ws,
                                        size_t ws_bytes, void* stream);

/*
 * Sparse attention of the pages' own shape, on the tensor cores: each of the batch*tq query rows
 * (64 heads x 512 channels, bf16) attends in ONE softmax to its selected latent entries and its
 * window rows, the latent being both key and value ([C] sec. VI, VII, XII):
 *   qpos [batch*tq] token of each row; idx [batch*tq][k] selected entries (-1 = none), each
 *   visible at its row ((qpos + 1) / ratio entries are); window tokens [max(swa_begin[b],
 *   qpos - win + 1, 0), qpos] with win <= 128 (swa_begin may be NULL: 0); sm_scale 0 gives
 *   1/sqrt(512); ratio 1 or 2 (the entry rule of csa2_shape.ratio). The window ring must hold
 *   every window token of the call: with several rows per sequence, swa_cap >= win + the spread of
 *   their positions.
 *   out [batch*tq][64][512] bf16; out_f32 (same shape, fp32) and lse [batch*tq][64] (natural
 *   log) may be NULL. A row with no key gives out = 0 and lse = -inf.
 *   ws: a workspace of at least 256 bytes initialised by csa2_workspace_init (its status word
 *   receives CSA2_DEV_BAD_INDEX for an index < -1, not visible or >= cap, which is skipped, and
 *   CSA2_DEV_TIMEOUT if a tensor-core wait ran out); NULL leaves such bits unrecorded.
 * Precision: q is rounded bf16 -> fp16 (exact for 2^-14 <= |q| <= 65504), the dequantised latent
 * is exact in fp16, logits and sums are fp32, probabilities are rounded to fp16.
 * Returns CSA2_ERR_INVALID_ARG for null / misaligned pointers, k < 0 or k > 2048, win outside
 * 0..128 or a bad ratio.
 */
CSA2_API csa2_status csa2_latent_attend(const csa2_latent_cache* cache, int batch, int tq, const int64_t* qpos,
                                        const uint16_t* q, const int32_t* idx, int k, const int64_t* swa_begin,
                                        int win, int ratio, float sm_scale, uint16_t* out, float* out_f32, float* lse,
                                        void* ws, size_t ws_bytes, void* stream);

/*
 * Indexer of the pages' own shape ([C] sec. VII: the indexer key is ONE 128-channel MXFP4 key per
 * entry; the configuration list: 32 indexer query heads of dimension 128; [B] "Technical Approach",
 * [C] sec. VI: Top-k of the visible entries). For each of the batch*tq query rows:
 *   idx_q [batch*tq][hi][128] bf16 (16-byte aligned), 1 <= hi <= 64, quantised on the device with
 *   the MXFP4 rule of csa2_mxfp4_quantize; keys from cache->k_data / k_scale of sequence row / tq;
 *   score(p) = sum_h q_h . k_p, or sum_h max(0, q_h . k_p) with flags & CSA2_SCORE_RELU (the
 *   reading taken here; the pages give no formula) over the (qpos + 1) / ratio visible entries;
 *   out_idx [batch*tq][k]: the Top-k by score descending, ties to the lower position, in ascending
 *   position order, padded with -1 (a row with qpos < 0 gives all -1).
 * Scores are evaluated exactly (integer block dots times power-of-two scales, fp64 sums) whenever
 * the 32-channel block maxima of a row's query and keys lie within 2^38 of each other.
 * ws: at least csa2_latent_index_workspace_size(batch*tq, hi, max_ctx) bytes, 256-byte aligned and
 * cleared once after allocation with csa2_workspace_init (its first 4 bytes are the status word,
 * read and cleared by csa2_get_device_status; the rest is scratch); max_ctx bounds the visible
 * entries of every row: a row with more, or whose entries run past the capacity, sets
 * CSA2_DEV_BAD_POS and gives all -1. batch*tq <= 65535, 1 <= k <= 2048, ratio 1 or 2.
 */
CSA2_API csa2_status csa2_latent_index_workspace_size(int rows, int hi, int64_t max_ctx, size_t* bytes /* host */);
CSA2_API csa2_status csa2_latent_index_topk(const csa2_latent_cache* cache, int batch, int tq, const int64_t* qpos,
                                            const uint16_t* idx_q, int hi, int k, int ratio, int64_t max_ctx,
                                            uint32_t flags, int32_t* out_idx, void* ws, size_t ws_bytes,
                                            void* stream);

/* Synchronises `stream`, then reads and clears the device status word in `ws`.
 * *host_status receives the CSA2_DEV_* bits; returns CSA2_ERR_DEVICE if any bit was set. */
CSA2_API csa2_status csa2_get_device_status(void* ws, void* stream, int32_t* host_status /* host */);

#ifdef __cplusplus
}
#endif

#endif /* CSA2_H */
