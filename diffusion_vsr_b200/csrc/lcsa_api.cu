// C ABI of the LCSA library: argument validation, TMA tensor maps, launches.
// Declarations and the meaning of every argument: include/lcsa.h.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "../../include/lcsa.h"

namespace {

using lcsa::kBlockTokens;
using lcsa::kHeadDim;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

}  // namespace

namespace lcsa {

// Facts about the current device, queried once per device (compute capability
// 10.0 = B200, sm_100a code, and the SM count).
const DeviceInfo *current_device_info() {
    static DeviceInfo infos[kMaxDevices];
    static std::atomic<bool> ready[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (ready[dev].load(std::memory_order_acquire)) return &infos[dev];
    std::lock_guard<std::mutex> lock(mu);
    if (!ready[dev].load(std::memory_order_relaxed)) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return nullptr;  // not cached: the next call queries again
        infos[dev].device = dev;
        infos[dev].status = (major == 10 && minor == 0) ? LCSA_OK : LCSA_ERR_UNSUPPORTED_DEVICE;
        infos[dev].sms = sms;
        ready[dev].store(true, std::memory_order_release);
    }
    return &infos[dev];
}

}  // namespace lcsa

namespace {

// The current device's facts, or an LCSA status when it cannot be used.
int device_of(const lcsa::DeviceInfo **info) {
    *info = lcsa::current_device_info();
    if (!*info) return LCSA_ERR_CUDA;
    return (*info)->status;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int window_of(const lcsa_kv_cache *c) { return c->window > 0 ? c->window : c->capacity; }

int check_cache(const lcsa_kv_cache *c) {
    if (!c || !c->k || !c->v || !c->kmean) return LCSA_ERR_INVALID_ARG;
    if (!aligned16(c->k) || !aligned16(c->v) || !aligned16(c->kmean)) return LCSA_ERR_INVALID_ARG;
    if (c->heads < 1 || c->grid_h < 1 || c->grid_w < 1 || c->capacity < 1) return LCSA_ERR_INVALID_ARG;
    if (c->window < 0 || c->window > c->capacity) return LCSA_ERR_INVALID_ARG;
    if (c->count < 0 || c->count > window_of(c) || c->oldest < 0 || c->oldest >= c->capacity)
        return LCSA_ERR_INVALID_ARG;
    if (c->appended < 0 || c->appended > c->capacity) return LCSA_ERR_INVALID_ARG;
    // every token row index of the ring must fit a signed 32-bit TMA coordinate
    const int64_t rows = static_cast<int64_t>(c->capacity) * c->heads * c->grid_h * c->grid_w * kBlockTokens;
    if (rows >= (int64_t(1) << 31)) return LCSA_ERR_INVALID_ARG;
    return LCSA_OK;
}

// A rotation is valid with base 0 (none) or a finite base > 1, and positions
// (frames of the call, token rows and columns) below 2^20, the range of the
// kernels' angle reduction.
bool rope_ok(const lcsa_rope *r, int64_t frames, int64_t tok_h, int64_t tok_w) {
    if (!r || r->base == 0.f) return true;
    if (!(r->base > 1.f) || std::isinf(r->base)) return false;
    const int64_t lim = int64_t(1) << 20;
    return r->frame0 >= 0 && static_cast<int64_t>(r->frame0) + frames <= lim && tok_h <= lim && tok_w <= lim;
}

int check_params(const lcsa_params *p, const lcsa_kv_cache *c) {
    if (!p) return LCSA_ERR_INVALID_ARG;
    if (p->head_dim != kHeadDim) return LCSA_ERR_INVALID_ARG;
    if (p->heads < 1 || p->grid_h < 1 || p->grid_w < 1 || p->q_layers < 1 || p->topk < 1) return LCSA_ERR_INVALID_ARG;
    if (p->local_mode != 0 && p->local_mode != 1) return LCSA_ERR_INVALID_ARG;
    if (p->local_range > 0 && (p->local_range % 2) == 0) return LCSA_ERR_INVALID_ARG;
    if (!(p->scale >= 0.f) || std::isinf(p->scale)) return LCSA_ERR_INVALID_ARG;
    if (p->heads != c->heads || p->grid_h != c->grid_h || p->grid_w != c->grid_w) return LCSA_ERR_INVALID_ARG;
    if (c->count < p->q_layers) return LCSA_ERR_INVALID_ARG;
    if (!rope_ok(&p->rope, 2 * static_cast<int64_t>(p->q_layers), 8LL * p->grid_h, 8LL * p->grid_w))
        return LCSA_ERR_INVALID_ARG;
    // frames * tokens must be addressable by 32-bit TMA coordinates
    const int64_t frames = static_cast<int64_t>(p->heads) * 2 * p->q_layers;
    if (frames >= (int64_t(1) << 31) || 8LL * p->grid_h >= (1 << 30) || 8LL * p->grid_w >= (1 << 30))
        return LCSA_ERR_INVALID_ARG;
    return LCSA_OK;
}

float eff_scale(const lcsa_params *p) {
    return p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->head_dim));
}

// Largest number of allowed key blocks of any query block (window x causal layers).
int64_t max_candidates(const lcsa_params *p, const lcsa_kv_cache *c) {
    auto span = [&](int n) -> int64_t {
        if (p->local_range <= 0) return n;
        if (p->local_mode == 0) return n <= p->local_range ? n : p->local_range;
        return std::min<int64_t>(n, p->local_range);  // truncated: at most r along an axis
    };
    return static_cast<int64_t>(c->count) * span(p->grid_h) * span(p->grid_w);
}

// Small per-thread cache of encoded tensor maps: a streaming caller passes the
// same buffers call after call, so their maps are encoded once.  Key: the kind
// of map, the base address and the extents.
enum MapKind { kTokenMap = 1, kChunkMap = 2, kRingMap = 3 };
struct MapKey {
    int kind;
    const void *base;
    int64_t a, b, c;
    bool operator==(const MapKey &o) const {
        return kind == o.kind && base == o.base && a == o.a && b == o.b && c == o.c;
    }
};
constexpr int kMapCacheSize = 16;
struct MapCache {
    MapKey key[kMapCacheSize] = {};
    CUtensorMap map[kMapCacheSize];
    int next = 0;
};

template <typename Encode>
bool cached_map(CUtensorMap *m, const MapKey &k, Encode encode) {
    thread_local MapCache cache;
    for (int i = 0; i < kMapCacheSize; ++i) {
        if (cache.key[i].kind != 0 && cache.key[i] == k) {
            *m = cache.map[i];
            return true;
        }
    }
    if (!encode(m)) return false;
    const int slot = cache.next;
    cache.next = (cache.next + 1) % kMapCacheSize;
    cache.key[slot] = k;
    cache.map[slot] = *m;
    return true;
}

// Rank-4 map over a token-layout bf16 tensor [H*T][8gh][8gw][128] with a
// (64 dims, 8, 8, 2 frames) box and 128-byte swizzle: one box pair is one
// (2,8,8) window block, so the partition is done by the copy engine.
bool encode_token_map(CUtensorMap *m, const void *base, int64_t frames, int tok_h, int tok_w) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(tok_w),
                                static_cast<cuuint64_t>(tok_h), static_cast<cuuint64_t>(frames)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHeadDim) * 2,
                                   static_cast<cuuint64_t>(kHeadDim) * 2 * tok_w,
                                   static_cast<cuuint64_t>(kHeadDim) * 2 * tok_w * tok_h};
    const cuuint32_t box[4] = {64, 8, 8, 2};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Rank-4 map over a chunk's k or v in token layout (dims, x, y, frames) with a
// whole-block box (128 dims, 8, 8, 2 frames), no swizzle: the box lands in
// shared memory in block order (intra index (t, y, x) row-major).
bool encode_chunk_map(CUtensorMap *m, const void *base, int64_t frames, int tok_h, int tok_w) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(tok_w),
                                static_cast<cuuint64_t>(tok_h), static_cast<cuuint64_t>(frames)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHeadDim) * 2,
                                   static_cast<cuuint64_t>(kHeadDim) * 2 * tok_w,
                                   static_cast<cuuint64_t>(kHeadDim) * 2 * tok_w * tok_h};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(kHeadDim), 8, 8, 2};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Rank-2 map over a block-layout ring [rows][128] with a (64 dims, 128 rows) box.
bool encode_ring_map(CUtensorMap *m, const void *base, int64_t rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kBlockTokens)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_token_map(CUtensorMap *m, const void *base, int64_t frames, int tok_h, int tok_w) {
    return cached_map(m, MapKey{kTokenMap, base, frames, tok_h, tok_w},
                      [&](CUtensorMap *o) { return encode_token_map(o, base, frames, tok_h, tok_w); });
}
bool make_chunk_map(CUtensorMap *m, const void *base, int64_t frames, int tok_h, int tok_w) {
    return cached_map(m, MapKey{kChunkMap, base, frames, tok_h, tok_w},
                      [&](CUtensorMap *o) { return encode_chunk_map(o, base, frames, tok_h, tok_w); });
}
bool make_ring_map(CUtensorMap *m, const void *base, int64_t rows) {
    return cached_map(m, MapKey{kRingMap, base, rows, 0, 0},
                      [&](CUtensorMap *o) { return encode_ring_map(o, base, rows); });
}

}  // namespace

extern "C" {

int lcsa_version(void) { return 102; }

const char *lcsa_status_string(int code) {
    switch (code) {
        case LCSA_OK: return "LCSA_OK";
        case LCSA_ERR_INVALID_ARG: return "LCSA_ERR_INVALID_ARG";
        case LCSA_ERR_UNSUPPORTED_DEVICE: return "LCSA_ERR_UNSUPPORTED_DEVICE";
        case LCSA_ERR_CUDA: return "LCSA_ERR_CUDA";
        case LCSA_ERR_TIMEOUT: return "LCSA_ERR_TIMEOUT";
        case LCSA_ERR_BAD_INDEX: return "LCSA_ERR_BAD_INDEX";
        case LCSA_ERR_TIMEOUT | LCSA_ERR_BAD_INDEX: return "LCSA_ERR_TIMEOUT|LCSA_ERR_BAD_INDEX";
        default: return "LCSA_ERR_UNKNOWN";
    }
}

int lcsa_cache_append(lcsa_kv_cache *cache, const void *k_tok, const void *v_tok, int32_t n_layers, int32_t flags,
                      const lcsa_rope *rope, int32_t *d_status, void *stream) {
    int rc = check_cache(cache);
    if (rc != LCSA_OK) return rc;
    if (!k_tok || !v_tok || !aligned16(k_tok) || !aligned16(v_tok)) return LCSA_ERR_INVALID_ARG;
    const int window = window_of(cache);
    if (n_layers < 1 || n_layers > window) return LCSA_ERR_INVALID_ARG;
    if (!rope_ok(rope, 2 * static_cast<int64_t>(n_layers), 8LL * cache->grid_h, 8LL * cache->grid_w))
        return LCSA_ERR_INVALID_ARG;
    const bool pdl = (flags & LCSA_FLAG_PDL) != 0;
    // overlapping the previous step is safe only while the new layers go to spare slots
    if (pdl && n_layers > cache->capacity - window) return LCSA_ERR_INVALID_ARG;
    const lcsa::DeviceInfo *dev = nullptr;
    if ((rc = device_of(&dev)) != LCSA_OK) return rc;

    const int64_t frames = static_cast<int64_t>(cache->heads) * 2 * n_layers;
    const int64_t units = static_cast<int64_t>(n_layers) * cache->heads * cache->grid_h * cache->grid_w;
    const int64_t nblk64 = static_cast<int64_t>(cache->grid_h) * cache->grid_w;
    // unit decomposition by multiply-high division, exact while dividend x divisor <= 2^32
    if (units * nblk64 > (1ll << 32) || static_cast<int64_t>(n_layers) * cache->heads * cache->heads > (1ll << 32) ||
        nblk64 * cache->grid_w > (1ll << 32))
        return LCSA_ERR_INVALID_ARG;
    CUtensorMap tk, tv;
    if (!make_chunk_map(&tk, k_tok, frames, 8 * cache->grid_h, 8 * cache->grid_w) ||
        !make_chunk_map(&tv, v_tok, frames, 8 * cache->grid_h, 8 * cache->grid_w))
        return LCSA_ERR_CUDA;

    lcsa::AppendArgs a{};
    a.k_cache = static_cast<uint16_t *>(cache->k);
    a.v_cache = static_cast<uint16_t *>(cache->v);
    a.kmean = cache->kmean;
    a.heads = cache->heads;
    a.grid_h = cache->grid_h;
    a.grid_w = cache->grid_w;
    a.nblk = cache->grid_h * cache->grid_w;
    a.n_layers = n_layers;
    a.m_nblk = lcsa::div_magic_host(static_cast<uint32_t>(a.nblk));
    a.m_heads = lcsa::div_magic_host(static_cast<uint32_t>(a.heads));
    a.m_gw = lcsa::div_magic_host(static_cast<uint32_t>(a.grid_w));
    a.status = d_status;
    a.timeout_ns = lcsa::kWatchdogNs;
    a.flags = flags;
    a.rope_base = rope ? rope->base : 0.f;
    a.rope_frame0 = rope ? rope->frame0 : 0;
    // each new layer goes to the slot after the newest one (layer i of the chunk
    // to first_slot + i); once `window` layers are resident the oldest is dropped
    a.first_slot = (cache->oldest + cache->count) % cache->capacity;
    a.capacity = cache->capacity;
    const int count = std::min(window, cache->count + n_layers);
    const int oldest = (cache->oldest + (cache->count + n_layers - count)) % cache->capacity;
    if (lcsa::launch_cache_append(tk, tv, a, pdl, *dev, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return LCSA_ERR_CUDA;
    cache->oldest = oldest;
    cache->count = count;
    cache->appended = n_layers;
    return LCSA_OK;
}

int lcsa_draft_mask(const lcsa_params *p, const void *q_tok, const lcsa_kv_cache *cache, int32_t *kept_idx,
                    int32_t *kept_cnt, float *scores_opt, float *qmean_opt, void *q_rot_opt, int32_t *d_status,
                    void *stream) {
    int rc = check_cache(cache);
    if (rc != LCSA_OK) return rc;
    if ((rc = check_params(p, cache)) != LCSA_OK) return rc;
    if (!q_tok || !aligned16(q_tok) || !kept_idx || !kept_cnt) return LCSA_ERR_INVALID_ARG;
    if (q_rot_opt) {
        // the rotated copy of q: only with a rotation, aligned, and apart from q
        const size_t bytes = static_cast<size_t>(p->heads) * 2 * p->q_layers * 64 * p->grid_h * p->grid_w *
                             LCSA_HEAD_DIM * 2;
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(q_tok), b0 = reinterpret_cast<uintptr_t>(q_rot_opt);
        if (p->rope.base == 0.f || !aligned16(q_rot_opt) || (b0 < a0 + bytes && a0 < b0 + bytes))
            return LCSA_ERR_INVALID_ARG;
    }
    const int64_t cand = max_candidates(p, cache);
    if (cand > lcsa::kMaxCandidates) return LCSA_ERR_INVALID_ARG;
    const lcsa::DeviceInfo *dev = nullptr;
    if ((rc = device_of(&dev)) != LCSA_OK) return rc;

    lcsa::DraftArgs a{};
    a.q = static_cast<const uint16_t *>(q_tok);
    a.kmean = cache->kmean;
    a.heads = p->heads;
    a.grid_h = p->grid_h;
    a.grid_w = p->grid_w;
    a.nblk = p->grid_h * p->grid_w;
    a.q_layers = p->q_layers;
    a.tq = 2 * p->q_layers;
    a.tok_h = 8 * p->grid_h;
    a.tok_w = 8 * p->grid_w;
    a.capacity = cache->capacity;
    a.oldest = cache->oldest;
    a.count = cache->count;
    // chained after an append (LCSA_FLAG_PDL), the layers it wrote are read only
    // after waiting for it: the query layers, and every layer of that append
    a.fresh_layers = std::max(p->q_layers, cache->appended);
    a.local_range = p->local_range;
    a.local_mode = p->local_mode;
    a.topk = p->topk;
    a.cand_cap = static_cast<int32_t>((cand + 31) / 32 * 32);
    a.scale = eff_scale(p);
    a.kept_idx = kept_idx;
    a.kept_cnt = kept_cnt;
    a.scores = scores_opt;
    a.qmean = qmean_opt;
    a.status = d_status;
    a.rope_base = p->rope.base;
    a.rope_frame0 = p->rope.frame0;
    a.q_rot = static_cast<uint16_t *>(q_rot_opt);
    if (lcsa::launch_draft(a, (p->flags & LCSA_FLAG_PDL) != 0, *dev, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return LCSA_ERR_CUDA;
    return LCSA_OK;
}

int lcsa_attention(const lcsa_params *p, const void *q_tok, const lcsa_kv_cache *cache, const int32_t *kept_idx,
                   const int32_t *kept_cnt, void *out_tok, float *lse_opt, int32_t *d_status, void *stream) {
    int rc = check_cache(cache);
    if (rc != LCSA_OK) return rc;
    if ((rc = check_params(p, cache)) != LCSA_OK) return rc;
    if (!q_tok || !out_tok || !aligned16(q_tok) || !aligned16(out_tok) || !kept_idx || !kept_cnt)
        return LCSA_ERR_INVALID_ARG;
    if (q_tok == out_tok) return LCSA_ERR_INVALID_ARG;
    const lcsa::DeviceInfo *dev = nullptr;
    if ((rc = device_of(&dev)) != LCSA_OK) return rc;

    const int nblk = p->grid_h * p->grid_w;
    const int64_t frames = static_cast<int64_t>(p->heads) * 2 * p->q_layers;
    const int64_t rows = static_cast<int64_t>(cache->capacity) * cache->heads * nblk * kBlockTokens;
    CUtensorMap tq, tk, tv, to;
    if (!make_token_map(&tq, q_tok, frames, 8 * p->grid_h, 8 * p->grid_w) || !make_ring_map(&tk, cache->k, rows) ||
        !make_ring_map(&tv, cache->v, rows) || !make_token_map(&to, out_tok, frames, 8 * p->grid_h, 8 * p->grid_w))
        return LCSA_ERR_CUDA;

    lcsa::AttnArgs a{};
    a.heads = p->heads;
    a.grid_h = p->grid_h;
    a.grid_w = p->grid_w;
    a.nblk = nblk;
    a.q_layers = p->q_layers;
    a.tq = 2 * p->q_layers;
    a.tok_h = 8 * p->grid_h;
    a.tok_w = 8 * p->grid_w;
    a.n_key_blocks = cache->count * nblk;
    a.capacity = cache->capacity;
    a.oldest = cache->oldest;
    a.topk = p->topk;
    a.n_units = p->heads * p->q_layers * nblk;
    a.scale_log2 = eff_scale(p) * 1.4426950408889634f;
    a.kept_idx = kept_idx;
    a.kept_cnt = kept_cnt;
    a.lse = lse_opt;
    a.status = d_status;
    a.timeout_ns = lcsa::kWatchdogNs;
    a.flags = p->flags;
    // multiply-high division stays exact while every dividend times its divisor is <= 2^32
    const int64_t nq = static_cast<int64_t>(p->q_layers) * nblk;
    if (static_cast<int64_t>(a.n_units) * nq > (1ll << 32) || static_cast<int64_t>(a.n_key_blocks) * nblk > (1ll << 32))
        return LCSA_ERR_INVALID_ARG;
    a.m_nq = lcsa::div_magic_host(static_cast<uint32_t>(nq));
    a.m_nblk = lcsa::div_magic_host(static_cast<uint32_t>(nblk));
    a.m_gw = lcsa::div_magic_host(static_cast<uint32_t>(p->grid_w));
    const lcsa::AttnRope rope{p->rope.base, p->rope.frame0};
    if (lcsa::launch_attention(tq, tk, tv, to, a, rope, (p->flags & LCSA_FLAG_PDL) != 0, out_tok, *dev,
                               static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return LCSA_ERR_CUDA;
    return LCSA_OK;
}

int lcsa_segment_mask(const int32_t *seg_tiles, int32_t n_seg, int32_t heads, int32_t topk, int32_t *kept_idx,
                      int32_t *kept_cnt, void *stream) {
    if (!seg_tiles || n_seg < 1 || n_seg > lcsa::kMaxSegments || heads < 1 || topk < 1) return LCSA_ERR_INVALID_ARG;
    if (!kept_idx || !kept_cnt || (reinterpret_cast<uintptr_t>(kept_idx) & 3u) ||
        (reinterpret_cast<uintptr_t>(kept_cnt) & 3u))
        return LCSA_ERR_INVALID_ARG;
    lcsa::SegmentArgs a{};
    int64_t tiles = 0;
    for (int s = 0; s < n_seg; ++s) {
        if (seg_tiles[s] < 1 || seg_tiles[s] > topk) return LCSA_ERR_INVALID_ARG;
        a.start[s] = static_cast<int32_t>(tiles);
        tiles += seg_tiles[s];
        if (tiles * heads >= (int64_t(1) << 31) || tiles * heads * topk >= (int64_t(1) << 40))
            return LCSA_ERR_INVALID_ARG;
    }
    a.start[n_seg] = static_cast<int32_t>(tiles);
    a.heads = heads;
    a.tiles = static_cast<int32_t>(tiles);
    a.topk = topk;
    a.n_seg = n_seg;
    a.kept_idx = kept_idx;
    a.kept_cnt = kept_cnt;
    const lcsa::DeviceInfo *dev = nullptr;
    int rc = device_of(&dev);
    if (rc != LCSA_OK) return rc;
    if (lcsa::launch_segment_mask(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) return LCSA_ERR_CUDA;
    return LCSA_OK;
}

}  // extern "C"
