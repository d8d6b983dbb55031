// Kernel argument blocks and launchers shared by the C-ABI layer and the kernels.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <utility>

namespace lcsa {

constexpr int kMaxDevices = 64;

// Facts about the current device, queried once per device and process: the
// LCSA status of its compute capability (only 10.0 is supported) and its SM
// count.  Returns null when the device cannot be queried.
struct DeviceInfo {
    int device;
    int status;  // LCSA_OK or LCSA_ERR_UNSUPPORTED_DEVICE
    int sms;
};
const DeviceInfo *current_device_info();

// Raises the dynamic shared memory limit of `kernel` on `dev` to `bytes`,
// calling the runtime only when the limit set so far on that device is lower.
// `done` holds the limit set so far per device (one array per kernel).
template <typename Kernel>
cudaError_t ensure_smem_limit(Kernel kernel, int dev, size_t bytes, std::atomic<int> (&done)[kMaxDevices]) {
    if (dev < 0 || dev >= kMaxDevices) {
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    }
    if (done[dev].load(std::memory_order_acquire) >= static_cast<int>(bytes)) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e == cudaSuccess) {
        int cur = done[dev].load(std::memory_order_relaxed);
        while (cur < static_cast<int>(bytes) &&
               !done[dev].compare_exchange_weak(cur, static_cast<int>(bytes), std::memory_order_release)) {
        }
    }
    return e;
}

// Launch of `kernel` on `stream`, optionally as a programmatic dependent of the
// stream's preceding kernel (it may start before that kernel completes and
// waits for it with griddepcontrol.wait where it reads its results).
template <typename... Params, typename... Args>
cudaError_t launch_kernel(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          bool pdl, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

constexpr int kBlockTokens = 128;
constexpr int kHeadDim = 128;
constexpr int kMaxCandidates = 4096;
constexpr uint64_t kWatchdogNs = 4000000000ull;  // 4 s per bounded wait

// Block-sparse attention (tcgen05 kernel).
struct AttnArgs {
    int32_t heads, grid_h, grid_w, nblk, q_layers, tq;  // tq = 2 * q_layers frames
    int32_t tok_h, tok_w;
    int32_t n_key_blocks;  // count * nblk
    int32_t capacity, oldest;
    int32_t topk;
    int32_t n_units;       // heads * q_layers * nblk
    float scale_log2;      // softmax scale * log2(e)
    const int32_t *kept_idx;
    const int32_t *kept_cnt;
    float *lse;            // may be null
    int32_t *status;       // may be null
    uint64_t timeout_ns;
    int32_t flags;
    // ceil(2^32 / d) for d = q_layers * nblk, nblk, grid_w: n / d = (n * m) >> 32
    // exactly while n * d <= 2^32 (checked by the caller for every n used)
    uint64_t m_nq, m_nblk, m_gw;
};

// Rotation of the Q tiles (a separate kernel argument: the kernel instance
// without rotation ignores it).
struct AttnRope {
    float base;            // 0: no rotation
    int32_t frame0;        // stream position of q's first frame
};

// Multiplier of the exact multiply-high division by d (1 <= d).
inline uint64_t div_magic_host(uint32_t d) { return ((1ull << 32) + d - 1) / d; }

cudaError_t launch_attention(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                             const CUtensorMap &tm_o, const AttnArgs &a, const AttnRope &rope, bool pdl, void *out,
                             const DeviceInfo &dev, cudaStream_t stream);

// Draft mask: q block means, scores over allowed candidates, top-k.
struct DraftArgs {
    const uint16_t *q;     // bf16 token layout
    const float *kmean;    // [cap][H][nblk][128]
    int32_t heads, grid_h, grid_w, nblk, q_layers, tq, tok_h, tok_w;
    int32_t capacity, oldest, count;
    int32_t fresh_layers;  // newest layers the preceding kernel may still be writing (PDL)
    int32_t local_range, local_mode, topk;
    int32_t cand_cap;      // most allowed candidates of a row, rounded up to 32
    float scale;
    int32_t *kept_idx;
    int32_t *kept_cnt;
    float *scores;         // may be null
    float *qmean;          // may be null
    int32_t *status;
    float rope_base;       // 0: no rotation of q
    int32_t rope_frame0;   // stream position of q's first frame
    uint16_t *q_rot;       // may be null: receives the rotated q (with rope_base != 0)
    // groups of horizontally adjacent query blocks (one CTA each) per block
    // row of a layer (set by launch_draft)
    int32_t groups_x;
};

cudaError_t launch_draft(const DraftArgs &a, bool pdl, const DeviceInfo &dev, cudaStream_t stream);

// Cache append: token layout -> block layout ring slots + k block means.
struct AppendArgs {
    uint16_t *k_cache;
    uint16_t *v_cache;
    float *kmean;
    int32_t heads, grid_h, grid_w, nblk, n_layers;
    int32_t first_slot, capacity;    // layer i of the chunk goes to slot (first_slot + i) % capacity
    uint64_t m_nblk, m_heads, m_gw;  // multiply-high multipliers of nblk, heads, grid_w
    int32_t *status;                 // may be null
    uint64_t timeout_ns;
    int32_t flags;
    float rope_base;                 // 0: no rotation of k
    int32_t rope_frame0;             // stream position of the chunk's first frame
};

// tm_k / tm_v: rank-4 maps over the chunk's k / v in token layout with a
// (128 dims, 8, 8, 2 frames) box, no swizzle (one box = one block, in block order).
cudaError_t launch_cache_append(const CUtensorMap &tm_k, const CUtensorMap &tm_v, const AppendArgs &a, bool pdl,
                                const DeviceInfo &dev, cudaStream_t stream);

// Kept lists of segment-masked dense attention: query tile i of segment s
// keeps key tiles start[s] .. start[s + 1] - 1.
constexpr int kMaxSegments = 256;
struct SegmentArgs {
    int32_t heads, tiles, topk, n_seg;
    int32_t start[kMaxSegments + 1];  // first tile of every segment, then the tile count
    int32_t *kept_idx;
    int32_t *kept_cnt;
};

cudaError_t launch_segment_mask(const SegmentArgs &a, cudaStream_t stream);

}  // namespace lcsa
