// Draft block mask of LCSA on sm_100a: q block means, fp32 draft scores over
// the allowed key blocks and an exact top-k, one warp per (head, query block).
//
// Operation (FlashVSR code walk-through "FlashVSR 是怎么工作的", learn.html,
// section 2.2, third step): avgpool of q and k over the 128 tokens of a
// block, scores = mean_q . mean_k / sqrt(D), -inf outside the local block
// mask (reading notes 关键设计 3) and outside the block-causal set (关键设计
// 1), keep the top-k key blocks.  Ties go to the lower key index; the draft
// softmax of the page is monotone and does not change the selection, so it
// is not computed.
//
// Work per warp (8 rows per 256-thread CTA):
//  1. mean of the 2 x 8 x 8 query tokens: lane l owns dims [4l, 4l+4); one
//     coalesced 256-byte token row per warp load, fp32 sums in token order,
//     times 1/128 (deterministic);
//  2. one allowed candidate per lane: the fp32 dot product of the q mean with
//     the key block mean (written by the cache-append kernel, float4 loads
//     through L1, shared by the neighbouring rows of the CTA), times the scale;
//     only the allowed candidates are scored (at most 4 layers x 11 x 11 for
//     the default window), enumerated in ascending key index;
//  3. exact selection of the k = min(topk, allowed) best: scores are mapped to
//     32-bit keys whose unsigned order is descending score; a 4-pass radix
//     select (8 bits per pass, warp histogram in shared memory) finds the
//     k-th key T; the kept set is every key < T plus the first (lowest-index)
//     keys equal to T, written in ascending key index by a ballot compaction.

#include <cfloat>

#include "internal.h"
#include "ptx.cuh"
#include "../../include/lcsa.h"

namespace lcsa {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kFull = 0xffffffffu;

__device__ __forceinline__ void window_1d(int i, int n, int r, int mode, int &lo, int &hi) {
    // Allowed block range [lo, hi) along one axis of the block grid.
    if (r <= 0 || (mode == 0 && n <= r)) {
        lo = 0;
        hi = n;
        return;
    }
    const int h = r / 2;
    if (mode == 0) {  // Boundary-Preserved: window of r blocks shifted inside the grid
        lo = min(max(i - h, 0), n - r);
        hi = lo + r;
    } else {          // Boundary-Truncated: |i - j| <= r/2
        lo = max(i - h, 0);
        hi = min(i + h + 1, n);
    }
}

// 32-bit key whose unsigned ascending order is the descending order of the
// score (-0 is folded onto +0 so that the two tie).
__device__ __forceinline__ uint32_t desc_key(float score) {
    uint32_t u = __float_as_uint(score);
    if (u == 0x80000000u) u = 0u;
    const uint32_t ordered = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ~ordered;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Exact k-th smallest of keys[0, n) (1 <= k <= n): returns its value T and, in
// k_eq, how many keys equal to T belong to the k smallest.
__device__ uint32_t radix_select(const uint32_t *keys, int n, int k, uint32_t *hist, int lane, int &k_eq) {
    uint32_t prefix = 0, mask = 0;
    uint32_t k_rem = static_cast<uint32_t>(k);
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int b = lane; b < 256; b += 32) hist[b] = 0u;
        __syncwarp();
        for (int c = lane; c < n; c += 32) {
            const uint32_t key = keys[c];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncwarp();
        uint32_t cnt[8];
        uint32_t sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            cnt[e] = hist[lane * 8 + e];
            sum += cnt[e];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += v;
        }
        const uint32_t excl = incl - sum;
        const bool here = excl < k_rem && k_rem <= incl;
        const int src = __ffs(__ballot_sync(kFull, here)) - 1;
        uint32_t digit = 0, below = 0;
        if (here) {
            uint32_t run = excl;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (run + cnt[e] >= k_rem) {
                    digit = static_cast<uint32_t>(lane * 8 + e);
                    below = run;
                    break;
                }
                run += cnt[e];
            }
        }
        digit = __shfl_sync(kFull, digit, src);
        below = __shfl_sync(kFull, below, src);
        k_rem -= below;
        prefix |= digit << shift;
        mask |= 255u << shift;
        __syncwarp();
    }
    k_eq = static_cast<int>(k_rem);
    return prefix;
}

__global__ void __launch_bounds__(kThreads) draft_kernel(const DraftArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nq = a.q_layers * a.nblk;
    const int unit = blockIdx.x * kWarps + warp;  // (head, query block) row
    if (unit >= a.heads * nq) return;             // no CTA-wide barrier below
    // per-warp shared memory: q mean (512 B), radix histogram (1 KB), keys
    uint8_t *base = smem + static_cast<size_t>(warp) * (512 + 1024 + 4 * a.cand_cap);
    float *mq = reinterpret_cast<float *>(base);
    uint32_t *hist = reinterpret_cast<uint32_t *>(base + 512);
    uint32_t *keys = reinterpret_cast<uint32_t *>(base + 1536);

    const int h = unit / nq;
    const int qi = unit - h * nq;
    const int ql = qi / a.nblk;
    const int qb = qi - ql * a.nblk;
    const int qby = qb / a.grid_w;
    const int qbx = qb - qby * a.grid_w;

    // ---- 1. block mean of q
    {
        float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
        const size_t frame = static_cast<size_t>(h) * a.tq + ql * 2;
#pragma unroll 16
        for (int n = 0; n < kBlockTokens; ++n) {  // tokens in (t, y, x) row-major order
            const int t = n >> 6, y = (n >> 3) & 7, x = n & 7;
            const size_t tok = ((frame + t) * a.tok_h + qby * 8 + y) * a.tok_w + qbx * 8 + x;
            const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(a.q + tok * kHeadDim) + lane);
            acc0 += __uint_as_float(raw.x << 16);
            acc1 += __uint_as_float(raw.x & 0xFFFF0000u);
            acc2 += __uint_as_float(raw.y << 16);
            acc3 += __uint_as_float(raw.y & 0xFFFF0000u);
        }
        const float4 m = make_float4(acc0 * (1.0f / 128.0f), acc1 * (1.0f / 128.0f), acc2 * (1.0f / 128.0f),
                                     acc3 * (1.0f / 128.0f));
        reinterpret_cast<float4 *>(mq)[lane] = m;
        if (a.qmean) reinterpret_cast<float4 *>(a.qmean + static_cast<size_t>(unit) * kHeadDim)[lane] = m;
    }

    // ---- 2. allowed candidates (ascending key index) and their scores
    const int q_layer_abs = a.count - a.q_layers + ql;  // key layer of this query block
    int y0, y1, x0, x1;
    window_1d(qby, a.grid_h, a.local_range, a.local_mode, y0, y1);
    window_1d(qbx, a.grid_w, a.local_range, a.local_mode, x0, x1);
    const int nx = x1 - x0;
    const int per_layer = (y1 - y0) * nx;
    const int ncand = (q_layer_abs + 1) * per_layer;
    const int n_keys = a.count * a.nblk;
    float *srow = a.scores ? a.scores + static_cast<size_t>(unit) * n_keys : nullptr;
    if (srow) {
        for (int j = lane; j < n_keys; j += 32) srow[j] = -INFINITY;
    }
    __syncwarp();

    const float4 *mq4 = reinterpret_cast<const float4 *>(mq);
    for (int c = lane; c < ncand; c += 32) {
        const int layer = c / per_layer;
        const int rem = c - layer * per_layer;
        const int yy = y0 + rem / nx;
        const int xx = x0 + rem - (rem / nx) * nx;
        const int b = yy * a.grid_w + xx;
        int slot = a.oldest + layer;
        if (slot >= a.capacity) slot -= a.capacity;
        const float4 *mk =
            reinterpret_cast<const float4 *>(a.kmean + ((static_cast<size_t>(slot) * a.heads + h) * a.nblk + b) * kHeadDim);
        float dot = 0.f;
#pragma unroll 8
        for (int d4 = 0; d4 < kHeadDim / 4; ++d4) {
            const float4 kv = __ldg(mk + d4);
            const float4 qv = mq4[d4];
            dot = fmaf(qv.x, kv.x, dot);
            dot = fmaf(qv.y, kv.y, dot);
            dot = fmaf(qv.z, kv.z, dot);
            dot = fmaf(qv.w, kv.w, dot);
        }
        const float score = dot * a.scale;
        keys[c] = desc_key(score);
        if (srow) srow[layer * a.nblk + b] = score;
    }
    __syncwarp();

    // ---- 3. exact top-k: k-th key by radix select, then an ordered compaction
    const int k = min(a.topk, ncand);
    int k_eq = 0;
    const uint32_t T = radix_select(keys, ncand, k, hist, lane, k_eq);
    int32_t *out = a.kept_idx + static_cast<size_t>(unit) * a.topk;
    const uint32_t lt_mask = lanemask_lt();
    int out_pos = 0, eq_seen = 0;
    for (int base_c = 0; base_c < ncand; base_c += 32) {
        const int c = base_c + lane;
        const bool valid = c < ncand;
        const uint32_t key = valid ? keys[c] : 0xFFFFFFFFu;
        const bool eq = valid && key == T;
        const uint32_t eqb = __ballot_sync(kFull, eq);
        const int eq_rank = eq_seen + __popc(eqb & lt_mask);
        const bool take = valid && (key < T || (eq && eq_rank < k_eq));
        const uint32_t tb = __ballot_sync(kFull, take);
        if (take) {
            const int layer = c / per_layer;
            const int rem = c - layer * per_layer;
            const int yy = y0 + rem / nx;
            const int xx = x0 + rem - (rem / nx) * nx;
            out[out_pos + __popc(tb & lt_mask)] = layer * a.nblk + yy * a.grid_w + xx;
        }
        out_pos += __popc(tb);
        eq_seen += __popc(eqb);
    }
    for (int i = out_pos + lane; i < a.topk; i += 32) out[i] = -1;
    if (lane == 0) {
        a.kept_cnt[unit] = out_pos;
        if (out_pos != k && a.status) atomicOr(a.status, LCSA_ERR_BAD_INDEX);  // cannot happen
    }
}

}  // namespace

cudaError_t launch_draft(const DraftArgs &a, cudaStream_t stream) {
    const int rows = a.heads * a.q_layers * a.nblk;
    const int ctas = (rows + kWarps - 1) / kWarps;
    const size_t smem = static_cast<size_t>(kWarps) * (512 + 1024 + 4 * static_cast<size_t>(a.cand_cap));
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(draft_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    draft_kernel<<<ctas, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace lcsa
