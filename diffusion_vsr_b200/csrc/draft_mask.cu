// Draft block mask of LCSA on sm_100a: q block means, fp32 draft scores over
// the allowed key blocks and top-k selection, one CTA per (head, query block).
//
// Operation (FlashVSR code walk-through "FlashVSR 是怎么工作的", learn.html,
// section 2.2, third step): avgpool of q and k over the 128 tokens of a
// block, scores = mean_q . mean_k / sqrt(D), -inf outside the local block
// mask (reading notes 关键设计 3) and outside the block-causal set (关键设计
// 1), keep the top-k key blocks.  Ties go to the lower key index; the draft
// softmax of the page is monotone and does not change the selection, so it
// is not computed.
//
// Work per CTA (256 threads):
//  1. mean of the 2 x 8 x 8 query tokens: 16-byte coalesced bf16 loads
//     straight from token layout (16 threads per 256-byte token row), fp32
//     partial sums reduced in shared memory in a fixed order, times 1/128;
//  2. scores only for the allowed candidates (at most 4 layers x 11 x 11 for
//     the default window), one warp per candidate: float4 loads of the key
//     block mean written by the cache-append kernel, warp-shuffle reduction;
//  3. a bitonic sort in shared memory of 64-bit keys
//     (descending score, ascending index), then a second small sort of the
//     kept indices so that the row is written in ascending key order.

#include <cfloat>

#include "internal.h"
#include "ptx.cuh"
#include "../../include/lcsa.h"

namespace lcsa {
namespace {

constexpr int kThreads = 256;

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

// Sort key: larger score first, then lower key index.  The float is mapped to
// an unsigned integer whose order matches the float order, then inverted.
__device__ __forceinline__ uint64_t make_key(float score, int j) {
    uint32_t u = __float_as_uint(score);
    if (u == 0x80000000u) u = 0u;  // -0 ties with +0
    const uint32_t ordered = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (static_cast<uint64_t>(~ordered) << 32) | static_cast<uint32_t>(j);
}

template <typename T>
__device__ __forceinline__ void bitonic_sort_smem(T *keys, int n_pow2) {
    for (int k = 2; k <= n_pow2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n_pow2; i += kThreads) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const T x = keys[i];
                    const T y = keys[ixj];
                    const bool up = (i & k) == 0;
                    if ((x > y) == up) {
                        keys[i] = y;
                        keys[ixj] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
}

__device__ __forceinline__ int next_pow2(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

__global__ void __launch_bounds__(kThreads) draft_kernel(const DraftArgs a) {
    // The partial-sum table of step 1 and the kept list of step 3 share the
    // storage of the sort keys (each is dead while the others are live).
    __shared__ __align__(16) uint64_t keys[kMaxCandidates];
    __shared__ __align__(16) float mq[kHeadDim];
    float(*red)[kHeadDim + 4] = reinterpret_cast<float(*)[kHeadDim + 4]>(keys);
    uint32_t *kept = reinterpret_cast<uint32_t *>(keys);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x;
    const int nq = a.q_layers * a.nblk;
    const int h = unit / nq;
    const int qi = unit - h * nq;
    const int ql = qi / a.nblk;
    const int qb = qi - ql * a.nblk;
    const int qby = qb / a.grid_w;
    const int qbx = qb - qby * a.grid_w;

    // ---- 1. block mean of q (fixed summation order -> deterministic)
    {
        const int chunk = tid & 15;  // dims [8*chunk, 8*chunk+8)
        const int sub = tid >> 4;    // token sub-group 0..15
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int n = sub + 16 * it;  // token of the block, (t, y, x) row-major
            const int t = n >> 6, y = (n >> 3) & 7, x = n & 7;
            const size_t tok = ((static_cast<size_t>(h) * a.tq + ql * 2 + t) * a.tok_h + qby * 8 + y) * a.tok_w +
                               qbx * 8 + x;
            const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(a.q + tok * kHeadDim + chunk * 8));
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] += __uint_as_float(w[e] << 16);
                acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red[sub][chunk * 8 + e] = acc[e];
    }
    __syncthreads();
    if (tid < kHeadDim) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < 16; ++g) s += red[g][tid];
        const float m = s * (1.0f / 128.0f);
        mq[tid] = m;
        if (a.qmean) a.qmean[static_cast<size_t>(unit) * kHeadDim + tid] = m;
    }

    // ---- 2. allowed candidates and their scores
    const int q_layer_abs = a.count - a.q_layers + ql;  // key layer of this query block
    int y0, y1, x0, x1;
    window_1d(qby, a.grid_h, a.local_range, a.local_mode, y0, y1);
    window_1d(qbx, a.grid_w, a.local_range, a.local_mode, x0, x1);
    const int ny = y1 - y0, nx = x1 - x0;
    const int per_layer = ny * nx;
    const int ncand = (q_layer_abs + 1) * per_layer;
    const int n_keys = a.count * a.nblk;
    float *srow = a.scores ? a.scores + static_cast<size_t>(unit) * n_keys : nullptr;
    if (srow) {
        for (int j = tid; j < n_keys; j += kThreads) srow[j] = -INFINITY;
    }
    __syncthreads();  // mq ready; -inf prefill ordered before the scattered scores

    const float4 mq4 = reinterpret_cast<const float4 *>(mq)[lane];
    for (int c = warp; c < ncand; c += kThreads / 32) {
        const int layer = c / per_layer;
        const int rem = c - layer * per_layer;
        const int yy = y0 + rem / nx;
        const int xx = x0 + rem % nx;
        const int b = yy * a.grid_w + xx;
        int slot = a.oldest + layer;
        if (slot >= a.capacity) slot -= a.capacity;
        const float4 mk = __ldg(reinterpret_cast<const float4 *>(
                                    a.kmean + ((static_cast<size_t>(slot) * a.heads + h) * a.nblk + b) * kHeadDim) +
                                lane);
        float part = mq4.x * mk.x;
        part = fmaf(mq4.y, mk.y, part);
        part = fmaf(mq4.z, mk.z, part);
        part = fmaf(mq4.w, mk.w, part);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        const float score = part * a.scale;
        if (lane == 0) {
            const int j = layer * a.nblk + b;
            keys[c] = make_key(score, j);
            if (srow) srow[j] = score;
        }
    }
    const int np = next_pow2(ncand);
    for (int c = ncand + tid; c < np; c += kThreads) keys[c] = ~0ull;
    __syncthreads();

    // ---- 3. top-k: sort (score desc, index asc), then the kept indices ascending
    bitonic_sort_smem(keys, np);
    const int k = min(a.topk, ncand);
    const int kp = next_pow2(k);
    // Gather the kept indices into registers before overwriting the keys.
    constexpr int kPerThread = kMaxCandidates / kThreads;
    uint32_t mine[kPerThread];
#pragma unroll
    for (int r = 0; r < kPerThread; ++r) {
        const int i = tid + r * kThreads;
        mine[r] = i < k ? static_cast<uint32_t>(keys[i]) : 0xFFFFFFFFu;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kPerThread; ++r) {
        const int i = tid + r * kThreads;
        if (i < kp) kept[i] = mine[r];
    }
    __syncthreads();
    bitonic_sort_smem(kept, kp);
    int32_t *out = a.kept_idx + static_cast<size_t>(unit) * a.topk;
    for (int i = tid; i < a.topk; i += kThreads) out[i] = i < k ? static_cast<int32_t>(kept[i]) : -1;
    if (tid == 0) a.kept_cnt[unit] = k;
}

}  // namespace

cudaError_t launch_draft(const DraftArgs &a, cudaStream_t stream) {
    const int units = a.heads * a.q_layers * a.nblk;
    draft_kernel<<<units, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace lcsa
