// Draft block mask of LCSA on sm_100a: q block means, fp32 draft scores over
// the allowed key blocks and an exact top-k.
//
// Operation (FlashVSR code walk-through "FlashVSR 是怎么工作的", learn.html,
// section 2.2, third step): avgpool of q and k over the 128 tokens of a
// block, scores = mean_q . mean_k / sqrt(D), -inf outside the local block
// mask (reading notes 关键设计 3) and outside the block-causal set (关键设计
// 1), keep the top-k key blocks.  Ties go to the lower key index; the draft
// softmax of the page is monotone and does not change the selection, so it
// is not computed.
//
// One CTA (8 warps) per group of 8 consecutive query blocks of one head and
// block-layer.  Neighbouring query blocks have overlapping windows, so the
// key-block means are read once per group:
//  1. warp w computes the mean of query block w: lane l owns dims
//     [4l, 4l+4), one coalesced 256-byte token row per load, 32 loads in
//     flight, fp32 sums in token order, times 1/128 (deterministic);
//  2. one candidate of the union of the 8 windows per thread, enumerated in
//     ascending key index: its 512-byte mean is loaded once and dotted (fp32)
//     with every query mean of the group whose own window contains it;
//     candidates outside a block's window get a sentinel key;
//  3. warp w selects for query block w the k = min(topk, allowed) best
//     exactly: scores become 32-bit keys whose unsigned order is descending
//     score; a 4-pass radix select (8 bits per pass, warp histogram in shared
//     memory) finds the k-th key T; the kept set is every key < T plus the
//     first (lowest-index) keys equal to T, written in ascending key index by
//     a ballot compaction.

#include <cfloat>

#include "internal.h"
#include "ptx.cuh"
#include "../../include/lcsa.h"

namespace lcsa {
namespace {

constexpr int kG = 8;  // query blocks per CTA (one warp each)
constexpr int kThreads = kG * 32;
constexpr uint32_t kFull = 0xffffffffu;
constexpr uint32_t kNotCandidate = 0xFFFFFFFFu;

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
// score (-0 is folded onto +0 so that the two tie).  Finite scores never map
// to the sentinel 0xFFFFFFFF.
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

struct DraftSmem {
    __align__(16) float mq[kG][kHeadDim];
    uint32_t hist[kG][256];
    int win[kG][4];  // y0, y1, x0, x1 of each block's window; y0 = -1 for no block
};

// Exact k-th smallest of the candidate keys in keys[0, n) (sentinels skipped,
// 1 <= k <= candidates): returns its value; k_eq = how many keys equal to it
// belong to the k smallest.  Whole warp.
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
            if (key != kNotCandidate && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
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
    __shared__ DraftSmem sm;
    extern __shared__ uint32_t keys[];  // [kG][cand_cap]
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int groups_per_layer = (a.nblk + kG - 1) / kG;
    int cta = blockIdx.x;
    const int gi = cta % groups_per_layer;
    cta /= groups_per_layer;
    const int ql = cta % a.q_layers;
    const int h = cta / a.q_layers;
    const int qb = gi * kG + warp;  // this warp's query block (within its layer)
    const bool has_block = qb < a.nblk;
    const int unit = (h * a.q_layers + ql) * a.nblk + qb;  // its (head, query block) row

    // ---- 1. block mean of q (warp w: query block w)
    const int qby = has_block ? qb / a.grid_w : 0;
    const int qbx = has_block ? qb - qby * a.grid_w : 0;
    if (has_block) {
        const size_t frame = static_cast<size_t>(h) * a.tq + ql * 2;
        float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll 1
        for (int n0 = 0; n0 < kBlockTokens; n0 += 32) {
            uint2 raw[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {  // tokens in (t, y, x) row-major order
                const int n = n0 + i;
                const int t = n >> 6, y = (n >> 3) & 7, x = n & 7;
                const size_t tok = ((frame + t) * a.tok_h + qby * 8 + y) * a.tok_w + qbx * 8 + x;
                raw[i] = __ldg(reinterpret_cast<const uint2 *>(a.q + tok * kHeadDim) + lane);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                acc0 += __uint_as_float(raw[i].x << 16);
                acc1 += __uint_as_float(raw[i].x & 0xFFFF0000u);
                acc2 += __uint_as_float(raw[i].y << 16);
                acc3 += __uint_as_float(raw[i].y & 0xFFFF0000u);
            }
        }
        const float4 m = make_float4(acc0 * (1.0f / 128.0f), acc1 * (1.0f / 128.0f), acc2 * (1.0f / 128.0f),
                                     acc3 * (1.0f / 128.0f));
        reinterpret_cast<float4 *>(sm.mq[warp])[lane] = m;
        if (a.qmean) reinterpret_cast<float4 *>(a.qmean + static_cast<size_t>(unit) * kHeadDim)[lane] = m;
        if (lane == 0) {
            int y0, y1, x0, x1;
            window_1d(qby, a.grid_h, a.local_range, a.local_mode, y0, y1);
            window_1d(qbx, a.grid_w, a.local_range, a.local_mode, x0, x1);
            sm.win[warp][0] = y0;
            sm.win[warp][1] = y1;
            sm.win[warp][2] = x0;
            sm.win[warp][3] = x1;
        }
    } else if (lane == 0) {
        sm.win[warp][0] = -1;
        sm.win[warp][1] = sm.win[warp][2] = sm.win[warp][3] = 0;
    }
    const int q_layer_abs = a.count - a.q_layers + ql;  // key layer of these query blocks
    const int n_layers = q_layer_abs + 1;
    const int n_keys = a.count * a.nblk;
    float *srow = (a.scores && has_block) ? a.scores + static_cast<size_t>(unit) * n_keys : nullptr;
    if (srow) {
        for (int j = lane; j < n_keys; j += 32) srow[j] = -INFINITY;
    }
    __syncthreads();  // means, windows and the -inf prefill are visible to every warp

    // union of the windows of the group (bounding box per layer)
    int uy0 = a.grid_h, uy1 = 0, ux0 = a.grid_w, ux1 = 0;
#pragma unroll
    for (int r = 0; r < kG; ++r) {
        if (sm.win[r][0] < 0) continue;
        uy0 = min(uy0, sm.win[r][0]);
        uy1 = max(uy1, sm.win[r][1]);
        ux0 = min(ux0, sm.win[r][2]);
        ux1 = max(ux1, sm.win[r][3]);
    }
    const int unx = ux1 - ux0;
    const int uper = (uy1 - uy0) * unx;
    const int ucnt = n_layers * uper;  // <= cand_cap

    // ---- 2. scores: one union candidate per thread, its mean read once
    for (int u = tid; u < ucnt; u += kThreads) {
        const int layer = u / uper;
        const int rem = u - layer * uper;
        const int yy = uy0 + rem / unx;
        const int xx = ux0 + rem - (rem / unx) * unx;
        const int b = yy * a.grid_w + xx;
        int slot = a.oldest + layer;
        if (slot >= a.capacity) slot -= a.capacity;
        const float4 *mk =
            reinterpret_cast<const float4 *>(a.kmean + ((static_cast<size_t>(slot) * a.heads + h) * a.nblk + b) * kHeadDim);
        bool in[kG];
#pragma unroll
        for (int r = 0; r < kG; ++r)
            in[r] = sm.win[r][0] <= yy && yy < sm.win[r][1] && sm.win[r][2] <= xx && xx < sm.win[r][3];
        float dot[kG];
#pragma unroll
        for (int r = 0; r < kG; ++r) dot[r] = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // 16 independent 16-byte loads in flight
            float4 kv[16];
#pragma unroll
            for (int d4 = 0; d4 < 16; ++d4) kv[d4] = __ldg(mk + half * 16 + d4);
#pragma unroll
            for (int r = 0; r < kG; ++r) {
                if (!in[r]) continue;
                const float4 *mq4 = reinterpret_cast<const float4 *>(sm.mq[r]) + half * 16;
#pragma unroll
                for (int d4 = 0; d4 < 16; ++d4) {
                    const float4 qv = mq4[d4];
                    dot[r] = fmaf(qv.x, kv[d4].x, dot[r]);
                    dot[r] = fmaf(qv.y, kv[d4].y, dot[r]);
                    dot[r] = fmaf(qv.z, kv[d4].z, dot[r]);
                    dot[r] = fmaf(qv.w, kv[d4].w, dot[r]);
                }
            }
        }
        const int j = layer * a.nblk + b;
#pragma unroll
        for (int r = 0; r < kG; ++r) {
            const float score = dot[r] * a.scale;
            keys[r * a.cand_cap + u] = in[r] ? desc_key(score) : kNotCandidate;
            if (in[r] && a.scores) {
                const int ur = (h * a.q_layers + ql) * a.nblk + gi * kG + r;
                a.scores[static_cast<size_t>(ur) * n_keys + j] = score;
            }
        }
    }
    __syncthreads();
    if (!has_block) return;

    // ---- 3. exact top-k of this warp's block, written in ascending key index
    const uint32_t *mykeys = keys + warp * a.cand_cap;
    const int ncand =
        n_layers * (sm.win[warp][1] - sm.win[warp][0]) * (sm.win[warp][3] - sm.win[warp][2]);  // >= 1
    const int k = min(a.topk, ncand);
    int k_eq = 0;
    const uint32_t T = radix_select(mykeys, ucnt, k, sm.hist[warp], lane, k_eq);
    int32_t *out = a.kept_idx + static_cast<size_t>(unit) * a.topk;
    const uint32_t lt_mask = lanemask_lt();
    int out_pos = 0, eq_seen = 0;
    for (int base_u = 0; base_u < ucnt; base_u += 32) {
        const int u = base_u + lane;
        const uint32_t key = u < ucnt ? mykeys[u] : kNotCandidate;
        const bool valid = key != kNotCandidate;
        const bool eq = valid && key == T;
        const uint32_t eqb = __ballot_sync(kFull, eq);
        const int eq_rank = eq_seen + __popc(eqb & lt_mask);
        const bool take = valid && (key < T || (eq && eq_rank < k_eq));
        const uint32_t tb = __ballot_sync(kFull, take);
        if (take) {
            const int layer = u / uper;
            const int rem = u - layer * uper;
            const int yy = uy0 + rem / unx;
            const int xx = ux0 + rem - (rem / unx) * unx;
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
    const int groups = a.heads * a.q_layers * ((a.nblk + kG - 1) / kG);
    const size_t smem = static_cast<size_t>(kG) * 4 * static_cast<size_t>(a.cand_cap);
    if (smem > 48 * 1024 - sizeof(DraftSmem)) {
        cudaError_t e = cudaFuncSetAttribute(draft_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    draft_kernel<<<groups, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace lcsa
