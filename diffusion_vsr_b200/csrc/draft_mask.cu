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
// One CTA of 8 warps per group of one or two horizontally adjacent query
// blocks (one head, query layer and block row; two on large grids), so that
// every SM holds several groups at once and each phase is a single round trip
// to memory:
//  1. block means of q, one block of the group after the other: warp w sums
//     tokens [16w, 16w + 16) of the block (16-byte loads, a half-warp per
//     token, 8 tokens in flight per lane), the 8 partial sums are added in a
//     fixed tree order, times 1/128 (deterministic); with RoPE every pair of q
//     is rotated (and rounded to bf16) before it is summed, from a table of
//     the block's (cos, sin) that the CTA builds while its loads are in
//     flight, and the rotated q is stored for the attention when the caller
//     asks for it;
//  2. the union of the group's windows (same window rows, overlapping column
//     windows), enumerated layer-major, eight keys per warp at a time: each
//     512-byte key mean is one coalesced warp load, dotted with every block's
//     q mean in fp32 (per-lane partial products, then a fixed reduce-scatter
//     butterfly that leaves one (block, key) sum per lane); a pair whose key
//     lies in the block's window becomes that block's candidate, stored at its
//     position in ascending key index (layer, window row, window column);
//     chained after the chunk's cache append, the keys of the older layers
//     are scored while the append still runs, those of the chunk's own layers
//     after it;
//  3. exact top-k of every block of the group (two blocks: one half of the
//     CTA each, at the same time): scores become 32-bit keys
//     whose unsigned order is the descending score order; a radix select of
//     up to 4 passes (8 bits per pass, block histogram in shared memory, one
//     atomic per distinct bin and warp; it stops after the pass whose bin
//     holding the k-th key is kept whole) finds the k-th key T; the team's
//     first warp writes every key < T plus the first (lowest-index) keys
//     equal to T, in ascending key index, by a ballot compaction.

#include <cfloat>
#include <climits>

#include "internal.h"
#include "ptx.cuh"
#include "rope.cuh"
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

// Exact n / d for 0 <= n, d < 2^16 (d >= 1) with m = ceil(2^32 / d): the
// rounding excess of n m / 2^32 over n / d is below n / 2^32 < 1 / d.
// ceil(2^32 / d) = floor((2^32 - 1) / d) + 1 for every d >= 1, a 32-bit division.
__device__ __forceinline__ uint64_t div_magic(uint32_t d) { return static_cast<uint64_t>(0xFFFFFFFFu / d) + 1u; }
__device__ __forceinline__ int div_by(int n, uint64_t m) {
    return static_cast<int>((static_cast<uint64_t>(static_cast<uint32_t>(n)) * m) >> 32);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// (cos, sin) of the block's tokens: 2 frames x 22 time pairs, then 8 token rows
// x 21 row pairs, then 8 token columns x 21 column pairs.
constexpr int kTabY = 2 * kRopePairsT;
constexpr int kTabX = kTabY + 8 * kRopePairsY;
constexpr int kTabEntries = kTabX + 8 * kRopePairsY;

// Per-CTA shared memory: the per-warp partial sums of q, the group's q means,
// the radix histogram and its hand-over words, and with RoPE the block's
// (cos, sin) table and the band frequencies.
template <bool kRope>
struct RopeSmem {};
template <>
struct RopeSmem<true> {
    float2 tab[kTabEntries];
    double freq[64];  // w of every dimension pair
};
template <bool kRope, int kR>
struct DraftSmem : RopeSmem<kRope> {
    __align__(16) float part[kWarps][kHeadDim];  // per-warp partial sums of q
    __align__(16) float mq[kR][kHeadDim];
    uint32_t hist[kR][256];  // radix histogram of each select team
    uint32_t digit[kR], below[kR], whole[kR];
};

// Dot products of 8 keys with the group's kR q means, summed over the 32 lanes
// (lane l holds dims 4l .. 4l + 3): d[8 b + u] is this lane's partial for block
// b and key u.  A fixed reduce-scatter (xor 16, 8, ... while more than one
// value is left per lane) then a butterfly over the remaining lane bits
// leaves in the lane the full sum of value reduce_index<kR>(lane).
template <int kR>
__device__ __forceinline__ float reduce_group(const float (&d)[8 * kR], int lane) {
    float v;
    if constexpr (kR == 1) {
        float d4[4], d2[2];
        bool hi = lane & 16;
#pragma unroll
        for (int i = 0; i < 4; ++i) d4[i] = (hi ? d[i + 4] : d[i]) + __shfl_xor_sync(kFull, hi ? d[i] : d[i + 4], 16);
        hi = lane & 8;
#pragma unroll
        for (int i = 0; i < 2; ++i) d2[i] = (hi ? d4[i + 2] : d4[i]) + __shfl_xor_sync(kFull, hi ? d4[i] : d4[i + 2], 8);
        hi = lane & 4;
        v = (hi ? d2[1] : d2[0]) + __shfl_xor_sync(kFull, hi ? d2[0] : d2[1], 4);
        v += __shfl_xor_sync(kFull, v, 2);
        v += __shfl_xor_sync(kFull, v, 1);
    } else {
        static_assert(kR == 2, "groups of one or two blocks");
        float d8[8], d4[4], d2[2];
        bool hi = lane & 16;
#pragma unroll
        for (int i = 0; i < 8; ++i) d8[i] = (hi ? d[i + 8] : d[i]) + __shfl_xor_sync(kFull, hi ? d[i] : d[i + 8], 16);
        hi = lane & 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) d4[i] = (hi ? d8[i + 4] : d8[i]) + __shfl_xor_sync(kFull, hi ? d8[i] : d8[i + 4], 8);
        hi = lane & 4;
#pragma unroll
        for (int i = 0; i < 2; ++i) d2[i] = (hi ? d4[i + 2] : d4[i]) + __shfl_xor_sync(kFull, hi ? d4[i] : d4[i + 2], 4);
        hi = lane & 2;
        v = (hi ? d2[1] : d2[0]) + __shfl_xor_sync(kFull, hi ? d2[0] : d2[1], 2);
        v += __shfl_xor_sync(kFull, v, 1);
    }
    return v;
}
// Value (8 b + u) that reduce_group leaves in a lane, and whether the lane is
// the first of those holding it.
template <int kR>
__device__ __forceinline__ int reduce_index(int lane) {
    if constexpr (kR == 1) return ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
    return ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
}
template <int kR>
__device__ __forceinline__ bool reduce_writer(int lane) {
    return (lane & (kR == 1 ? 3 : 1)) == 0;
}

// One CTA per group of kR horizontally adjacent query blocks (one head, query
// layer and block row).  kRope: q is rotated (RoPE) before its block means
// (and, when a.q_rot is set, the rotated q is stored there).
template <bool kRope, int kR>
__global__ void __launch_bounds__(kThreads, kR == 1 ? 6 : 4) draft_kernel(const DraftArgs a) {
    __shared__ DraftSmem<kRope, kR> sm;
    extern __shared__ uint32_t keys[];  // [kR][cand_cap]
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    int t = blockIdx.x;  // (head, query layer, block row, group)
    const int hq = t / (a.grid_h * a.groups_x);
    t -= hq * a.grid_h * a.groups_x;
    const int qby = t / a.groups_x;
    const int qbx0 = (t - qby * a.groups_x) * kR;
    const int nb = min(kR, a.grid_w - qbx0);  // blocks of the group: qbx0 .. qbx0 + nb - 1
    const int h = hq / a.q_layers, ql = hq - h * a.q_layers;
    const int unit0 = hq * a.nblk + qby * a.grid_w + qbx0;  // row of block b: unit0 + b
    const int n_keys = a.count * a.nblk;
    grid_dep_launch();  // the attention may start its set-up; it waits for this grid's lists

    if (a.scores) {  // -inf outside the allowed candidates of the group's rows
        for (int b = 0; b < nb; ++b) {
            float *srow = a.scores + static_cast<size_t>(unit0 + b) * n_keys;
            for (int j = tid; j < n_keys; j += kThreads) srow[j] = -INFINITY;
        }
    }
    if constexpr (kRope) {
        if (tid < 64) sm.freq[tid] = rope_freq(tid, a.rope_base);
    }

    // ---- 1. block means of q (input of the caller: not written by the preceding kernel)
    const size_t frame = static_cast<size_t>(h) * a.tq + ql * 2;
#pragma unroll 1
    for (int b = 0; b < nb; ++b) {
        const int qbx = qbx0 + b;
        const int half = lane >> 4, d8 = lane & 15;  // token parity, dims [8 d8, 8 d8 + 8)
        uint4 raw[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // tokens n = 16 w + 2 i + half, (t, y, x) row-major
            const int n = warp * 16 + 2 * i + half;
            const int tt = n >> 6, y = (n >> 3) & 7, x = n & 7;
            const size_t tok = ((frame + tt) * a.tok_h + qby * 8 + y) * a.tok_w + qbx * 8 + x;
            raw[i] = __ldg(reinterpret_cast<const uint4 *>(a.q + tok * kHeadDim) + d8);
        }
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        if constexpr (kRope) {
            // the block's rotation table, built while the loads above are in flight
            __syncthreads();  // (the frequencies; the previous block's table is no longer read)
            for (int e = tid; e < kTabEntries; e += kThreads) {
                int pos, pair;
                if (e < kTabY) {
                    pos = a.rope_frame0 + 2 * ql + e / kRopePairsT;
                    pair = e % kRopePairsT;
                } else if (e < kTabX) {
                    pos = qby * 8 + (e - kTabY) / kRopePairsY;
                    pair = kRopeFirstY + (e - kTabY) % kRopePairsY;
                } else {
                    pos = qbx * 8 + (e - kTabX) / kRopePairsY;
                    pair = kRopeFirstX + (e - kTabX) % kRopePairsY;
                }
                sm.tab[e] = rope_cs(pos, sm.freq[pair]);
            }
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int n = warp * 16 + 2 * i + half;  // token (t, y, x) = (n / 64, n / 8 % 8, n % 8)
                const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
                uint32_t r4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int pair = 4 * d8 + e;
                    const int axis = rope_axis(pair);
                    const int idx = axis == 0 ? (n >> 6) * kRopePairsT + pair
                                  : axis == 1 ? kTabY + ((n >> 3) & 7) * kRopePairsY + pair - kRopeFirstY
                                              : kTabX + (n & 7) * kRopePairsY + pair - kRopeFirstX;
                    const float2 cs = sm.tab[idx];
                    r4[e] = rope_rotate(w4[e], cs.x, cs.y);
                    add_bf16x2(acc[2 * e], acc[2 * e + 1], r4[e]);
                }
                if (a.q_rot) {
                    const size_t tok = ((frame + (n >> 6)) * a.tok_h + qby * 8 + ((n >> 3) & 7)) * a.tok_w + qbx * 8 +
                                       (n & 7);
                    reinterpret_cast<uint4 *>(a.q_rot + tok * kHeadDim)[d8] = make_uint4(r4[0], r4[1], r4[2], r4[3]);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) add_bf16x2(acc[2 * e], acc[2 * e + 1], w4[e]);
            }
        }
        // even tokens (lanes 0-15) + odd tokens (lanes 16-31)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float o = __shfl_xor_sync(kFull, acc[e], 16);
            acc[e] = half == 0 ? acc[e] + o : o + acc[e];
        }
        if (half == 0) {
            float4 *dst = reinterpret_cast<float4 *>(&sm.part[warp][8 * d8]);
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        __syncthreads();
        if (tid < kHeadDim) {
            const float (*p)[kHeadDim] = sm.part;
            const float s = ((p[0][tid] + p[1][tid]) + (p[2][tid] + p[3][tid])) +
                            ((p[4][tid] + p[5][tid]) + (p[6][tid] + p[7][tid]));
            const float m = s * (1.0f / 128.0f);
            sm.mq[b][tid] = m;
            if (a.qmean) a.qmean[static_cast<size_t>(unit0 + b) * kHeadDim + tid] = m;
        }
        __syncthreads();  // the q mean (and the -inf prefill) are visible; the partial sums are free
    }

    // ---- 2. scores over the union of the group's windows (the blocks share their
    //         window rows; their column windows overlap), layer-major: warp w
    //         takes union keys c_begin + 64i + 8w ... + 7; lane l reads dims
    //         [4l, 4l + 4) of each (one coalesced 512-byte row per load, 8 in
    //         flight), fp32 products with every block's q mean, then a fixed
    //         reduce-scatter butterfly
    int uy0, uy1, ux0, ux1, lo, hi;
    window_1d(qby, a.grid_h, a.local_range, a.local_mode, uy0, uy1);
    window_1d(qbx0, a.grid_w, a.local_range, a.local_mode, ux0, hi);
    window_1d(qbx0 + nb - 1, a.grid_w, a.local_range, a.local_mode, lo, ux1);
    const int UX = ux1 - ux0, UYX = (uy1 - uy0) * UX;
    const int n_layers = a.count - a.q_layers + ql + 1;  // key layers up to the group's own
    const int nu = n_layers * UYX;
    const uint64_t m_uyx = div_magic(static_cast<uint32_t>(UYX)), m_ux = div_magic(static_cast<uint32_t>(UX));
    float4 qv[kR];  // dims [4 lane, 4 lane + 4) of every block's q mean (0 past the group)
#pragma unroll
    for (int b = 0; b < kR; ++b)
        qv[b] = b < nb ? reinterpret_cast<const float4 *>(sm.mq[b])[lane] : make_float4(0.f, 0.f, 0.f, 0.f);
    // the (block, key) value this lane ends with, and that block's window
    const int vsel = reduce_index<kR>(lane);
    const int rb = vsel >> 3, uk = vsel & 7;
    const bool writer = reduce_writer<kR>(lane) && rb < nb;
    int wx0, wx1;
    window_1d(qbx0 + (rb < nb ? rb : 0), a.grid_w, a.local_range, a.local_mode, wx0, wx1);
    const int bwx = wx1 - wx0, bwsz = (uy1 - uy0) * bwx;
    uint32_t *bkeys = keys + (rb < nb ? rb : 0) * a.cand_cap;
    float *bsrow = a.scores ? a.scores + static_cast<size_t>(unit0 + (rb < nb ? rb : 0)) * n_keys : nullptr;
    auto score_range = [&](int c_begin, int c_end) {
        constexpr int kU = 8;
        for (int c0 = c_begin + warp * kU; c0 < c_end; c0 += kWarps * kU) {
            // lane u < kU locates union key c0 + u (one division pair per lane),
            // then every lane loads its 16 bytes of each of the kU rows
            uint32_t row = 0;
            int info_layer = 0, info_yx = 0;
            if (lane < kU) {
                const int c = min(c0 + lane, c_end - 1);
                const int layer = div_by(c, m_uyx);
                const int rem = c - layer * UYX;
                const int ry = div_by(rem, m_ux);
                const int ky = uy0 + ry, kx = ux0 + rem - ry * UX;
                int slot = a.oldest + layer;
                if (slot >= a.capacity) slot -= a.capacity;
                row = static_cast<uint32_t>((slot * a.heads + h) * a.nblk + ky * a.grid_w + kx);
                info_layer = layer;
                info_yx = (ky << 16) | kx;
            }
            float4 kv[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const uint32_t r = __shfl_sync(kFull, row, u);
                kv[u] = __ldg(reinterpret_cast<const float4 *>(a.kmean + static_cast<size_t>(r) * kHeadDim) + lane);
            }
            float d[8 * kR];
#pragma unroll
            for (int b = 0; b < kR; ++b) {
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    float s = qv[b].x * kv[u].x;
                    s = fmaf(qv[b].y, kv[u].y, s);
                    s = fmaf(qv[b].z, kv[u].z, s);
                    d[8 * b + u] = fmaf(qv[b].w, kv[u].w, s);
                }
            }
            const float dot = reduce_group<kR>(d, lane);
            const int layer = __shfl_sync(kFull, info_layer, uk);
            const int yx = __shfl_sync(kFull, info_yx, uk);
            const int kx = yx & 0xFFFF;
            if (writer && c0 + uk < c_end && kx >= wx0 && kx < wx1) {
                const int ky = yx >> 16;
                const float score = dot * a.scale;
                bkeys[layer * bwsz + (ky - uy0) * bwx + (kx - wx0)] = desc_key(score);
                if (bsrow) bsrow[layer * a.nblk + ky * a.grid_w + kx] = score;
            }
        }
    };
    // Keys of the layers resident before the chunk's append (logical layers
    // below count - fresh_layers, written by earlier, completed appends) are
    // scored at once; those of the newest layers only after the wait below.
    const int u_split = min(nu, max(a.count - a.fresh_layers, 0) * UYX);
    score_range(0, u_split);
    // Launched as a programmatic dependent of the cache append of the chunk:
    // the key means of its layers are read only from here on (returns at once
    // otherwise).
    grid_dep_wait();
    score_range(u_split, nu);

    // ---- 3. exact top-k of every block of the group: radix select of the k-th
    //         smallest key, then the kept list in ascending key index.  With two
    //         blocks each half of the CTA (a team of 4 warps, its own histogram
    //         and named barrier) selects one of them, the two at the same time.
    __syncthreads();  // every block's candidates are complete
    const int team_warps = kWarps / nb;
    const int team = warp / team_warps;  // = the block this team selects
    const int twarp = warp - team * team_warps;
    const int tthreads = team_warps * 32;
    const int ttid = tid - team * tthreads;
    auto team_sync = [&]() {
        if constexpr (kR == 1) {
            __syncthreads();
        } else if (team == 0) {
            bar_sync_id<1>(tthreads);
        } else {
            bar_sync_id<2>(tthreads);
        }
    };
    const uint32_t lt_mask = lanemask_lt();
    uint32_t *hist = sm.hist[team];
    {
        const int b = team;
        int x0, x1;
        window_1d(qbx0 + b, a.grid_w, a.local_range, a.local_mode, x0, x1);
        const int wx = x1 - x0;
        const int wsz = (uy1 - uy0) * wx;
        const int ncand = n_layers * wsz;  // >= 1 (the block itself)
        const uint32_t *bk = keys + b * a.cand_cap;
        const int k = min(a.topk, ncand);
        uint32_t prefix = 0, mask = 0, k_rem = static_cast<uint32_t>(k);
        bool whole = false;
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int i = ttid; i < 256; i += tthreads) hist[i] = 0u;
            team_sync();
            for (int c0 = twarp * 32; c0 < ncand; c0 += tthreads) {  // whole warps, one add per distinct bin
                const int c = c0 + lane;
                const uint32_t key = c < ncand ? bk[c] : 0u;
                const bool hit = c < ncand && (key & mask) == prefix;
                const uint32_t bin = hit ? ((key >> shift) & 255u) : 256u;
                const uint32_t peers = __match_any_sync(kFull, bin);
                if (hit && (peers & lt_mask) == 0u) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
            }
            team_sync();
            if (twarp == 0) {
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
                if (excl < k_rem && k_rem <= incl) {  // exactly one lane holds the k-th key's digit
                    uint32_t run = excl;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (run + cnt[e] >= k_rem) {
                            sm.digit[team] = static_cast<uint32_t>(lane * 8 + e);
                            sm.below[team] = run;
                            sm.whole[team] = run + cnt[e] == k_rem;  // every key of the bin is kept
                            break;
                        }
                        run += cnt[e];
                    }
                }
            }
            team_sync();
            k_rem -= sm.below[team];
            prefix |= sm.digit[team] << shift;
            mask |= 255u << shift;
            if (sm.whole[team]) {  // the k-th key's bin is kept whole: no further digit is needed
                prefix |= (1u << shift) - 1u;  // T = the largest key of the bin
                whole = true;
                break;
            }
        }
        if (twarp != 0) return;
        const uint32_t T = prefix;
        // keys equal to T that belong to the k smallest (all of them when the bin is kept whole)
        const int k_eq = whole ? INT_MAX : static_cast<int>(k_rem);
        const int unit = unit0 + b;
        int32_t *out = a.kept_idx + static_cast<size_t>(unit) * a.topk;
        const uint64_t m_wsz = div_magic(static_cast<uint32_t>(wsz)), m_wx = div_magic(static_cast<uint32_t>(wx));
        int out_pos = 0, eq_seen = 0;
        for (int base = 0; base < ncand; base += 32) {
            const int c = base + lane;
            const bool valid = c < ncand;
            const uint32_t key = valid ? bk[c] : 0xFFFFFFFFu;
            const bool eq = valid && key == T;
            const uint32_t eqb = __ballot_sync(kFull, eq);
            const int eq_rank = eq_seen + __popc(eqb & lt_mask);
            const bool take = valid && (key < T || (eq && eq_rank < k_eq));
            const uint32_t tb = __ballot_sync(kFull, take);
            if (take) {
                const int layer = div_by(c, m_wsz);
                const int rem = c - layer * wsz;
                const int ry = div_by(rem, m_wx);
                out[out_pos + __popc(tb & lt_mask)] = layer * a.nblk + (uy0 + ry) * a.grid_w + x0 + rem - ry * wx;
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
}

template <bool kRope, int kR>
cudaError_t launch_group(const DraftArgs &a, bool pdl, const DeviceInfo &dev, cudaStream_t stream) {
    static std::atomic<int> smem_set[kMaxDevices];
    const size_t smem = 4 * static_cast<size_t>(kR) * a.cand_cap;
    if (smem > 48 * 1024 - sizeof(DraftSmem<kRope, kR>)) {
        const cudaError_t e = ensure_smem_limit(draft_kernel<kRope, kR>, dev.device, smem, smem_set);
        if (e != cudaSuccess) return e;
    }
    const int grid = a.heads * a.q_layers * a.grid_h * a.groups_x;
    return launch_kernel(draft_kernel<kRope, kR>, dim3(grid), dim3(kThreads), smem, stream, pdl, a);
}

}  // namespace

cudaError_t launch_draft(const DraftArgs &in, bool pdl, const DeviceInfo &dev, cudaStream_t stream) {
    // Groups of two horizontally adjacent query blocks on large grids: each key
    // mean read from L2 serves both (their windows share rows and most
    // columns), and the per-key work (location, load, butterfly) is shared.
    // Measured: 5-9 % faster from 3,024 rows up, but slower at 720 rows, where
    // one block per CTA keeps more CTAs (and warps) in flight.
    constexpr int kGroupMinRows = 2048;
    DraftArgs a = in;
    const int64_t rows = static_cast<int64_t>(a.heads) * a.q_layers * a.nblk;
    const int group = (a.grid_w >= 2 && rows >= kGroupMinRows) ? 2 : 1;
    a.groups_x = (a.grid_w + group - 1) / group;
    const bool rope = a.rope_base != 0.f;
    if (group == 2)
        return rope ? launch_group<true, 2>(a, pdl, dev, stream) : launch_group<false, 2>(a, pdl, dev, stream);
    return rope ? launch_group<true, 1>(a, pdl, dev, stream) : launch_group<false, 1>(a, pdl, dev, stream);
}

}  // namespace lcsa
