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
// One CTA of 8 warps per tile of TY x TX neighbouring query blocks of one
// head and one query layer (the host picks the tile).  Neighbouring blocks
// have overlapping windows, so the key means of the union of their windows
// are staged in shared memory once and scored against every block of the
// tile:
//  1. q block means: TMA loads of whole (2,8,8) blocks of q (a box that lands
//     in block order, so the partition costs nothing) through a ring of two
//     32 KB stages; each block is summed in a fixed order (per thread four
//     chains of 8 tokens, then a tree over chains and token quarters), times
//     1/128.
//  2. scores: the union key means (every visible layer) are copied into
//     shared memory 8 dimensions at a time (cp.async, double-buffered, rows
//     padded so that the per-key loads are conflict-free); thread t owns
//     union keys t, t + 256, ... and accumulates, for every block of the tile,
//     the fp32 dot product sum_d mq_d * mk_d in ascending d with one FMA per
//     term (the q means are read as warp-uniform loads).  Each (block, key)
//     product whose key lies in that block's window becomes the block's
//     candidate key, a 32-bit integer whose unsigned order is the descending
//     score order, at its position in ascending key index.
//  3. exact top-k, one warp per block: radix select of up to 4 passes (8 bits
//     per pass, warp-private histogram, one atomic per distinct bin; it stops
//     after the pass whose bin holding the k-th key is kept whole) finds the
//     k-th key T; the warp writes every key < T plus the first (lowest-index)
//     keys equal to T, in ascending key index, by a ballot compaction.
// Chained after the cache append (LCSA_FLAG_PDL), the q phase runs while the
// append streams; the key means are read only after waiting for it.
// Every wait is bounded; on expiry the CTA drains its copies and reports
// LCSA_ERR_TIMEOUT.

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
constexpr int kQStages = 2;
constexpr uint32_t kQBytes = kBlockTokens * kHeadDim * 2;  // one bf16 q block, 32 KB
constexpr int kChunkDims = 8;                             // key-mean dimensions per staging chunk
constexpr int kChunkStride = 12;                          // floats per staged key (8 + 4 padding)
constexpr int kChunks = kHeadDim / kChunkDims;

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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Geometry of one CTA: its tile of query blocks and the union of their windows.
struct Tile {
    int h, ql, ty0, tx0, ny, nx;  // tile origin and extent (clipped to the grid)
    int uy0, uy1, ux0, ux1;       // union window rows / columns
    int ulayer;                   // union keys per layer
    int layers;                   // visible key layers (0 .. count - q_layers + ql)
    int total;                    // union keys over all visible layers
};

__device__ __forceinline__ Tile tile_of(const DraftArgs &a) {
    Tile t;
    int u = blockIdx.x;
    const int per_layer = a.tiles_y * a.tiles_x;
    const int hq = div_by(u, a.m_tiles);
    const int in = u - hq * per_layer;
    t.h = div_by(hq, a.m_ql);
    t.ql = hq - t.h * a.q_layers;
    const int ty = div_by(in, a.m_tiles_x);
    const int tx = in - ty * a.tiles_x;
    t.ty0 = ty * a.tile_h;
    t.tx0 = tx * a.tile_w;
    t.ny = min(a.tile_h, a.grid_h - t.ty0);
    t.nx = min(a.tile_w, a.grid_w - t.tx0);
    int lo, hi;
    window_1d(t.ty0, a.grid_h, a.local_range, a.local_mode, t.uy0, hi);
    window_1d(t.ty0 + t.ny - 1, a.grid_h, a.local_range, a.local_mode, lo, t.uy1);
    window_1d(t.tx0, a.grid_w, a.local_range, a.local_mode, t.ux0, hi);
    window_1d(t.tx0 + t.nx - 1, a.grid_w, a.local_range, a.local_mode, lo, t.ux1);
    t.ulayer = (t.uy1 - t.uy0) * (t.ux1 - t.ux0);
    t.layers = a.count - a.q_layers + t.ql + 1;
    t.total = t.layers * t.ulayer;
    return t;
}

// Shared memory: [mbarriers | q partial sums | row windows | mq | candidate
// keys | region A]; region A holds, one after the other: the q stages
// (phase 1), the staged key means (phase 2), the per-warp histograms (phase 3).
struct DraftLayout {
    uint32_t bar, part, win, mq, keys, tab, region, total;
};

__host__ __device__ constexpr uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int RMAX, int KPT>
__host__ __device__ DraftLayout draft_layout(int cand_cap, int rope_entries) {
    DraftLayout L;
    L.bar = 0;
    L.part = 64;                                                    // 4 quarters x 64 float2
    L.win = L.part + 4 * 64 * 8;                                    // RMAX x int4 (y0, y1, x0, x1)
    L.mq = L.win + RMAX * 16;                                       // RMAX x 128 fp32
    L.keys = L.mq + RMAX * kHeadDim * 4;                            // RMAX x cand_cap u32
    L.tab = L.keys + RMAX * static_cast<uint32_t>(cand_cap) * 4;    // rope_entries x float2 (cos, sin)
    L.region = align_up(L.tab + static_cast<uint32_t>(rope_entries) * 8, 1024);
    const uint32_t q_bytes = kQStages * kQBytes;
    const uint32_t k_bytes = 2u * kThreads * KPT * kChunkStride * 4;
    const uint32_t h_bytes = kWarps * 256 * 4;
    uint32_t r = q_bytes > k_bytes ? q_bytes : k_bytes;
    r = r > h_bytes ? r : h_bytes;
    L.total = L.region + r;
    return L;
}

template <int RMAX, int KPT>
__global__ void __launch_bounds__(kThreads, 2)
    draft_kernel(const __grid_constant__ CUtensorMap tm_q, const DraftArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const DraftLayout Lo = draft_layout<RMAX, KPT>(a.cand_cap, a.rope_entries);
    uint64_t *bar_q = reinterpret_cast<uint64_t *>(sm + Lo.bar);
    float2 *part = reinterpret_cast<float2 *>(sm + Lo.part);
    int4 *win = reinterpret_cast<int4 *>(sm + Lo.win);
    float *mq = reinterpret_cast<float *>(sm + Lo.mq);
    uint32_t *keys = reinterpret_cast<uint32_t *>(sm + Lo.keys);
    float2 *tab = reinterpret_cast<float2 *>(sm + Lo.tab);
    uint8_t *region = sm + Lo.region;
    int *abort_word = reinterpret_cast<int *>(sm + Lo.bar + 32);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const Tile T = tile_of(a);
    const int R = T.ny * T.nx;  // query blocks of the tile, row-major in the tile
    grid_dep_launch();          // the attention may start its set-up; it waits for this grid's lists

    if (tid == 0) {
        for (int s = 0; s < kQStages; ++s) mbar_init(smem_u32(&bar_q[s]), 1);
        *abort_word = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_q);
    }
    if ((R & 1) && tid < kHeadDim) mq[(R >> 1) * 2 * kHeadDim + 2 * tid + 1] = 0.f;  // unused row of the last pair
    const bool rope = a.rope_base != 0.f;
    // Rotation table of the tile's tokens: (cos, sin) of the 2 frames x 22 time
    // pairs, then of its 8 tile_h token rows x 21 row pairs, then of its 8 tile_w
    // token columns x 21 column pairs.
    const int tab_y = 2 * kRopePairsT, tab_x = tab_y + 8 * a.tile_h * kRopePairsY;
    if (rope) {
        for (int e = tid; e < a.rope_entries; e += kThreads) {
            int pos, pair;
            if (e < tab_y) {
                pos = a.rope_frame0 + 2 * T.ql + e / kRopePairsT;
                pair = e % kRopePairsT;
            } else if (e < tab_x) {
                pos = T.ty0 * 8 + (e - tab_y) / kRopePairsY;
                pair = kRopeFirstY + (e - tab_y) % kRopePairsY;
            } else {
                pos = T.tx0 * 8 + (e - tab_x) / kRopePairsY;
                pair = kRopeFirstX + (e - tab_x) % kRopePairsY;
            }
            tab[e] = rope_cs(pos, rope_freq(pair, a.rope_base));
        }
    }
    if (tid < R) {  // window of every block of the tile
        const int ry = tid / T.nx, rx = tid - ry * T.nx;
        int4 wv;
        window_1d(T.ty0 + ry, a.grid_h, a.local_range, a.local_mode, wv.x, wv.y);
        window_1d(T.tx0 + rx, a.grid_w, a.local_range, a.local_mode, wv.z, wv.w);
        win[tid] = wv;
    }
    __syncthreads();

    // ---- 1. q block means (q is the caller's input: not written by the preceding kernel)
    const int frames = 2 * a.q_layers;
    auto issue_q = [&](int r) {  // block r of the tile into stage r % kQStages
        const int ry = r / T.nx, rx = r - ry * T.nx;
        const uint32_t bar = smem_u32(&bar_q[r % kQStages]);
        mbar_arrive_expect_tx(bar, kQBytes);
        tma_load_4d(smem_u32(region + (r % kQStages) * kQBytes), &tm_q, bar, 0, (T.tx0 + rx) * 8,
                    (T.ty0 + ry) * 8, T.h * frames + T.ql * 2);
    };
    int issued = 0;
    if (tid == 0) {
        for (; issued < kQStages && issued < R; ++issued) issue_q(issued);
    }
    const int nq = a.q_layers * a.nblk;
    const int n_keys = a.count * a.nblk;
    bool ok = true;
    {
        const int pr = tid & 63;    // dimensions 2 pr, 2 pr + 1
        const int qt = tid >> 6;    // tokens [32 qt, 32 qt + 32)
        volatile int *abort_v = abort_word;
        for (int r = 0; r < R; ++r) {
            const int s = r % kQStages;
            // one thread waits for the copy; the others wait at the block barrier
            // (a spinning wait in every thread would take the issue slots of the
            // CTA sharing the SM)
            bool got = true;
            if (tid == 0) got = mbar_wait(smem_u32(&bar_q[s]), (r / kQStages) & 1, abort_v, a.timeout_ns);
            if (!__syncthreads_and(got)) {
                ok = false;
                break;
            }
            const uint32_t *w = reinterpret_cast<const uint32_t *>(region + s * kQBytes) + qt * 32 * 64 + pr;
            float lo[4] = {0.f, 0.f, 0.f, 0.f}, hi[4] = {0.f, 0.f, 0.f, 0.f};
            if (!rope) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) add_bf16x2(lo[c], hi[c], w[(4 * i + c) * 64]);  // token 32 qt + 4 i + c
                }
            } else {
                // token 32 qt + 4 i + c sits at frame qt / 2, block row 4 (qt & 1) + i / 2,
                // block column 4 (i & 1) + c; its pair pr is rotated, rounded to bf16, then summed
                const int ry = r / T.nx, rx = r - ry * T.nx;
                const int axis = rope_axis(pr);
                const int base = axis == 0 ? (qt >> 1) * kRopePairsT + pr
                               : axis == 1 ? tab_y + (ry * 8 + 4 * (qt & 1)) * kRopePairsY + pr - kRopeFirstY
                                           : tab_x + rx * 8 * kRopePairsY + pr - kRopeFirstX;
                const int sy = axis == 1 ? kRopePairsY : 0, sx = axis == 2 ? kRopePairsY : 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float2 cs = tab[base + (i >> 1) * sy + (4 * (i & 1) + c) * sx];
                        add_bf16x2(lo[c], hi[c], rope_rotate(w[(4 * i + c) * 64], cs.x, cs.y));
                    }
                }
            }
            part[qt * 64 + pr] = make_float2((lo[0] + lo[1]) + (lo[2] + lo[3]), (hi[0] + hi[1]) + (hi[2] + hi[3]));
            __syncthreads();  // the stage is read; the quarter sums are visible
            if (tid == 0 && issued < R) issue_q(issued++);
            if (tid < 64) {
                const float2 p0 = part[tid], p1 = part[64 + tid], p2 = part[128 + tid], p3 = part[192 + tid];
                const float m0 = ((p0.x + p1.x) + (p2.x + p3.x)) * (1.0f / 128.0f);
                const float m1 = ((p0.y + p1.y) + (p2.y + p3.y)) * (1.0f / 128.0f);
                // row pairs interleaved: element (r, d) at (r / 2) * 256 + 2 d + (r & 1)
                float *pair = mq + (r >> 1) * 2 * kHeadDim + (r & 1);
                pair[4 * tid] = m0;
                pair[4 * tid + 2] = m1;
                if (a.qmean) {
                    const int ry = r / T.nx, rx = r - ry * T.nx;
                    const size_t row = static_cast<size_t>(T.h) * nq + T.ql * a.nblk + (T.ty0 + ry) * a.grid_w +
                                       T.tx0 + rx;
                    reinterpret_cast<float2 *>(a.qmean + row * kHeadDim)[tid] = make_float2(m0, m1);
                }
            }
            __syncthreads();  // the quarter sums may be overwritten
        }
    }
    if (!ok) {
        // a wait gave up: the loads still in flight land before the CTA exits
        if (tid == 0) {
            for (int i = issued > kQStages ? issued - kQStages : 0; i < issued; ++i)
                mbar_wait_drain(smem_u32(&bar_q[i % kQStages]), (i / kQStages) & 1, a.timeout_ns);
            if (a.status) atomicOr(a.status, LCSA_ERR_TIMEOUT);
        }
        return;
    }
    if (a.scores) {  // -inf everywhere but the allowed pairs, written below
        for (int r = 0; r < R; ++r) {
            const int ry = r / T.nx, rx = r - ry * T.nx;
            const size_t row = static_cast<size_t>(T.h) * nq + T.ql * a.nblk + (T.ty0 + ry) * a.grid_w + T.tx0 + rx;
            for (int j = tid; j < n_keys; j += kThreads) a.scores[row * n_keys + j] = -INFINITY;
        }
    }
    // Launched as a programmatic dependent of the cache append of the chunk: the
    // key means are read only from here on (returns at once otherwise).
    grid_dep_wait();

    // ---- 2. scores over the union keys, KPT * 256 keys per round
    const int uw = T.ux1 - T.ux0;
    const uint64_t m_ul = div_magic(static_cast<uint32_t>(T.ulayer)), m_uw = div_magic(static_cast<uint32_t>(uw));
    const int per_round = kThreads * KPT;
    float *stage = reinterpret_cast<float *>(region);
    const uint32_t stage_u32 = smem_u32(region);
    const uint32_t buf_floats = static_cast<uint32_t>(per_round) * kChunkStride;
    for (int k0 = 0; k0 < T.total; k0 += per_round) {
        const int nk = min(per_round, T.total - k0);
        // Copy of chunk c (8 dims = two 16-byte pieces per key) into buffer c & 1.
        // Thread t copies pieces t + 256 m, i.e. half (t & 1) of keys t / 2 + 128 m:
        // their key-mean rows are located once per round.
        uint32_t krow[2 * KPT];
#pragma unroll
        for (int m = 0; m < 2 * KPT; ++m) {
            const int sk = (tid >> 1) + 128 * m;
            krow[m] = 0u;
            if (sk < nk) {
                const int u = k0 + sk;
                const int layer = div_by(u, m_ul);
                const int rem = u - layer * T.ulayer;
                const int yy = div_by(rem, m_uw);
                const int b = (T.uy0 + yy) * a.grid_w + T.ux0 + rem - yy * uw;
                int slot = a.oldest + layer;
                if (slot >= a.capacity) slot -= a.capacity;
                krow[m] = static_cast<uint32_t>((slot * a.heads + T.h) * a.nblk + b);
            }
        }
        const int half = tid & 1;
        auto stage_chunk = [&](int c) {
            const uint32_t dst0 = stage_u32 + (c & 1) * buf_floats * 4;
#pragma unroll
            for (int m = 0; m < 2 * KPT; ++m) {
                const int sk = (tid >> 1) + 128 * m;
                if (sk < nk) {
                    const float *src = a.kmean + static_cast<size_t>(krow[m]) * kHeadDim + c * kChunkDims + 4 * half;
                    cp_async16(dst0 + (sk * kChunkStride + 4 * half) * 4, src);
                }
            }
            cp_async_commit();
        };
        // acc[rp][j]: the dot products of rows 2 rp and 2 rp + 1 with key j, as one
        // packed pair (fma.rn.f32x2 rounds each lane exactly like fmaf)
        uint64_t acc[RMAX / 2][KPT];
#pragma unroll
        for (int rp = 0; rp < RMAX / 2; ++rp) {
#pragma unroll
            for (int j = 0; j < KPT; ++j) acc[rp][j] = 0ull;
        }
        stage_chunk(0);
        stage_chunk(1);
#pragma unroll 1
        for (int c = 0; c < kChunks; ++c) {
            if (c + 1 < kChunks) cp_async_wait<1>();
            else cp_async_wait<0>();
            __syncthreads();  // chunk c landed for every thread
            const float *buf = stage + (c & 1) * buf_floats;
            uint64_t kd[KPT][kChunkDims];  // (k_d, k_d) pairs
#pragma unroll
            for (int j = 0; j < KPT; ++j) {
                const int sk = min(tid + j * kThreads, nk - 1);  // (duplicates beyond nk are not written)
                const float4 v0 = *reinterpret_cast<const float4 *>(buf + sk * kChunkStride);
                const float4 v1 = *reinterpret_cast<const float4 *>(buf + sk * kChunkStride + 4);
                kd[j][0] = f32x2_pack(v0.x, v0.x);
                kd[j][1] = f32x2_pack(v0.y, v0.y);
                kd[j][2] = f32x2_pack(v0.z, v0.z);
                kd[j][3] = f32x2_pack(v0.w, v0.w);
                kd[j][4] = f32x2_pack(v1.x, v1.x);
                kd[j][5] = f32x2_pack(v1.y, v1.y);
                kd[j][6] = f32x2_pack(v1.z, v1.z);
                kd[j][7] = f32x2_pack(v1.w, v1.w);
            }
#pragma unroll
            for (int rp = 0; rp < RMAX / 2; ++rp) {
                if (2 * rp < R) {  // (uniform over the CTA)
                    // (q_2rp[d], q_2rp+1[d]) for the chunk's 8 dims: four 16-byte loads
                    const ulonglong2 *qp =
                        reinterpret_cast<const ulonglong2 *>(mq + rp * 2 * kHeadDim + 2 * c * kChunkDims);
                    const ulonglong2 q01 = qp[0], q23 = qp[1], q45 = qp[2], q67 = qp[3];
#pragma unroll
                    for (int j = 0; j < KPT; ++j) {
                        uint64_t d = acc[rp][j];
                        d = f32x2_fma(q01.x, kd[j][0], d);
                        d = f32x2_fma(q01.y, kd[j][1], d);
                        d = f32x2_fma(q23.x, kd[j][2], d);
                        d = f32x2_fma(q23.y, kd[j][3], d);
                        d = f32x2_fma(q45.x, kd[j][4], d);
                        d = f32x2_fma(q45.y, kd[j][5], d);
                        d = f32x2_fma(q67.x, kd[j][6], d);
                        d = f32x2_fma(q67.y, kd[j][7], d);
                        acc[rp][j] = d;
                    }
                }
            }
            __syncthreads();  // buffer c & 1 is read: chunk c + 2 may overwrite it
            if (c + 2 < kChunks) stage_chunk(c + 2);
        }
        // candidate keys of every block whose window holds the key
#pragma unroll
        for (int j = 0; j < KPT; ++j) {
            const int s = tid + j * kThreads;
            if (s < nk) {
                const int u = k0 + s;
                const int layer = div_by(u, m_ul);
                const int rem = u - layer * T.ulayer;
                const int yy = div_by(rem, m_uw);
                const int ky = T.uy0 + yy, kx = T.ux0 + rem - yy * uw;
                const int jl = layer * a.nblk + ky * a.grid_w + kx;
#pragma unroll
                for (int r = 0; r < RMAX; ++r) {
                    if (r < R) {
                        const int4 wv = win[r];  // (y0, y1, x0, x1)
                        if (ky >= wv.x && ky < wv.y && kx >= wv.z && kx < wv.w) {
                            const int ry = r / T.nx, rx = r - ry * T.nx;
                            const int wx = wv.w - wv.z;
                            const int c = (layer * (wv.y - wv.x) + (ky - wv.x)) * wx + (kx - wv.z);
                            float lo, hi;
                            f32x2_unpack(acc[r >> 1][j], lo, hi);
                            const float score = ((r & 1) ? hi : lo) * a.scale;
                            keys[r * a.cand_cap + c] = desc_key(score);
                            if (a.scores) {
                                const size_t row = static_cast<size_t>(T.h) * nq + T.ql * a.nblk +
                                                   (T.ty0 + ry) * a.grid_w + T.tx0 + rx;
                                a.scores[row * n_keys + jl] = score;
                            }
                        }
                    }
                }
            }
        }
    }
    __syncthreads();  // every candidate key is in shared memory; region A is free

    // ---- 3. exact top-k per block, one warp per block
    uint32_t *hist = reinterpret_cast<uint32_t *>(region) + warp * 256;
    const uint32_t lt_mask = lanemask_lt();
    for (int r = warp; r < R; r += kWarps) {
        const int ry = r / T.nx, rx = r - ry * T.nx;
        const int4 wv = win[r];
        const int y0 = wv.x, x0 = wv.z;
        const int wx = wv.w - wv.z, wsz = (wv.y - wv.x) * wx;
        const int ncand = T.layers * wsz;
        const int k = min(a.topk, ncand);
        const uint32_t *rk = keys + r * a.cand_cap;
        uint32_t prefix = 0, mask = 0, k_rem = static_cast<uint32_t>(k);
        bool whole = false;
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
#pragma unroll
            for (int e = 0; e < 8; ++e) hist[lane * 8 + e] = 0u;
            __syncwarp();
            for (int c0 = 0; c0 < ncand; c0 += 32) {  // one add per distinct bin
                const int c = c0 + lane;
                const uint32_t key = c < ncand ? rk[c] : 0u;
                const bool hit = c < ncand && (key & mask) == prefix;
                const uint32_t bin = hit ? ((key >> shift) & 255u) : 256u;
                const uint32_t peers = __match_any_sync(kFull, bin);
                if (hit && (peers & lt_mask) == 0u) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
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
            uint32_t digit = 0, below = 0, is_whole = 0;
            const bool holder = excl < k_rem && k_rem <= incl;  // exactly one lane holds the k-th key's digit
            if (holder) {
                uint32_t run = excl;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (run + cnt[e] >= k_rem) {
                        digit = static_cast<uint32_t>(lane * 8 + e);
                        below = run;
                        is_whole = run + cnt[e] == k_rem;  // every key of the bin is kept
                        break;
                    }
                    run += cnt[e];
                }
            }
            const int src = __ffs(__ballot_sync(kFull, holder)) - 1;
            digit = __shfl_sync(kFull, digit, src);
            below = __shfl_sync(kFull, below, src);
            is_whole = __shfl_sync(kFull, is_whole, src);
            __syncwarp();  // the histogram is read before the next pass clears it
            k_rem -= below;
            prefix |= digit << shift;
            mask |= 255u << shift;
            if (is_whole) {  // the k-th key's bin is kept whole: no further digit is needed
                prefix |= (1u << shift) - 1u;  // T = the largest key of the bin
                whole = true;
                break;
            }
        }
        const uint32_t Tk = prefix;
        // keys equal to T that belong to the k smallest (all of them when the bin is kept whole)
        const int k_eq = whole ? INT_MAX : static_cast<int>(k_rem);
        const size_t row = static_cast<size_t>(T.h) * nq + T.ql * a.nblk + (T.ty0 + ry) * a.grid_w + T.tx0 + rx;
        int32_t *out = a.kept_idx + row * a.topk;
        const uint64_t m_wsz = div_magic(static_cast<uint32_t>(wsz)), m_wx = div_magic(static_cast<uint32_t>(wx));
        int out_pos = 0, eq_seen = 0;
        for (int base = 0; base < ncand; base += 32) {
            const int c = base + lane;
            const bool valid = c < ncand;
            const uint32_t key = valid ? rk[c] : 0xFFFFFFFFu;
            const bool eq = valid && key == Tk;
            const uint32_t eqb = __ballot_sync(kFull, eq);
            const int eq_rank = eq_seen + __popc(eqb & lt_mask);
            const bool take = valid && (key < Tk || (eq && eq_rank < k_eq));
            const uint32_t tb = __ballot_sync(kFull, take);
            if (take) {
                const int layer = div_by(c, m_wsz);
                const int rem = c - layer * wsz;
                const int yy = div_by(rem, m_wx);
                out[out_pos + __popc(tb & lt_mask)] = layer * a.nblk + (y0 + yy) * a.grid_w + x0 + rem - yy * wx;
            }
            out_pos += __popc(tb);
            eq_seen += __popc(eqb);
        }
        for (int i = out_pos + lane; i < a.topk; i += 32) out[i] = -1;
        if (lane == 0) {
            a.kept_cnt[row] = out_pos;
            if (out_pos != k && a.status) atomicOr(a.status, LCSA_ERR_BAD_INDEX);  // cannot happen
        }
        __syncwarp();  // the histogram of this warp is free for its next block
    }
}

template <int RMAX, int KPT>
cudaError_t launch_draft_t(const CUtensorMap &tm_q, const DraftArgs &a, bool pdl, const DeviceInfo &dev,
                           cudaStream_t stream) {
    static std::atomic<int> smem_set[kMaxDevices];
    const size_t smem = draft_layout<RMAX, KPT>(a.cand_cap, a.rope_entries).total + 1024;  // + alignment slack
    const cudaError_t e = ensure_smem_limit(draft_kernel<RMAX, KPT>, dev.device, smem, smem_set);
    if (e != cudaSuccess) return e;
    const int grid = a.heads * a.q_layers * a.tiles_y * a.tiles_x;
    return launch_kernel(draft_kernel<RMAX, KPT>, dim3(grid), dim3(kThreads), smem, stream, pdl, tm_q, a);
}

}  // namespace

size_t draft_smem_bytes(int rmax, int kpt, int cand_cap, int rope_entries) {
#define LCSA_DRAFT_CASE(R, K) \
    if (rmax == R && kpt == K) return draft_layout<R, K>(cand_cap, rope_entries).total + 1024;
    LCSA_DRAFT_CASE(4, 1) LCSA_DRAFT_CASE(4, 2) LCSA_DRAFT_CASE(4, 3)
    LCSA_DRAFT_CASE(8, 1) LCSA_DRAFT_CASE(8, 2) LCSA_DRAFT_CASE(8, 3)
    LCSA_DRAFT_CASE(12, 1) LCSA_DRAFT_CASE(12, 2) LCSA_DRAFT_CASE(12, 3)
    LCSA_DRAFT_CASE(16, 1) LCSA_DRAFT_CASE(16, 2) LCSA_DRAFT_CASE(16, 3)
#undef LCSA_DRAFT_CASE
    return 0;
}

cudaError_t launch_draft(const CUtensorMap &tm_q, const DraftArgs &a, bool pdl, const DeviceInfo &dev,
                         cudaStream_t stream) {
#define LCSA_DRAFT_CASE(R, K) \
    if (a.rmax == R && a.kpt == K) return launch_draft_t<R, K>(tm_q, a, pdl, dev, stream);
    LCSA_DRAFT_CASE(4, 1) LCSA_DRAFT_CASE(4, 2) LCSA_DRAFT_CASE(4, 3)
    LCSA_DRAFT_CASE(8, 1) LCSA_DRAFT_CASE(8, 2) LCSA_DRAFT_CASE(8, 3)
    LCSA_DRAFT_CASE(12, 1) LCSA_DRAFT_CASE(12, 2) LCSA_DRAFT_CASE(12, 3)
    LCSA_DRAFT_CASE(16, 1) LCSA_DRAFT_CASE(16, 2) LCSA_DRAFT_CASE(16, 3)
#undef LCSA_DRAFT_CASE
    return cudaErrorInvalidValue;
}

}  // namespace lcsa
