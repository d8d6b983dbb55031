// Streaming KV-cache append on sm_100a.
//
// Operation (FlashVSR code walk-through "FlashVSR 是怎么工作的", learn.html,
// section 2.3): the cache carries the partitioned k/v of the newest kv_len
// block-layers and drops the oldest one when a new layer arrives.  Here each
// new layer is written once, in block layout, into its ring slot (the slot of
// the oldest layer when the ring is full), so that dropping the oldest layer
// costs nothing and every kept K/V tile of the attention kernel is one
// contiguous 32 KB block.  The fp32 block means of k used by the draft mask
// (section 2.2, avgpool_k) are produced in the same pass.
//
// A copy engine kernel: one 128-thread CTA per SM walks the (new layer, head,
// block) units grid-stride.  For each unit one thread issues two TMA loads
// (a (128 dims, 8, 8, 2 frames) box of k and of v lands in shared memory
// already in block order: intra index (t, y, x) row-major) and, once the
// threads have read the k tile for its mean, two 32 KB bulk stores into the
// ring slot.  Two stages: the loads of the next unit are in flight while the
// current one is reduced and stored.  The k mean of a dimension is the sum of
// the 128 tokens in a fixed order (two halves of 64 tokens, then half 0 +
// half 1), times 1/128: deterministic.  Few registers and one CTA per SM, so
// that the grid fits the SMs a finishing kernel leaves free next to the CTAs
// of the kernel chained after it.

#include "internal.h"
#include "ptx.cuh"
#include "rope.cuh"
#include "../../include/lcsa.h"

namespace lcsa {
namespace {

constexpr int kThreads = 128;
constexpr int kStages = 2;
constexpr uint32_t kTileBytes = kBlockTokens * kHeadDim * 2;  // 32 KB

struct __align__(1024) AppendSmem {
    uint16_t k[kStages][kBlockTokens * kHeadDim];
    uint16_t v[kStages][kBlockTokens * kHeadDim];
    float2 part[kStages][kHeadDim / 2];  // sums over tokens 64..127, per dimension pair
    uint64_t full[kStages];
    int abort_word;
};

__device__ __forceinline__ int mul_div(int n, uint64_t m) {
    return static_cast<int>((static_cast<uint64_t>(static_cast<uint32_t>(n)) * m) >> 32);
}

struct Unit {
    int li, h, b;
};

// unit = (layer within the chunk, head, block), block fastest
__device__ __forceinline__ Unit unit_of(const AppendArgs &a, int u) {
    Unit r;
    const int hb = mul_div(u, a.m_nblk);
    r.b = u - hb * a.nblk;
    r.li = mul_div(hb, a.m_heads);
    r.h = hb - r.li * a.heads;
    return r;
}

__global__ void __launch_bounds__(kThreads, 1)
    cache_append_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const AppendArgs a) {
    // a draft mask launched as a programmatic dependent may start now; it waits
    // for this grid before it reads what this grid writes
    grid_dep_launch();
    // (a preceding kernel this grid depends on programmatically is waited for
    // at the end: the k/v inputs are the caller's and the slots are spare)
    extern __shared__ uint8_t smem_raw[];
    AppendSmem &sm = *reinterpret_cast<AppendSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                      ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x;
    const int n_units = a.n_layers * a.heads * a.nblk;
    const int n_mine = blockIdx.x < n_units ? (n_units - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;
    const int tc = 2 * a.n_layers;  // frames of the chunk
    volatile int *abort_word = &sm.abort_word;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&sm.full[s]), 1);
        sm.abort_word = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    __syncthreads();

    auto issue_load = [&](int i) {  // the i-th unit of this CTA into stage i % kStages
        const Unit un = unit_of(a, static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x));
        const int by = mul_div(un.b, a.m_gw), bx = un.b - by * a.grid_w;
        const int s = i % kStages;
        const uint32_t bar = smem_u32(&sm.full[s]);
        mbar_arrive_expect_tx(bar, 2 * kTileBytes);
        tma_load_4d(smem_u32(sm.k[s]), &tm_k, bar, 0, bx * 8, by * 8, un.h * tc + 2 * un.li);
        tma_load_4d(smem_u32(sm.v[s]), &tm_v, bar, 0, bx * 8, by * 8, un.h * tc + 2 * un.li);
    };
    int issued = 0;  // loads issued (thread 0)
    if (tid == 0) {
        for (; issued < kStages && issued < n_mine; ++issued) issue_load(issued);
    }

    const int pr = tid & 63;   // dimensions 2 pr, 2 pr + 1
    const int half = tid >> 6;  // tokens [64 half, 64 half + 64)
    const bool rope = a.rope_base != 0.f;
    const int rope_axis_pr = rope_axis(pr);
    const double rope_w = rope ? rope_freq(pr, a.rope_base) : 0.0;
    // (cos, sin) of pos * w and of w, for the angle-addition steps along a row or column
    double step_c = 1.0, step_s = 0.0;
    if (rope && rope_axis_pr != 0) rope_sincos(rope_w, step_s, step_c);
    bool ok = true;
    for (int i = 0; i < n_mine; ++i) {
        const int s = i % kStages;
        ok = mbar_wait(smem_u32(&sm.full[s]), (i / kStages) & 1, abort_word, a.timeout_ns);
        if (i == 0 && tid == 0 && (a.flags & LCSA_FLAG_FORCE_TIMEOUT)) ok = false;  // test hook
        if (!__syncthreads_and(ok)) {
            ok = false;
            break;
        }
        const Unit un = unit_of(a, static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x));
        int slot = a.first_slot + un.li;  // < 2 * capacity
        if (slot >= a.capacity) slot -= a.capacity;
        const size_t blk = (static_cast<size_t>(slot) * a.heads + un.h) * a.nblk + un.b;
        if (rope) {
            // Pair pr of this thread's 64 tokens (frame `half` of the block), rotated
            // in place.  cs[i]: the angle of the i-th row (row band) or column (column
            // band) of the block, or of the frame (time band: every entry), from one
            // fp64 sincos and exact angle-addition steps in fp64.
            const int by = mul_div(un.b, a.m_gw), bx = un.b - by * a.grid_w;
            const int pos0 = rope_axis_pr == 0 ? a.rope_frame0 + 2 * un.li + half
                                               : (rope_axis_pr == 1 ? by * 8 : bx * 8);
            double c, sn;
            rope_sincos(static_cast<double>(pos0) * rope_w, sn, c);
            float2 cs[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cs[i] = make_float2(__double2float_rn(c), __double2float_rn(sn));
                const double c2 = c * step_c - sn * step_s;
                sn = sn * step_c + c * step_s;
                c = c2;
            }
            uint32_t *kw_rw = reinterpret_cast<uint32_t *>(sm.k[s]) + half * 64 * (kHeadDim / 2) + pr;
#pragma unroll
            for (int yy = 0; yy < 8; ++yy) {
#pragma unroll
                for (int xx = 0; xx < 8; ++xx) {
                    const float2 v = rope_axis_pr == 2 ? cs[xx] : cs[yy];  // (time band: all equal)
                    uint32_t *p = kw_rw + (8 * yy + xx) * (kHeadDim / 2);
                    *p = rope_rotate(*p, v.x, v.y);
                }
            }
            fence_proxy_async_smem();  // the rotated tile is read by the bulk store (async proxy)
            __syncthreads();           // every pair of the tile is rotated before the means read it
        }
        // k mean: this thread sums its 64 tokens of two dimensions
        const uint32_t *kw = reinterpret_cast<const uint32_t *>(sm.k[s]) + half * 64 * (kHeadDim / 2) + pr;
        float lo = 0.f, hi = 0.f;
#pragma unroll 16
        for (int n = 0; n < 64; ++n) add_bf16x2(lo, hi, kw[n * (kHeadDim / 2)]);
        if (half == 1) sm.part[s][pr] = make_float2(lo, hi);
        __syncthreads();  // every thread has read the k tile; the upper-half sums are visible
        if (tid == 0) {
            // the tiles go to the ring slot unchanged: two bulk stores
            fence_proxy_async_smem();
            bulk_store(a.k_cache + blk * kBlockTokens * kHeadDim, smem_u32(sm.k[s]), kTileBytes);
            bulk_store(a.v_cache + blk * kBlockTokens * kHeadDim, smem_u32(sm.v[s]), kTileBytes);
            bulk_commit_group();
            if (issued < n_mine) {
                // stage s is refilled once the stores above have read it
                bulk_wait_group_read0();
                issue_load(issued++);
            }
        }
        if (half == 0) {
            const float2 up = sm.part[s][pr];
            reinterpret_cast<float2 *>(a.kmean + blk * kHeadDim)[pr] =
                make_float2((lo + up.x) * (1.0f / 128.0f), (hi + up.y) * (1.0f / 128.0f));
        }
    }
    if (tid == 0) {
        if (!ok) {
            // a wait gave up: the loads still in flight (among the last kStages
            // issued; a consumed one passes at once) land before the CTA exits
            for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
                mbar_wait_drain(smem_u32(&sm.full[i % kStages]), (i / kStages) & 1, a.timeout_ns);
            if (a.status) atomicOr(a.status, LCSA_ERR_TIMEOUT);
        }
        bulk_wait_group0();  // the stores have completed before the shared memory is released
    }
    // Launched as a programmatic dependent of the previous step's attention (it
    // writes spare slots that kernel does not read), this grid completes only
    // after that kernel: whoever waits for this grid waits for both.  One CTA
    // waiting is enough for that (a grid completes when its last CTA exits); the
    // others exit at once and leave their SMs to the kernels chained after
    // this one.
    if (blockIdx.x == 0) grid_dep_wait();
}

}  // namespace

cudaError_t launch_cache_append(const CUtensorMap &tm_k, const CUtensorMap &tm_v, const AppendArgs &a, bool pdl,
                                const DeviceInfo &dev, cudaStream_t stream) {
    static std::atomic<int> smem_set[kMaxDevices];
    const int units = a.n_layers * a.heads * a.nblk;
    const size_t smem = sizeof(AppendSmem) + 1024;  // + alignment slack
    const cudaError_t e = ensure_smem_limit(cache_append_kernel, dev.device, smem, smem_set);
    if (e != cudaSuccess) return e;
    const int grid = units < dev.sms ? units : dev.sms;
    return launch_kernel(cache_append_kernel, dim3(grid), dim3(kThreads), smem, stream, pdl, tm_k, tm_v, a);
}

}  // namespace lcsa
