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
// 256-thread CTAs walk the (new layer, head, block) units grid-stride (a
// grid of at most two CTAs per SM, so that it also fits the SMs a finishing
// kernel leaves free): 16 threads per 256-byte token row, 16-byte loads and
// stores, 128 tokens of k and of v per unit; the k means are reduced in shared
// memory in a fixed order (deterministic).

#include "internal.h"
#include "ptx.cuh"

namespace lcsa {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) cache_append_kernel(const AppendArgs a) {
    // a draft mask launched as a programmatic dependent may start its q-mean
    // phase now; it waits for this grid before reading the ring
    grid_dep_launch();
    // (a preceding kernel this grid depends on programmatically is waited for
    // at the end: the k/v inputs are the caller's and the slot is a spare)
    __shared__ float red[16][kHeadDim + 4];
    const int tid = threadIdx.x;
    const int chunk = tid & 15;  // dims [8*chunk, 8*chunk+8)
    const int sub = tid >> 4;    // token sub-group 0..15
    const int tc = 2 * a.n_layers;  // frames of the chunk
    const int n_units = a.n_layers * a.heads * a.nblk;
    // grid-stride over (layer, head, block) units: a grid of a few CTAs per SM
    // fits into whatever SMs are free when it is launched
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        int unit = u;
        const int b = unit % a.nblk;
        unit /= a.nblk;
        const int h = unit % a.heads;
        const int li = unit / a.heads;  // layer within the appended chunk
        const int by = b / a.grid_w, bx = b - by * a.grid_w;
        const int slot = a.slots[li];

        const size_t dst_block = ((static_cast<size_t>(slot) * a.heads + h) * a.nblk + b) * kBlockTokens;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int n = sub + 16 * it;  // token of the block, (t, y, x) row-major
            const int t = n >> 6, y = (n >> 3) & 7, x = n & 7;
            const size_t src = ((static_cast<size_t>(h) * tc + li * 2 + t) * a.tok_h + by * 8 + y) * a.tok_w + bx * 8 + x;
            const size_t so = src * kHeadDim + chunk * 8;
            const size_t dof = (dst_block + n) * kHeadDim + chunk * 8;
            const uint4 kr = __ldg(reinterpret_cast<const uint4 *>(a.k_tok + so));
            const uint4 vr = __ldg(reinterpret_cast<const uint4 *>(a.v_tok + so));
            *reinterpret_cast<uint4 *>(a.k_cache + dof) = kr;
            *reinterpret_cast<uint4 *>(a.v_cache + dof) = vr;
            const uint32_t w[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] += __uint_as_float(w[e] << 16);
                acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red[sub][chunk * 8 + e] = acc[e];
        __syncthreads();
        if (tid < kHeadDim) {
            float s = 0.f;
#pragma unroll
            for (int g = 0; g < 16; ++g) s += red[g][tid];
            a.kmean[((static_cast<size_t>(slot) * a.heads + h) * a.nblk + b) * kHeadDim + tid] = s * (1.0f / 128.0f);
        }
        __syncthreads();  // red is reused by the next unit
    }
    // Launched as a programmatic dependent of the previous step's attention (it
    // writes a spare slot that kernel does not read), this grid completes only
    // after that kernel: whoever waits for this grid waits for both.  One CTA
    // waiting is enough for that (a grid completes when its last CTA exits); the
    // others exit at once and leave their SM slots to the kernels chained after
    // this one.
    if (blockIdx.x == 0) grid_dep_wait();
}

}  // namespace

cudaError_t launch_cache_append(const AppendArgs &a, bool pdl, cudaStream_t stream) {
    const int units = a.n_layers * a.heads * a.nblk;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int grid = units < 2 * sms ? units : 2 * sms;  // each CTA keeps 64 KB of loads in flight
    return launch_kernel(cache_append_kernel, dim3(grid), dim3(kThreads), 0, stream, pdl, a);
}

}  // namespace lcsa
