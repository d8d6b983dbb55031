// Kept lists of segment-masked dense attention on sm_100a.
//
// Operation: the Stage-1 teacher of the reading notes "FlashVSR: Towards
// Real-time Diffusion-Based Streaming Video Super Resolution", 关键设计 1 (the
// alpha_ij equation): over a packed sequence of clips (videos, and images as
// single-frame videos) every token attends to every token of its own segment
// and to none of any other.  With the sequence cut into 128-token tiles and
// every segment a whole number of tiles, that attention is the block-sparse
// attention whose kept list of a query tile is every key tile of its segment:
// this kernel writes those lists, and lcsa_attention computes the attention
// exactly over them (dense inside a segment, nothing across).
//
// One warp per (head, query tile) row: the segment is found by a binary
// search over the segments' first tiles; lane l writes entries l, l + 32, ...
// of the row (the segment's tiles in ascending order, then -1).

#include "internal.h"
#include "../../include/lcsa.h"

namespace lcsa {
namespace {

constexpr int kWarpsPerBlock = 8;

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    segment_mask_kernel(const __grid_constant__ SegmentArgs a) {
    const int row = static_cast<int>(blockIdx.x) * kWarpsPerBlock + static_cast<int>(threadIdx.x >> 5);
    if (row >= a.heads * a.tiles) return;
    const int lane = threadIdx.x & 31;
    const int i = row % a.tiles;  // query tile
    // segment s with start[s] <= i < start[s + 1]
    int lo = 0, hi = a.n_seg;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (a.start[mid] <= i) lo = mid;
        else hi = mid;
    }
    const int s0 = a.start[lo];
    const int n = a.start[lo + 1] - s0;
    int32_t *out = a.kept_idx + static_cast<size_t>(row) * a.topk;
    for (int j = lane; j < a.topk; j += 32) out[j] = j < n ? s0 + j : -1;
    if (lane == 0) a.kept_cnt[row] = n;
}

}  // namespace

cudaError_t launch_segment_mask(const SegmentArgs &a, cudaStream_t stream) {
    const int rows = a.heads * a.tiles;
    const int grid = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
    return launch_kernel(segment_mask_kernel, dim3(grid), dim3(kWarpsPerBlock * 32), 0, stream, false, a);
}

}  // namespace lcsa
