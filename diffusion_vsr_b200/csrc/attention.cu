// Block-sparse exact attention over kept 128x128 tiles on sm_100a.
//
// Operation: block_sparse_attn_func of the FlashVSR code walk-through
// ("FlashVSR 是怎么工作的", learn.html, section 2.2) / reading notes 关键设计 2:
// for every query token of a (2,8,8) block, softmax(q k^T * scale) V over the
// 128 tokens of each kept key block only; tiles that are not kept are never
// loaded or multiplied.
//
// Persistent kernel: one CTA per SM walks the (head, query block) rows
// blockIdx.x, blockIdx.x + gridDim.x, ... (head-major, so the CTAs running at
// the same time share the key/value tiles of one or two heads in L2).
// 384 threads, warp-specialised:
//   warp 0         producer: validates each row's kept list (whole warp; the
//                  next row's list is loaded one row ahead), then
//                  lane 0 issues the TMA copies — the Q tile straight from
//                  token layout (rank-4 box of 2 x 8 x 8 tokens x 64 dims, so
//                  the window partition costs nothing) into one of two Q
//                  buffers, and every kept K and V tile (block layout in the
//                  ring, two 16 KB boxes per tile) into separate K and V
//                  rings, 128-byte swizzled.  It runs ahead into the next row.
//   warps 1, 2     MMA issuers, one per softmax group (issuing a tcgen05.mma
//                  costs its thread ~90 cycles, so one issuer per group keeps
//                  the tensor pipe fed): S_w = Q K^T (both operands in shared
//                  memory, fp32 accumulator in TMEM) and O_w += P_w V (P read from
//                  TMEM, V from shared memory), in dependency order; the PV of a
//                  tile runs quarter by quarter (32 keys) as the softmax writes
//                  P.  A QK starts only once the CTA's previous QK (the other
//                  group's) completed, so the two groups run staggered: one
//                  group's softmax overlaps the other group's MMAs.
//   warps 4-7, 8-11 two softmax warpgroups.  Warpgroup w takes the kept tiles
//                  j = w, w+2, ... of a row with its own S and O in TMEM: one
//                  query row per thread, online softmax in the log2 domain with
//                  lazy rescaling of O (only when the row maximum grew by more
//                  than 2^8), P written as bf16 over S.  At the end of a row the
//                  group holding its last tile merges (m, l, O) of both groups,
//                  stages the bf16 output tile in the row's Q buffer and writes
//                  it with two TMA stores into token layout (the reverse
//                  partition); the other group hands over its (m, l) through
//                  shared memory and starts the next row at once.
//   warp 3         with RoPE only: rotates each Q tile in place once it has
//                  landed; the MMA issuers wait for the rotated tile.
// TMEM (512 columns): S_w at 128*w, O_w at 256 + 128*w.
// Launched as a programmatic dependent of the draft mask (LCSA_FLAG_PDL), the
// set-up overlaps the draft's tail and the producer waits for it before it
// reads any kept list.
// Every wait is bounded; on expiry the CTA drains its copies and MMAs, frees
// TMEM and reports LCSA_ERR_TIMEOUT.

#include "internal.h"
#include "ptx.cuh"
#include "rope.cuh"
#include "../../include/lcsa.h"

namespace lcsa {
namespace {

constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kTileBytes = 32768;
constexpr uint32_t kHalfBytes = 16384;
constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
// Registers: launched at 168 per thread (384 x 168 = 64,512); the control
// warpgroup gives registers to the two softmax warpgroups:
// 128 x 80 + 256 x 208 = 63,488 <= 64,512.
constexpr uint32_t kRegsControl = 80;
constexpr uint32_t kRegsSoftmax = 208;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows by > 2^8
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kInfoSlots = 4;  // rows the producer may publish ahead of the consumers

struct __align__(1024) AttnSmem {
    uint8_t q[2][kTileBytes];  // Q tiles of two consecutive rows; the (m, l) exchange of a
                               // row's epilogue lives in its Q buffer once its QKs are done
    uint8_t k[kKStages][kTileBytes];
    uint8_t v[kVStages][kTileBytes];
    uint64_t bar_qfull[2];
    uint64_t bar_qrot[2];   // with RoPE: the Q tile of the buffer is rotated (warp 3)
    uint64_t bar_qempty[2];
    uint64_t bar_kfull[kKStages];
    uint64_t bar_kempty[kKStages];
    uint64_t bar_vfull[kVStages];
    uint64_t bar_vempty[kVStages];
    uint64_t bar_sfull[2];
    uint64_t bar_pq[4][2];  // [quarter][group]: P of keys 32q..32q+31 written (quarter 0:
                            // also O rescaled)
    uint64_t bar_pvdone[2];
    uint64_t bar_ofinal;
    uint64_t bar_ofree;
    uint64_t bar_mlready;  // the early group's (m, l) of the row are in ml_early
    uint64_t bar_mlfree;   // the late group has read them
    uint64_t bar_drain[2];
    uint64_t bar_info_full[kInfoSlots];
    uint64_t bar_info_empty[kInfoSlots];
    int32_t info_n[kInfoSlots];  // validated kept count of row r in slot r % kInfoSlots
    uint32_t tmem_base;
    int32_t abort_word;
    float2 ml_early[128];  // (m, l) per query row of the group that finishes a row first
};

// the layout plus the 1 KB alignment slack fits the 227 KB a CTA may opt into
static_assert(sizeof(AttnSmem) + 1024 <= 232448, "shared memory layout too large");

__device__ __forceinline__ uint32_t col_s(int w) { return static_cast<uint32_t>(w) * 128u; }
__device__ __forceinline__ uint32_t col_o(int w) { return 256u + static_cast<uint32_t>(w) * 128u; }

// Kept tiles of a row, or 0 when its count or an index is out of range (whole
// warp).  cnt and idx0 (kept index number `lane` of the row) were prefetched.
__device__ __forceinline__ int row_tiles(const AttnArgs &a, int unit, int cnt, int idx0, int lane, bool &bad) {
    bad = cnt < 0 || cnt > a.topk;
    if (!bad) {
        if (lane < cnt) bad = idx0 < 0 || idx0 >= a.n_key_blocks;
        const int32_t *row = a.kept_idx + static_cast<size_t>(unit) * a.topk;
        for (int i = lane + 32; i < cnt; i += 32) {
            const int j = row[i];
            bad |= (j < 0 || j >= a.n_key_blocks);
        }
    }
    bad = __any_sync(0xffffffffu, bad);
    return bad ? 0 : cnt;
}

// Count and first 32 kept indices of row u (lane l: index l), or zeros past the end.
__device__ __forceinline__ void fetch_row(const AttnArgs &a, int u, int lane, int &cnt, int &idx) {
    cnt = 0;
    idx = 0;
    if (u < a.n_units) {
        cnt = __ldg(a.kept_cnt + u);
        if (lane < a.topk) idx = __ldg(a.kept_idx + static_cast<size_t>(u) * a.topk + lane);
    }
}

struct RowGeom {
    int h, ql, qby, qbx, frame0;
};

__device__ __forceinline__ int mul_div(int n, uint64_t m) {
    return static_cast<int>((static_cast<uint64_t>(static_cast<uint32_t>(n)) * m) >> 32);
}

__device__ __forceinline__ RowGeom row_geom(const AttnArgs &a, int unit) {
    RowGeom g;
    const int nq = a.q_layers * a.nblk;
    g.h = mul_div(unit, a.m_nq);
    const int qi = unit - g.h * nq;
    g.ql = mul_div(qi, a.m_nblk);
    const int qb = qi - g.ql * a.nblk;
    g.qby = mul_div(qb, a.m_gw);
    g.qbx = qb - g.qby * a.grid_w;
    g.frame0 = g.h * a.tq + g.ql * 2;  // first frame of the block in the Q/O maps
    return g;
}

// Descriptors of the first Q / K / V buffer; buffer i starts i * 32 KB later,
// which only moves the start-address field (addresses stay below 256 KB).
struct MmaCtx {
    uint32_t tmem, idesc_qk, idesc_pv;
    uint64_t qdesc0, kdesc0, vdesc0;
};

constexpr uint64_t kTileDescStep = kTileBytes >> 4;

// S_w = Q K_j^T for tile j of the current row (w = j & 1); t = the group's
// running tile count (all rows), gk = the running tile count of the CTA.
// prev_t >= 0: the CTA's previous tile belongs to the other group as its tile
// prev_t; this QK starts only once that QK completed, so the two groups' QKs
// alternate on the tensor pipe and their softmaxes run staggered.
__device__ __forceinline__ bool issue_qk(AttnSmem &sm, const MmaCtx &m, int qb, int w, int t, int gk, int prev_t,
                                         volatile int *abort_word, uint64_t to) {
    const int ks = gk % kKStages;
    if (!mbar_wait(smem_u32(&sm.bar_kfull[ks]), (gk / kKStages) & 1, abort_word, to)) return false;
    // S_w also holds P of this group's previous tile: that PV must have finished.
    if (t >= 1 && !mbar_wait(smem_u32(&sm.bar_pvdone[w]), (t - 1) & 1, abort_word, to)) return false;
    if (prev_t >= 0 && !mbar_wait(smem_u32(&sm.bar_sfull[1 - w]), prev_t & 1, abort_word, to)) return false;
    tc_fence_after();
    const uint64_t qd = m.qdesc0 + qb * kTileDescStep, kd = m.kdesc0 + ks * kTileDescStep;
    const uint32_t d = m.tmem + col_s(w);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        // K-major Q and K: 16 dims = 32 bytes per MMA inside the 128-byte
        // swizzle row; dims 64-127 live in the second 16 KB half.
        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
        mma_ss(d, qd + off, kd + off, m.idesc_qk, kk > 0 ? 1u : 0u);
    }
    mma_commit(smem_u32(&sm.bar_sfull[w]));
    mma_commit(smem_u32(&sm.bar_kempty[ks]));
    return true;
}

// O_w += P_w V_j for the group's tile; `first` = its first tile of the row.
__device__ __forceinline__ bool issue_pv(AttnSmem &sm, const MmaCtx &m, int w, int t, int gk, bool first, int act,
                                         volatile int *abort_word, uint64_t to) {
    const int vs = gk % kVStages;
    if (!mbar_wait(smem_u32(&sm.bar_vfull[vs]), (gk / kVStages) & 1, abort_word, to)) return false;
    // The first PV of a row overwrites O_w: the previous row's epilogue must
    // have read both accumulators.
    if (first && act >= 1 && !mbar_wait(smem_u32(&sm.bar_ofree), (act - 1) & 1, abort_word, to)) return false;
    const uint64_t vd = m.vdesc0 + vs * kTileDescStep;
    const uint32_t d = m.tmem + col_o(w), p = m.tmem + col_s(w);
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
        // each quarter of 32 keys as soon as its P is written
        const uint32_t bar = smem_u32(&sm.bar_pq[qq][w]);
        if (!mbar_wait(bar, t & 1, abort_word, to)) return false;
        tc_fence_after();
#pragma unroll
        for (int k4 = 0; k4 < 2; ++k4) {
            // 16 keys per MMA = two 8-row swizzle atoms (2 KB).
            const int kk = qq * 2 + k4;
            mma_ts(d, p + kk * 8, vd + static_cast<uint64_t>((kk * 2048) >> 4), m.idesc_pv,
                   (!first || kk > 0) ? 1u : 0u);
        }
    }
    mma_commit(smem_u32(&sm.bar_vempty[vs]));
    mma_commit(smem_u32(&sm.bar_pvdone[w]));
    return true;
}

// kRope: the Q tiles are rotated by warp 3 (RoPE) before the MMAs read them.
template <bool kRope>
__global__ void __launch_bounds__(kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                     const AttnArgs a, const AttnRope rope, uint16_t *__restrict__ out) {
    extern __shared__ uint8_t smem_raw[];
    AttnSmem &sm = *reinterpret_cast<AttnSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                  ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_word = &sm.abort_word;
    const uint64_t to = a.timeout_ns;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&sm.bar_qfull[b]), 1);
            mbar_init(smem_u32(&sm.bar_qrot[b]), 1);
            mbar_init(smem_u32(&sm.bar_qempty[b]), 1);  // the late group's output copy read the buffer
            mbar_init(smem_u32(&sm.bar_sfull[b]), 1);
            for (int qq = 0; qq < 4; ++qq) mbar_init(smem_u32(&sm.bar_pq[qq][b]), 4);  // one arrival per warp
            mbar_init(smem_u32(&sm.bar_drain[b]), 1);
            mbar_init(smem_u32(&sm.bar_pvdone[b]), 1);
        }
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(smem_u32(&sm.bar_kfull[s]), 1);
            mbar_init(smem_u32(&sm.bar_kempty[s]), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(smem_u32(&sm.bar_vfull[s]), 1);
            mbar_init(smem_u32(&sm.bar_vempty[s]), 1);
        }
        mbar_init(smem_u32(&sm.bar_ofinal), 2);  // one commit per MMA issuer
        mbar_init(smem_u32(&sm.bar_ofree), 4);    // the late group's warps read both accumulators
        mbar_init(smem_u32(&sm.bar_mlready), 4);  // the early group's warps
        mbar_init(smem_u32(&sm.bar_mlfree), 4);   // the late group's warps
        for (int i = 0; i < kInfoSlots; ++i) {
            mbar_init(smem_u32(&sm.bar_info_full[i]), 1);
            // 2 MMA issuers + 8 softmax warps (+ the rotation warp)
            mbar_init(smem_u32(&sm.bar_info_empty[i]), kRope ? 11 : 10);
        }
        sm.abort_word = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_o);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // Launched as a programmatic dependent of the draft mask, the set-up above
    // overlapped its tail; its kept lists (and the ring the append before it
    // wrote) are read only from here on.
    grid_dep_wait();
    // The next step's cache append may be launched as a programmatic dependent
    // (its blocks take the SMs this grid's CTAs leave; it writes a spare ring
    // slot).  Signalled only now: past the wait above, the previous step's
    // kernels, which read that slot, have completed.
    grid_dep_launch();

    // Copies issued by the producer (global counters), for the error-path drain.
    int k_issued = 0, v_issued = 0, q_issued = 0;

    if (warp < kSoftmaxWarp0) setmaxnreg_dec<kRegsControl>();
    if (warp == 0) {
        // ---------------------------------------------------------- producer
        // The whole warp walks the rows: it validates each kept list, publishes
        // the row's tile count to the consumers, and reads the kept indices 32 at
        // a time (one coalesced load, then shuffles; the count and the first 32
        // indices of the next row are loaded one row ahead); lane 0 issues the
        // copies.
        int g = 0, act = 0, r = 0;  // tiles, non-empty rows and rows so far
        bool ok = true;
        int cnt_next, idx_next;  // the next row's kept list, loaded one row ahead
        fetch_row(a, blockIdx.x, lane, cnt_next, idx_next);
        for (int unit = blockIdx.x; unit < a.n_units; unit += gridDim.x, ++r) {
            const int cnt = cnt_next, idx0 = idx_next;
            fetch_row(a, unit + gridDim.x, lane, cnt_next, idx_next);
            bool bad;
            const int n = row_tiles(a, unit, cnt, idx0, lane, bad);
            if (lane == 0) {
                if (bad && a.status) atomicOr(a.status, LCSA_ERR_BAD_INDEX);
                const int is = r % kInfoSlots;
                if (r >= kInfoSlots)
                    ok = mbar_wait(smem_u32(&sm.bar_info_empty[is]), ((r / kInfoSlots) - 1) & 1, abort_word, to);
                if (ok) {
                    sm.info_n[is] = n;
                    mbar_arrive(smem_u32(&sm.bar_info_full[is]));  // release: the count is visible
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            if (n == 0) continue;
            const RowGeom rg = row_geom(a, unit);
            const int qb = act & 1;
            if (lane == 0) {
                if (act >= 2)
                    ok = mbar_wait(smem_u32(&sm.bar_qempty[qb]), ((act >> 1) - 1) & 1, abort_word, to);
                if (ok) {
                    const uint32_t qf = smem_u32(&sm.bar_qfull[qb]);
                    mbar_arrive_expect_tx(qf, kTileBytes);
                    tma_load_4d(smem_u32(sm.q[qb]), &tm_q, qf, 0, rg.qbx * 8, rg.qby * 8, rg.frame0);
                    tma_load_4d(smem_u32(sm.q[qb]) + kHalfBytes, &tm_q, qf, 64, rg.qbx * 8, rg.qby * 8, rg.frame0);
                    q_issued = act + 1;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            const int32_t *kept_row = a.kept_idx + static_cast<size_t>(unit) * a.topk;
            int idx = 0;
            for (int j = 0; ok && j < n; ++j) {
                if ((j & 31) == 0) idx = j == 0 ? idx0 : ((j + lane < n) ? __ldg(kept_row + j + lane) : 0);
                const int kb = __shfl_sync(0xffffffffu, idx, j & 31);
                if (lane == 0) {
                    const int gk = g + j;
                    const int layer = mul_div(kb, a.m_nblk);
                    const int b = kb - layer * a.nblk;
                    int slot = a.oldest + layer;
                    if (slot >= a.capacity) slot -= a.capacity;
                    const int r0 = ((slot * a.heads + rg.h) * a.nblk + b) * kBlockTokens;
                    const int ks = gk % kKStages;
                    if (gk >= kKStages)
                        ok = mbar_wait(smem_u32(&sm.bar_kempty[ks]), ((gk / kKStages) - 1) & 1, abort_word, to);
                    if (ok) {
                        const uint32_t kf = smem_u32(&sm.bar_kfull[ks]);
                        mbar_arrive_expect_tx(kf, kTileBytes);
                        tma_load_2d(smem_u32(sm.k[ks]), &tm_k, kf, 0, r0);
                        tma_load_2d(smem_u32(sm.k[ks]) + kHalfBytes, &tm_k, kf, 64, r0);
                        k_issued = gk + 1;
                        const int vs = gk % kVStages;
                        if (gk >= kVStages)
                            ok = mbar_wait(smem_u32(&sm.bar_vempty[vs]), ((gk / kVStages) - 1) & 1, abort_word, to);
                        if (ok) {
                            const uint32_t vf = smem_u32(&sm.bar_vfull[vs]);
                            mbar_arrive_expect_tx(vf, kTileBytes);
                            tma_load_2d(smem_u32(sm.v[vs]), &tm_v, vf, 0, r0);
                            tma_load_2d(smem_u32(sm.v[vs]) + kHalfBytes, &tm_v, vf, 64, r0);
                            v_issued = gk + 1;
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            }
            if (!ok) break;
            g += n;
            ++act;
        }
        __syncwarp();
    } else if (warp == 1 || warp == 2) {
        // ---------------------------------------------- MMA issuer of group w
        // Tiles j = w, w+2, ... of each row: QK, then per tile PV (as P becomes
        // available) and the next QK into the same S buffer once that PV completed.
        const int w = warp - 1;
        if (lane == 0) {
            MmaCtx m;
            m.tmem = tmem;
            m.idesc_qk = idesc_bf16_f32(128, 128, 0);
            m.idesc_pv = idesc_bf16_f32(128, 128, 1);
            // Descriptors of the first buffer of each kind; per-MMA steps only move
            // the start address.  V is [key][dim]: dims (N) contiguous -> MN-major B
            // operand, the two 64-dim halves 16 KB apart (leading byte offset).
            m.qdesc0 = smem_desc_sw128(smem_u32(sm.q[0]), 16, 1024);
            m.kdesc0 = smem_desc_sw128(smem_u32(sm.k[0]), 16, 1024);
            m.vdesc0 = smem_desc_sw128(smem_u32(sm.v[0]), kHalfBytes, 1024);
            int g = 0, act = 0, r = 0;
            int t = 0;      // tiles of this group so far (all rows)
            int t_oth = 0;  // tiles of the other group before the current row
            int n_prev = 0; // tiles of the previous non-empty row
            bool ok = true;
            for (int unit = blockIdx.x; ok && unit < a.n_units; unit += gridDim.x, ++r) {
                const int is = r % kInfoSlots;
                if (!(ok = mbar_wait(smem_u32(&sm.bar_info_full[is]), (r / kInfoSlots) & 1, abort_word, to))) break;
                const int n = *reinterpret_cast<volatile int32_t *>(&sm.info_n[is]);
                mbar_arrive(smem_u32(&sm.bar_info_empty[is]));
                if (n == 0) continue;
                const int qb = act & 1;
                const int n_mine = (n - w + 1) >> 1;
                // the Q tile has landed (and, with RoPE, been rotated by warp 3)
                ok = mbar_wait(smem_u32(kRope ? &sm.bar_qrot[qb] : &sm.bar_qfull[qb]), (act >> 1) & 1, abort_word,
                               to);
                // Tile w + 2i of the row follows tile w + 2i - 1 of the other group
                // (for group 0's first tile: the previous row's last tile, when
                // that row had an even count).
                auto prev_of = [&](int i) -> int {
                    if (w == 1) return t_oth + i;
                    if (i >= 1) return t_oth + i - 1;
                    return (act >= 1 && (n_prev & 1) == 0) ? t_oth - 1 : -1;
                };
                if (ok && n_mine > 0) ok = issue_qk(sm, m, qb, w, t, g + w, prev_of(0), abort_word, to);
                for (int i = 0; ok && i < n_mine; ++i) {
                    ok = issue_pv(sm, m, w, t + i, g + w + 2 * i, i == 0, act, abort_word, to);
                    if (ok && i + 1 < n_mine)
                        ok = issue_qk(sm, m, qb, w, t + i + 1, g + w + 2 * (i + 1), prev_of(i + 1), abort_word, to);
                }
                // An issuer without a tile in this row has not waited for the
                // previous row's epilogue (its first PV would have): wait here,
                // so that its commit cannot count toward the previous row's
                // phase of bar_ofinal.
                if (ok && n_mine == 0 && act >= 1)
                    ok = mbar_wait(smem_u32(&sm.bar_ofree), (act - 1) & 1, abort_word, to);
                if (ok) mma_commit(smem_u32(&sm.bar_ofinal));
                t += n_mine;
                t_oth += n - n_mine;
                n_prev = n;
                g += n;
                ++act;
            }
            // Every MMA issued must be complete before TMEM is freed.
            mma_commit(smem_u32(&sm.bar_drain[w]));
            mbar_wait_drain(smem_u32(&sm.bar_drain[w]), 0, to);
        }
        __syncwarp();
    } else if (warp == 3) {
        // ------------------------------------------------- Q rotation (RoPE)
        // Lane l rotates pairs l (dims 2l, 2l+1, first 16 KB half of the Q tile)
        // and l + 32 (same place in the second half) of all 128 tokens, in place
        // in the 128-byte swizzled tile: token n's 16-byte chunk c sits at chunk
        // position c ^ (n & 7).  Pair l turns with the frame (l < 22) or the token
        // row; pair l + 32 with the token row (l < 11) or the token column.  (cos,
        // sin) are evaluated (fp64, rounded to fp32) per frame, row or column as
        // the rows of the tile are walked: few registers, as this warp runs with
        // the control warpgroup's budget.
        if (kRope) {
            const int p0 = lane, p1 = lane + 32;
            const int ax0 = rope_axis(p0), ax1 = rope_axis(p1);
            const double w0 = rope_freq(p0, rope.base), w1 = rope_freq(p1, rope.base);
            const uint32_t word = static_cast<uint32_t>(((lane >> 2) << 4) + (lane & 3) * 4);  // chunk, word
            int act = 0, r = 0;
            bool ok = true;
            for (int unit = blockIdx.x; unit < a.n_units; unit += gridDim.x, ++r) {
                const int is = r % kInfoSlots;
                ok = __all_sync(0xffffffffu,
                                mbar_wait(smem_u32(&sm.bar_info_full[is]), (r / kInfoSlots) & 1, abort_word, to));
                if (!ok) break;
                const int n = *reinterpret_cast<volatile int32_t *>(&sm.info_n[is]);
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sm.bar_info_empty[is]));
                if (n == 0) continue;
                const int qb = act & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.bar_qfull[qb]), (act >> 1) & 1, abort_word, to));
                if (!ok) break;
                const RowGeom rg = row_geom(a, unit);
                // column-band angles of pair l + 32 for the block's 8 token columns
                float2 cx[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) cx[x] = rope_cs(rg.qbx * 8 + x, w1);
                uint8_t *tile = sm.q[qb];
#pragma unroll 1
                for (int ty = 0; ty < 16; ++ty) {  // frame ty / 8, token row ty % 8 of the block
                    const int t = ty >> 3, y = ty & 7;
                    const float2 v0 = rope_cs(ax0 == 0 ? rope.frame0 + 2 * rg.ql + t : rg.qby * 8 + y, w0);
                    const float2 vy = rope_cs(rg.qby * 8 + y, w1);
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        const int tok = 8 * ty + x;
                        uint32_t *w_lo = reinterpret_cast<uint32_t *>(tile + tok * 128 + (word ^ (x << 4)));
                        uint32_t *w_hi = reinterpret_cast<uint32_t *>(tile + kHalfBytes + tok * 128 + (word ^ (x << 4)));
                        const float2 v1 = ax1 == 1 ? vy : cx[x];
                        *w_lo = rope_rotate(*w_lo, v0.x, v0.y);
                        *w_hi = rope_rotate(*w_hi, v1.x, v1.y);
                    }
                }
                fence_proxy_async_smem();  // the MMAs read the tile through the async proxy
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sm.bar_qrot[qb]));
                ++act;
            }
        }
        __syncwarp();
    } else if (warp >= kSoftmaxWarp0) {
        // ------------------------------------------------------- softmax
        setmaxnreg_inc<kRegsSoftmax>();
        const int w = (warp - kSoftmaxWarp0) >> 2;  // warpgroup 0 or 1
        const int quad = warp & 3;                   // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + col_s(w);
        const uint32_t o_addr = tmem + lane_off + col_o(w);
        const float c = a.scale_log2;
        const int tok_t = row >> 6, tok_y = (row >> 3) & 7, tok_x = row & 7;  // token of this row
        int act = 0, t = 0, r = 0;
        bool ok = true;
        // One thread per group issues the group's output copies.  The Q buffer
        // a copy reads from is handed back to the producer (bar_qempty) only
        // once the copy has read it, which is checked later, when it has long
        // completed, rather than waited for.
        const bool elected = quad == 0 && lane == 0;
        int pending_q = -1;
        auto release_q = [&](int b) {
            bulk_wait_group_read0();
            mbar_arrive(smem_u32(&sm.bar_qempty[b]));
            pending_q = -1;
        };
        for (int unit = blockIdx.x; unit < a.n_units; unit += gridDim.x, ++r) {
            const int is = r % kInfoSlots;
            if (ok)
                ok = __all_sync(0xffffffffu,
                                mbar_wait(smem_u32(&sm.bar_info_full[is]), (r / kInfoSlots) & 1, abort_word, to));
            // the four warps of the group leave together when a wait gave up
            // (constant barrier ids: the barrier count stays known)
            const bool go = !*abort_word;
            if (!(w == 0 ? named_bar_and(2, 128, ok && go) : named_bar_and(3, 128, ok && go))) {
                ok = false;
                break;
            }
            const int n = *reinterpret_cast<volatile int32_t *>(&sm.info_n[is]);
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.bar_info_empty[is]));
            const RowGeom rg = row_geom(a, unit);
            const size_t tok = (static_cast<size_t>(rg.frame0 + tok_t) * a.tok_h + rg.qby * 8 + tok_y) * a.tok_w +
                               rg.qbx * 8 + tok_x;
            uint4 *dst = reinterpret_cast<uint4 *>(out + tok * kHeadDim + w * 64);
            if (n == 0) {
                // nothing kept: zeros (lse -inf)
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int i = 0; i < 8; ++i) dst[i] = z;
                if (w == 0 && a.lse) a.lse[tok] = -INFINITY;
                continue;
            }
            const int qb = act & 1;
            const int n_mine = (n - w + 1) >> 1;  // tiles w, w+2, ...
            const int n_other = (n - (1 - w) + 1) >> 1;
            float m_used = -INFINITY;
            float l = 0.f;
            for (int i = 0; ok && i < n_mine; ++i, ++t) {
                if (act == 0 && i == 0 && w == 0 && (a.flags & LCSA_FLAG_FORCE_TIMEOUT)) {
                    *abort_word = 1;
                    ok = false;
                    break;
                }
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.bar_sfull[w]), t & 1, abort_word, to));
                if (!ok) break;
                tc_fence_after();
                uint32_t s[128];
                tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
                tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
                tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
                tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
                tmem_wait_ld();
                // row maximum: eight independent chains of 3-input maxima, then a small tree
                float mx8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float acc = fmax3(__uint_as_float(s[e]), __uint_as_float(s[8 + e]), __uint_as_float(s[16 + e]));
#pragma unroll
                    for (int k = 24; k < 120; k += 16)
                        acc = fmax3(acc, __uint_as_float(s[k + e]), __uint_as_float(s[k + 8 + e]));
                    mx8[e] = fmaxf(acc, __uint_as_float(s[120 + e]));
                }
                const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                const float m_new = mx * c;
                const bool warp_need = __any_sync(0xffffffffu, m_new > m_used + kRescaleThreshold);
                float m_next = m_used;
                float alpha = 1.f;
                if (warp_need) {
                    m_next = fmaxf(m_used, m_new);
                    alpha = ex2_approx(m_used - m_next);
                }
                if (warp_need && i > 0) {
                    // Rescale O_w before this tile's PV accumulates into it.  O_w is
                    // stable: the QK of this tile was issued only after the group's
                    // previous PV completed (it reuses S_w).
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + cc * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                        tmem_st32(o_addr + cc * 32, o);
                    }
                }
                // P = 2^(s*c - m) (scale and shift as packed f32x2 FMAs), summed in
                // eight independent chains (four packed pairs), packed to bf16 and
                // written over S in four 32-key quarters, each announced as soon as it
                // is in TMEM so that its PV MMAs can start.
                const uint64_t c2 = f32x2_pack(c, c), nm2 = f32x2_pack(-m_next, -m_next);
                uint64_t sum4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int col = qq * 32 + 2 * k;
                        float x0, x1;
                        f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(s[col]), __uint_as_float(s[col + 1])), c2, nm2),
                                     x0, x1);
                        const float p0 = ex2_approx(x0);
                        const float p1 = ex2_approx(x1);
                        sum4[k & 3] = f32x2_add(sum4[k & 3], f32x2_pack(p0, p1));
                        pk[k] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(s_addr + qq * 16, pk);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&sm.bar_pq[qq][w]));
                }
                float sum8[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) f32x2_unpack(sum4[e], sum8[2 * e], sum8[2 * e + 1]);
                const float rs =
                    ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
                l = l * alpha + rs;
                m_used = m_next;
                if (i == 0 && elected && pending_q >= 0) release_q(pending_q);
            }
            const int late = (n - 1) & 1;  // the group of the row's last tile runs the epilogue
            if (w != late) {
                // ---------------------------------------------- early group
                // Hand this group's (m, l) of the row to the late group, once that
                // has read the previous row's, and go on to the next row: its first
                // tile overlaps the late group's epilogue (its PV waits for the
                // accumulators to be read, bar_ofree).
                if (ok && act >= 1)
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(smem_u32(&sm.bar_mlfree), (act - 1) & 1, abort_word, to));
                if (ok) {
                    sm.ml_early[row] = make_float2(m_used, l);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&sm.bar_mlready));  // release: ml_early written
                    if (elected && pending_q >= 0) release_q(pending_q);
                }
                ++act;
                continue;
            }
            // -------------------------------------------- late group: epilogue
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.bar_ofinal), act & 1, abort_word, to));
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.bar_mlready), act & 1, abort_word, to));
            // the group's warps take the same decision on going through the epilogue
            const bool go_epi = !*abort_word;
            if (!(w == 0 ? named_bar_and(2, 128, ok && go_epi) : named_bar_and(3, 128, ok && go_epi))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float2 mle = sm.ml_early[row];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.bar_mlfree));
            const float m_o = mle.x, l_o = mle.y;
            const float m = fmaxf(m_used, m_o);
            const float a_self = ex2_approx(m_used - m);  // the late group always holds a tile
            const float a_oth = n_other > 0 ? ex2_approx(m_o - m) : 0.f;
            const float L = l * a_self + l_o * a_oth;
            const float inv_l = L > 0.f ? 1.f / L : 0.f;
            const float f_self = a_self * inv_l, f_oth = a_oth * inv_l;
            // Both 64-dim halves of the row's output, one at a time: the two
            // accumulators read, merged, packed to bf16 and staged in the row's Q
            // buffer (every QK of the row completed), 128-byte swizzled as the TMA
            // box expects (row = token of the block, 16-byte chunk c of the row at
            // chunk position c ^ (row & 7)).
            uint8_t *tile = sm.q[qb];
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[2][16];
                uint32_t o0[2][32], o1[2][32];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint32_t col = static_cast<uint32_t>(h * 64 + cc * 32);
                    // (without tiles the early group's accumulator is stale: read, not used)
                    tmem_ld32(tmem + lane_off + col_o(w) + col, o0[cc]);
                    tmem_ld32(tmem + lane_off + col_o(1 - w) + col, o1[cc]);
                }
                tmem_wait_ld();
                if (n_other > 0) {  // (uniform over the group) both accumulators hold tiles
                    const uint64_t fs2 = f32x2_pack(f_self, f_self), fo2 = f32x2_pack(f_oth, f_oth);
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const uint64_t b = f32x2_mul(
                                f32x2_pack(__uint_as_float(o1[cc][2 * k]), __uint_as_float(o1[cc][2 * k + 1])), fo2);
                            float r0, r1;
                            f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(o0[cc][2 * k]),
                                                              __uint_as_float(o0[cc][2 * k + 1])),
                                                   fs2, b),
                                         r0, r1);
                            pk[cc][k] = pack_bf16x2(r0, r1);
                        }
                    }
                } else {
                    // the early group had no tile
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            pk[cc][k] = pack_bf16x2(__uint_as_float(o0[cc][2 * k]) * f_self,
                                                    __uint_as_float(o0[cc][2 * k + 1]) * f_self);
                    }
                }
                uint8_t *half_buf = tile + h * kHalfBytes;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
                    for (int qd = 0; qd < 4; ++qd) {
                        const int chunk = cc * 4 + qd;
                        *reinterpret_cast<uint4 *>(half_buf + row * 128 + ((chunk ^ (row & 7)) << 4)) =
                            make_uint4(pk[cc][4 * qd], pk[cc][4 * qd + 1], pk[cc][4 * qd + 2], pk[cc][4 * qd + 3]);
                    }
                }
            }
            // O of both groups has been read: the next row's PVs may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.bar_ofree));
            if (a.lse) a.lse[tok] = L > 0.f ? (m + __log2f(L)) * kLn2 : -INFINITY;
            // the staged tile goes out with two TMA stores (one per 64-dim half)
            // into token layout (the reverse partition)
            fence_proxy_async_smem();
            if (w == 0) named_bar_sync(4, 128);  // (constant ids: the barrier count stays known)
            else named_bar_sync(5, 128);
            if (elected) {
                if (pending_q >= 0) release_q(pending_q);
                tma_store_4d(&tm_o, smem_u32(tile), 0, rg.qbx * 8, rg.qby * 8, rg.frame0);
                tma_store_4d(&tm_o, smem_u32(tile) + kHalfBytes, 64, rg.qbx * 8, rg.qby * 8, rg.frame0);
                bulk_commit_group();
                pending_q = qb;  // released once the copy has read it (this group's next tile)
            }
            ++act;
        }
        // the output copies of this group have landed before the CTA exits
        if (elected) {
            if (pending_q >= 0) release_q(pending_q);
            bulk_wait_group0();
        }
    }

    __syncthreads();
    if (sm.abort_word && warp == 0 && lane == 0) {
        // Error path: every copy still in flight must land before the CTA exits.
        for (int i = (q_issued > 2 ? q_issued - 2 : 0); i < q_issued; ++i)
            mbar_wait_drain(smem_u32(&sm.bar_qfull[i & 1]), (i >> 1) & 1, to);
        for (int j = (k_issued > kKStages ? k_issued - kKStages : 0); j < k_issued; ++j)
            mbar_wait_drain(smem_u32(&sm.bar_kfull[j % kKStages]), (j / kKStages) & 1, to);
        for (int j = (v_issued > kVStages ? v_issued - kVStages : 0); j < v_issued; ++j)
            mbar_wait_drain(smem_u32(&sm.bar_vfull[j % kVStages]), (j / kVStages) & 1, to);
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && sm.abort_word && a.status) atomicOr(a.status, LCSA_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_attention(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                             const CUtensorMap &tm_o, const AttnArgs &a, const AttnRope &rope, bool pdl, void *out,
                             const DeviceInfo &dev, cudaStream_t stream) {
    static std::atomic<int> smem_set[2][kMaxDevices];
    const size_t smem = sizeof(AttnSmem) + 1024;
    const bool rot = rope.base != 0.f;
    const cudaError_t e = rot ? ensure_smem_limit(attention_kernel<true>, dev.device, smem, smem_set[1])
                              : ensure_smem_limit(attention_kernel<false>, dev.device, smem, smem_set[0]);
    if (e != cudaSuccess) return e;
    const int grid = a.n_units < dev.sms ? a.n_units : dev.sms;
    if (rot)
        return launch_kernel(attention_kernel<true>, dim3(grid), dim3(kThreads), smem, stream, pdl, tm_q, tm_k, tm_v,
                             tm_o, a, rope, static_cast<uint16_t *>(out));
    return launch_kernel(attention_kernel<false>, dim3(grid), dim3(kThreads), smem, stream, pdl, tm_q, tm_k, tm_v, tm_o,
                         a, rope, static_cast<uint16_t *>(out));
}

}  // namespace lcsa
