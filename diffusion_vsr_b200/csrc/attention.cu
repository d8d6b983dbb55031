// Block-sparse exact attention over kept 128x128 tiles on sm_100a.
//
// Operation: block_sparse_attn_func of the FlashVSR code walk-through
// ("FlashVSR 是怎么工作的", learn.html, section 2.2) / reading notes 关键设计 2:
// for every query token of a (2,8,8) block, softmax(q k^T * scale) V over the
// 128 tokens of each kept key block only; tiles that are not kept are never
// loaded or multiplied.
//
// One CTA per (head, query block) row, 256 threads, warp-specialised:
//   warp 0 lane 0  producer: TMA of the Q tile (straight from token layout:
//                  a rank-4 box of 2 x 8 x 8 tokens x 64 dims, so the window
//                  partition costs nothing) and of each kept K/V tile (block
//                  layout in the ring, two 16 KB boxes per tile) into a
//                  3-stage shared-memory ring, 128-byte swizzled;
//   warp 1 lane 0  MMA issuer: S = Q K^T (tcgen05.mma, both operands in
//                  shared memory, fp32 accumulator in TMEM, double-buffered)
//                  and O += P V (P read from TMEM, V from shared memory);
//   warps 4-7      softmax: one query row per thread; reads S from TMEM,
//                  online softmax in the log2 domain with lazy rescaling of O
//                  (only when the row maximum grew by more than 2^8), writes
//                  P as bf16 back over S, and finally normalises O and stores
//                  it with a TMA store into token layout (reverse partition).
// TMEM: S0 cols [0,128), S1 [128,256), O [256,384) of a 512-column allocation.
// Every wait is bounded; on expiry the CTA drains its copies and MMAs, frees
// TMEM and reports LCSA_ERR_TIMEOUT.

#include "internal.h"
#include "ptx.cuh"
#include "../../include/lcsa.h"

namespace lcsa {
namespace {

constexpr int kStages = 3;
constexpr uint32_t kTileBytes = 32768;
constexpr uint32_t kHalfBytes = 16384;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows by > 2^8
constexpr float kLn2 = 0.6931471805599453f;

struct __align__(1024) AttnSmem {
    uint8_t q[kTileBytes];  // Q tile; reused as the bf16 output staging tile
    uint8_t k[kStages][kTileBytes];
    uint8_t v[kStages][kTileBytes];
    uint64_t bar_q;
    uint64_t bar_kfull[kStages];
    uint64_t bar_vfull[kStages];
    uint64_t bar_empty[kStages];
    uint64_t bar_sfull[2];
    uint64_t bar_pfull[2];
    uint64_t bar_pvdone;
    uint64_t bar_ofinal;
    uint64_t bar_drain;
    uint32_t tmem_base;
    int32_t n_tiles;
    int32_t abort_word;
};

__global__ void __launch_bounds__(kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                     const AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    AttnSmem &sm = *reinterpret_cast<AttnSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                  ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.x;
    const int nq = a.q_layers * a.nblk;
    const int h = unit / nq;
    const int qi = unit - h * nq;
    const int ql = qi / a.nblk;
    const int qb = qi - ql * a.nblk;
    const int qby = qb / a.grid_w;
    const int qbx = qb - qby * a.grid_w;
    const int frame0 = h * a.tq + ql * 2;  // coordinate of the block's first frame in the Q/O maps
    volatile int *abort_word = &sm.abort_word;
    const uint64_t to = a.timeout_ns;
    const int32_t *kept_row = a.kept_idx + static_cast<size_t>(unit) * a.topk;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&sm.bar_q), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&sm.bar_kfull[s]), 1);
            mbar_init(smem_u32(&sm.bar_vfull[s]), 1);
            mbar_init(smem_u32(&sm.bar_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&sm.bar_sfull[b]), 1);
            mbar_init(smem_u32(&sm.bar_pfull[b]), 128);
        }
        mbar_init(smem_u32(&sm.bar_pvdone), 1);
        mbar_init(smem_u32(&sm.bar_ofinal), 1);
        mbar_init(smem_u32(&sm.bar_drain), 1);
        sm.abort_word = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        // Validate the kept list of this row before anything is loaded.
        const int cnt = a.kept_cnt[unit];
        bool bad = cnt < 0 || cnt > a.topk;
        if (!bad) {
            for (int i = lane; i < cnt; i += 32) {
                const int j = kept_row[i];
                bad |= (j < 0 || j >= a.n_key_blocks);
            }
        }
        bad = __any_sync(0xffffffffu, bad);
        if (lane == 0) {
            sm.n_tiles = bad ? 0 : cnt;
            if (bad && a.status) atomicOr(a.status, LCSA_ERR_BAD_INDEX);
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            prefetch_tensormap(&tm_o);
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int n = sm.n_tiles;

    const uint32_t bar_q = smem_u32(&sm.bar_q);
    const uint32_t q_smem = smem_u32(sm.q);
    int issued = 0;  // K/V tiles whose loads the producer issued

    if (warp == 0) {
        if (lane == 0 && n > 0) {
            // ------------------------------------------------------ producer
            mbar_arrive_expect_tx(bar_q, kTileBytes);
            tma_load_4d(q_smem, &tm_q, bar_q, 0, qbx * 8, qby * 8, frame0);
            tma_load_4d(q_smem + kHalfBytes, &tm_q, bar_q, 64, qbx * 8, qby * 8, frame0);
            for (int j = 0; j < n; ++j) {
                const int s = j % kStages;
                if (j >= kStages &&
                    !mbar_wait(smem_u32(&sm.bar_empty[s]), ((j / kStages) - 1) & 1, abort_word, to))
                    break;
                const int kb = kept_row[j];
                const int layer = kb / a.nblk;
                const int b = kb - layer * a.nblk;
                int slot = a.oldest + layer;
                if (slot >= a.capacity) slot -= a.capacity;
                const int r0 = ((slot * a.heads + h) * a.nblk + b) * kBlockTokens;
                const uint32_t kf = smem_u32(&sm.bar_kfull[s]);
                const uint32_t vf = smem_u32(&sm.bar_vfull[s]);
                mbar_arrive_expect_tx(kf, kTileBytes);
                tma_load_2d(smem_u32(sm.k[s]), &tm_k, kf, 0, r0);
                tma_load_2d(smem_u32(sm.k[s]) + kHalfBytes, &tm_k, kf, 64, r0);
                mbar_arrive_expect_tx(vf, kTileBytes);
                tma_load_2d(smem_u32(sm.v[s]), &tm_v, vf, 0, r0);
                tma_load_2d(smem_u32(sm.v[s]) + kHalfBytes, &tm_v, vf, 64, r0);
                issued = j + 1;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && n > 0) {
            // ---------------------------------------------------- MMA issuer
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 1);
            const uint32_t pvdone = smem_u32(&sm.bar_pvdone);
            auto issue_pv = [&](int i) -> bool {
                const int s = i % kStages;
                const int b = i & 1;
                if (!mbar_wait(smem_u32(&sm.bar_vfull[s]), (i / kStages) & 1, abort_word, to)) return false;
                if (!mbar_wait(smem_u32(&sm.bar_pfull[b]), (i >> 1) & 1, abort_word, to)) return false;
                tc_fence_after();
                const uint32_t v_smem = smem_u32(sm.v[s]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // V is [key][dim]: dims (N) contiguous -> MN-major B operand.
                    // 16 keys per MMA = two 8-row swizzle atoms (2 KB); the two
                    // 64-dim halves are 16 KB apart (leading byte offset).
                    const uint64_t bdesc = smem_desc_sw128(v_smem + kk * 2048, kHalfBytes, 1024);
                    mma_ts(tmem + kColO, tmem + (b ? 128u : 0u) + kk * 8, bdesc, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(smem_u32(&sm.bar_empty[s]));
                mma_commit(pvdone);
                return true;
            };
            bool ok = mbar_wait(bar_q, 0, abort_word, to);
            for (int j = 0; ok && j < n; ++j) {
                const int s = j % kStages;
                const int b = j & 1;
                if (!mbar_wait(smem_u32(&sm.bar_kfull[s]), (j / kStages) & 1, abort_word, to)) {
                    ok = false;
                    break;
                }
                // S[b] also holds P of tile j-2: wait until that PV finished reading it.
                if (j >= 2 && !mbar_wait(pvdone, (j - 2) & 1, abort_word, to)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t k_smem = smem_u32(sm.k[s]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // K-major Q and K: 16 dims = 32 bytes per MMA inside the
                    // 128-byte swizzle row; dims 64-127 live in the second half.
                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + (b ? 128u : 0u), smem_desc_sw128(q_smem + off, 16, 1024),
                           smem_desc_sw128(k_smem + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(&sm.bar_sfull[b]));
                if (j >= 1 && !issue_pv(j - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok) ok = issue_pv(n - 1);
            if (ok) mma_commit(smem_u32(&sm.bar_ofinal));
            // Every MMA issued must be complete before TMEM is freed.
            mma_commit(smem_u32(&sm.bar_drain));
            mbar_wait_drain(smem_u32(&sm.bar_drain), 0, to);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------- softmax
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const float c = a.scale_log2;
        float m_used = -INFINITY;
        float l = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int b = j & 1;
            if (j == 0 && (a.flags & LCSA_FLAG_FORCE_TIMEOUT)) {
                *abort_word = 1;
                ok = false;
                break;
            }
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.bar_sfull[b]), (j >> 1) & 1, abort_word, to));
            if (!ok) break;
            tc_fence_after();
            uint32_t s[128];
            tmem_ld32(tmem + lane_off + (b ? 128u : 0u) + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
            tmem_ld32(tmem + lane_off + (b ? 128u : 0u) + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
            tmem_ld32(tmem + lane_off + (b ? 128u : 0u) + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
            tmem_ld32(tmem + lane_off + (b ? 128u : 0u) + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
            tmem_wait_ld();
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 128; ++i) mx = fmaxf(mx, __uint_as_float(s[i]));
            const float m_new = mx * c;
            const bool warp_need = __any_sync(0xffffffffu, m_new > m_used + kRescaleThreshold);
            float m_next = m_used;
            float alpha = 1.f;
            if (warp_need) {
                m_next = fmaxf(m_used, m_new);
                alpha = ex2_approx(m_used - m_next);
            }
            float rs = 0.f;
            uint32_t pk[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(s[2 * i]), c, -m_next));
                const float p1 = ex2_approx(fmaf(__uint_as_float(s[2 * i + 1]), c, -m_next));
                rs += p0 + p1;
                pk[i] = pack_bf16x2(p0, p1);
            }
            l = l * alpha + rs;
            tmem_st32(tmem + lane_off + (b ? 128u : 0u) + 0, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
            tmem_st32(tmem + lane_off + (b ? 128u : 0u) + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
            if (warp_need && j > 0) {
                // O must hold the finished PV of tile j-1 before it is rescaled.
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.bar_pvdone), (j - 1) & 1, abort_word, to));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + kColO + cc * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(tmem + lane_off + kColO + cc * 32, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&sm.bar_pfull[b]));
            m_used = m_next;
        }
        if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.bar_ofinal), 0, abort_word, to));
        if (ok) {
            // --------------------------------------------------- epilogue
            tc_fence_after();
            const float inv_l = n > 0 ? 1.f / l : 0.f;
            const uint32_t row_base = q_smem + static_cast<uint32_t>(row) * 128;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t o[32];
                if (n > 0) {
                    tmem_ld32(tmem + lane_off + kColO + cc * 32, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
                // 32 columns = 64 bytes = four 16-byte chunks of the 128-byte
                // swizzled row of half (cc >> 1); chunk index XOR (row % 8).
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const uint32_t chunk = static_cast<uint32_t>((cc & 1) * 4 + qd);
                    const uint32_t addr = row_base + (cc >> 1) * kHalfBytes + ((chunk ^ (row & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * qd]),
                                 "r"(pk[4 * qd + 1]), "r"(pk[4 * qd + 2]), "r"(pk[4 * qd + 3])
                                 : "memory");
                }
            }
            if (a.lse) {
                const int t = row >> 6, y = (row >> 3) & 7, x = row & 7;
                const size_t idx = (static_cast<size_t>(frame0 + t) * a.tok_h + qby * 8 + y) * a.tok_w + qbx * 8 + x;
                a.lse[idx] = n > 0 ? (m_used + __log2f(l)) * kLn2 : -INFINITY;
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (row == 0) {
                tma_store_4d(&tm_o, q_smem, 0, qbx * 8, qby * 8, frame0);
                tma_store_4d(&tm_o, q_smem + kHalfBytes, 64, qbx * 8, qby * 8, frame0);
                bulk_commit_group();
                bulk_wait_group_read0();
            }
        }
    }

    __syncthreads();
    if (sm.abort_word && warp == 0 && lane == 0 && n > 0) {
        // Error path: every copy still in flight must land before the CTA exits.
        mbar_wait_drain(bar_q, 0, to);
        for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j) {
            const int s = j % kStages;
            mbar_wait_drain(smem_u32(&sm.bar_kfull[s]), (j / kStages) & 1, to);
            mbar_wait_drain(smem_u32(&sm.bar_vfull[s]), (j / kStages) & 1, to);
        }
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && sm.abort_word && a.status) atomicOr(a.status, LCSA_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_attention(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                             const CUtensorMap &tm_o, const AttnArgs &a, cudaStream_t stream) {
    const size_t smem = sizeof(AttnSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attention_kernel<<<a.n_units, kThreads, smem, stream>>>(tm_q, tm_k, tm_v, tm_o, a);
    return cudaGetLastError();
}

}  // namespace lcsa
