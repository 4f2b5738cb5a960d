// Block attention backward, dK/dV pass (key-tile stationary), sm_100a.
//
// For one 128-key tile of one (example, head) this kernel visits the query
// tiles that can see it (from the diagonal to the last query whose window
// still reaches the tile) and accumulates, with P recomputed from the
// forward's lse and Delta from the dQ pass:
//   dV = sum_i P_i^T dO_i,   dK = (1/sqrt(D)) sum_i dS_i^T Q_i,
//   dS_i = P_i o (dO_i V^T - Delta_i).
// dK and dV are accumulated on chip and written once; nothing is reduced
// across CTAs.
//
// Tensor-core plan per query tile i (tcgen05, fp32 accumulators in TMEM):
//   S^T  = K Q_i^T    A = K smem, B = Q_i smem (both K-major)
//   dP^T = V dO_i^T   A = V smem, B = dO_i smem
//   dV  += P^T dO_i   A = P^T from TMEM (bf16), B = dO_i smem (MN-major)
//   dK  += dS^T Q_i   A = dS^T from TMEM (bf16), B = Q_i smem (MN-major)
//
// MMA order per query tile m (one issuing thread, so the tensor pipe runs
// them in this order):
//   ... dV(m-1) | S^T(m) | dK(m-1) | dP^T(m) | dV(m) | S^T(m+1) | dK(m) ...
// dV(m) needs only P^T(m), so it is issued as soon as the compute warps have
// turned S^T(m) into P^T(m); S^T(m+1) then reuses those columns. dK(m) waits
// for dS^T(m) and dP^T(m+1) reuses its columns. The compute warps alternate
// P (phase A) and dS (phase B) while the tensor core runs the products of the
// other phase, so the per-tile time is the larger of the two, not their sum.
// Q and dO sit in separate rings: dO(m) is free after dV(m), Q(m) after dK(m).
//
// CTA roles (persistent, round-robin over (key tile, head) items):
//   warps 0-3 / 4-7  two compute warpgroups; thread t owns key row t (TMEM
//              lane t), group g the queries [64g, 64g+64) of each query tile.
//              Phase A: read S^T, write P^T (bf16) over the first 32 of the
//              group's S^T columns. Phase B: read dP^T, write dS^T (bf16) over
//              the first 32 of the group's dP^T columns.
//   warps 8-11 epilogue: at the end of an item, move dV and dK from TMEM to
//              global memory while the compute warps start the next item.
//   warp 12    TMA producer: K, V per item (with an L2 prefetch of the next
//              item's); Q and dO per query tile into their rings, with an L2
//              prefetch two tiles ahead.
//   warp 13    MMA issuer.
// TMEM columns: S^T / P^T [0,128), dP^T / dS^T [128,256), dV [256, 256+D),
// dK [256+D, 256+2D).
//
// Fused backward (kDq; masks under which every query tile sees only its own key
// tile, so each item has one query tile, the key tile's own rows): the same pass
// also forms dQ = (1/sqrt(D)) dS K. The compute warps write dS a second time, as
// bf16 into shared memory with the keys as rows (the MN-major A operand of
// dQ = dS K; TMEM holds dS^T with the keys on the lanes, the wrong way round for
// an A operand), and dQ accumulates over the dS^T columns after the dK product
// has read them. The epilogue stores dQ first, which frees those columns for the
// next item's dP^T. Keys past the example enter the dQ sum, so their dS is
// written as zero and an example's partial key tile is read from a zero-padded
// copy. -Delta and -lse log2(e) come from a separate per-row pass.
#include "ba_common.cuh"
#include "ba_kernels.cuh"
#include "ba_ptx.cuh"
#include "ba_sched.cuh"

#include <cuda_bf16.h>

namespace ba {

namespace {

template <int D, bool kDq = false>
struct DkvLayout {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkBytes = kTile * 128;
    static constexpr int kTileBytes = kTile * D * 2;
    // Q ring and dO ring. Q(m) is read until dK(m), late in tile m's step, and
    // S^T(m+1) needs Q(m+1): three Q slots keep its load well ahead. dO(m) is free
    // after dV(m), early in the step, so at D = 128 one dO slot is enough.
    // The fused backward has one query tile per item, and its dS buffer takes a slot's room.
    static constexpr int kQSlots = kDq ? 2 : (D == 64 ? 4 : 3);
    static constexpr int kOSlots = kDq ? (D == 64 ? 2 : 1) : (D == 64 ? 4 : 1);
    static constexpr int kK = 0;
    static constexpr int kV = kTileBytes;
    static constexpr int kQ0 = 2 * kTileBytes;           // Q slot s at kQ0 + s tile
    static constexpr int kO0 = kQ0 + kQSlots * kTileBytes; // dO slot s at kO0 + s tile
    static constexpr int kStage = kO0 + kOSlots * kTileBytes; // epilogue staging: 128 rows x 64 columns
    // fused backward: dS (bf16) as two 64-query chunks of 128 key rows, 128-byte swizzled
    static constexpr int kDS = kStage + kChunkBytes;
    static constexpr int kDSChunkBytes = kTile * 128;
    static constexpr int kBytes = kDS + (kDq ? 2 * kDSChunkBytes : 0);
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr int kThreads = 448;
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
    static constexpr uint32_t kColDQ = kColDP; // fused backward: over dS^T once dK has read it
    static constexpr uint32_t kTmemCols = 512;
};

struct DkvBarriers {
    uint64_t k_full, k_empty, v_full, v_empty, dkv_full, dv_free, dk_free, dq_free;
    uint64_t q_full[4], q_empty[4], o_full[4], o_empty[4];
    uint64_t s_full, dp_full, pa_done[2], pb_done[2];
    uint64_t epi_sync; // group barrier of the epilogue warps
    ItemRing ring;     // unused: this pass deals its items statically (StaticItems)
    uint32_t tmem_base;
    int abort;
    // per Q slot: -lse in log2 units and -Delta of the tile's 128 queries
    // (-inf and 0 past the example's end), filled with the Q tile
    __align__(16) float stat[4][2][kTile];
};

template <bool kCross>
__device__ __forceinline__ void query_tile_range(const TileRef &r, int64_t B, int64_t W, int &ilo, int &ihi)
{
    if (kCross) { // cross-attention: every query tile of the example's own query set
        ilo = 0;
        ihi = (r.oL + kTile - 1) / kTile - 1;
        return;
    }
    const int64_t kmax = (int64_t(r.t) * kTile + kTile < r.L ? int64_t(r.t) * kTile + kTile : r.L) - 1;
    ilo = r.t;
    ihi = int(last_query_seeing(kmax, r.L, B, W) / kTile);
}

} // namespace

template <int D, bool kRope, int A, bool kCross, bool kDq>
__global__ void __launch_bounds__(448, 1)
    bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                          const __grid_constant__ CUtensorMap tm_qt, const __grid_constant__ CUtensorMap tm_dot,
                          const Problem p, const float *__restrict__ nlse2, const float *__restrict__ neg_delta,
                          __nv_bfloat16 *__restrict__ dk, __nv_bfloat16 *__restrict__ dv,
                          const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_dq,
                          __nv_bfloat16 *__restrict__ dq)
{
    using Lay = DkvLayout<D, kDq>;
    constexpr int QS = Lay::kQSlots, OS = Lay::kOSlots;
    extern __shared__ uint8_t smem_raw[];
    __shared__ DkvBarriers sb;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&sb.k_full, 1);
        mbar_init(&sb.k_empty, 1);
        mbar_init(&sb.v_full, 1);
        mbar_init(&sb.v_empty, 1);
        mbar_init(&sb.dkv_full, 1);
        mbar_init(&sb.dv_free, 4);
        mbar_init(&sb.dk_free, 4);
        mbar_init(&sb.dq_free, 4);
        for (int i = 0; i < 4; ++i) {
            mbar_init(&sb.q_full[i], 1 + 32); // the Q tile's expect_tx arrival + one per lane's copies
            mbar_init(&sb.q_empty[i], 1);
            mbar_init(&sb.o_full[i], 1);
            mbar_init(&sb.o_empty[i], 1);
        }
        mbar_init(&sb.s_full, 1);
        mbar_init(&sb.dp_full, 1);
        mbar_init(&sb.epi_sync, 128);
        for (int g = 0; g < 2; ++g) {
            mbar_init(&sb.pa_done[g], 4);
            mbar_init(&sb.pb_done[g], 4);
        }
        sb.abort = 0;
        fence_mbar_init();
    }
    if (warp == 12 && lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
        tma_prefetch_map(&tm_do);
        tma_prefetch_map(&tm_qt);
        tma_prefetch_map(&tm_dot);
    }
    if (warp == 13) {
        tmem_alloc(&sb.tmem_base, Lay::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sb.tmem_base;
    volatile int *abort = &sb.abort;
    const int64_t B = p.block, W = p.window;
    const int64_t T = p.total_tokens;
    const int32_t ntiles = live_tile_count(p);

    if (warp == 12) {
        // ------------------------------------------------ TMA producer ---
        uint32_t it = 0, item_cnt = 0;
        TileRef r;
        bool ok = true;
        StaticItems items(p.tile_info, ntiles, p.heads, p.other_offsets);
        for (; ok && items.advance(r, sb.ring, abort, ok); ++item_cnt) {
            int ilo, ihi;
            query_tile_range<kCross>(r, B, W, ilo, ihi);
            for (int i = ilo; i <= ihi; ++i, ++it) {
                const int qs = it % QS, os = it % OS;
                if (!mbar_wait(&sb.q_empty[qs], ((it / QS) & 1) ^ 1, abort)) {
                    ok = false;
                    break;
                }
                // the example's last query tile, when partial, comes from the staged copy whose
                // rows past the example are zeros (Q here, dO below): dK += dS^T Q and
                // dV += P^T dO multiply those rows by zeros, which must not meet a neighbour's
                // Inf or NaN
                const bool part = r.oL - i * kTile < kTile; // query rows: the example's own, or its query set
                const CUtensorMap *mq = part ? &tm_qt : &tm_q, *mo = part ? &tm_dot : &tm_do;
                const int32_t qy = part ? r.b * kTile : r.os0 + i * kTile;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sb.q_full[qs], Lay::kTileBytes);
                    for (int c = 0; c < Lay::kChunks; ++c)
                        tma_load_2d(smem + Lay::kQ0 + qs * Lay::kTileBytes + c * Lay::kChunkBytes, mq,
                                    &sb.q_full[qs], r.h * D + c * 64, qy);
                }
                // the tile's -lse (log2 units) and -Delta, four queries per lane, copied
                // asynchronously; each lane's copies arrive on q_full when they land. Rows past
                // the example's end copy its last row (those queries are masked out).
                if constexpr (A == kSoftmax) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int qr = 4 * lane + e;
                        const int64_t q = int64_t(i) * kTile + qr;
                        const int64_t gi = int64_t(r.h) * T + r.s0 + (q < r.L ? q : r.L - 1);
                        cp_async_4(&sb.stat[qs][0][qr], nlse2 + gi);
                        cp_async_4(&sb.stat[qs][1][qr], neg_delta + gi);
                    }
                    cp_async_arrive_noinc(&sb.q_full[qs]);
                } else {
                    mbar_arrive(&sb.q_full[qs]); // generalized attention has no per-query statistics
                }
                __syncwarp();
                if (i == ilo) {
                    // the item's K and V, once the previous item's last S^T (K) and dP^T (V)
                    // are done; the first Q tile went out first, since its slot frees earlier
                    if (!mbar_wait(&sb.k_empty, (item_cnt & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    const CUtensorMap *mk = &tm_k;
                    int32_t ky = r.s0 + r.t * kTile;
                    if constexpr (kDq) {
                        // dQ sums over the key rows: an example's partial key tile comes from its
                        // zero-padded copy
                        if (r.L - r.t * kTile < kTile) {
                            mk = &tm_kt;
                            ky = r.b * kTile;
                        }
                    }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&sb.k_full, Lay::kTileBytes);
                        for (int c = 0; c < Lay::kChunks; ++c)
                            tma_load_2d(smem + Lay::kK + c * Lay::kChunkBytes, mk, &sb.k_full, r.h * D + c * 64, ky);
                    }
                    __syncwarp();
                    if (!mbar_wait(&sb.v_empty, (item_cnt & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&sb.v_full, Lay::kTileBytes);
                        for (int c = 0; c < Lay::kChunks; ++c)
                            tma_load_2d(smem + Lay::kV + c * Lay::kChunkBytes, &tm_v, &sb.v_full, r.h * D + c * 64,
                                        r.s0 + r.t * kTile);
                    }
                    __syncwarp();
                }
                if (!mbar_wait(&sb.o_empty[os], ((it / OS) & 1) ^ 1, abort)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sb.o_full[os], Lay::kTileBytes);
                    for (int c = 0; c < Lay::kChunks; ++c)
                        tma_load_2d(smem + Lay::kO0 + os * Lay::kTileBytes + c * Lay::kChunkBytes, mo,
                                    &sb.o_full[os], r.h * D + c * 64, qy);
                    // warm L2 two query tiles ahead, and with the next item's K, V and first tiles
                    if (i + 2 <= ihi)
                        for (int c = 0; c < Lay::kChunks; ++c) {
                            tma_prefetch_l2_2d(&tm_q, r.h * D + c * 64, r.os0 + (i + 2) * kTile);
                            tma_prefetch_l2_2d(&tm_do, r.h * D + c * 64, r.os0 + (i + 2) * kTile);
                        }
                    TileRef rn;
                    if (i == ilo && items.peek(rn)) {
                        int nlo, nhi;
                        query_tile_range<kCross>(rn, B, W, nlo, nhi);
                        for (int c = 0; c < Lay::kChunks; ++c) {
                            tma_prefetch_l2_2d(&tm_k, rn.h * D + c * 64, rn.s0 + rn.t * kTile);
                            tma_prefetch_l2_2d(&tm_v, rn.h * D + c * 64, rn.s0 + rn.t * kTile);
                            for (int i2 = nlo; i2 <= nhi && i2 < nlo + 2; ++i2) {
                                tma_prefetch_l2_2d(&tm_q, rn.h * D + c * 64, rn.os0 + i2 * kTile);
                                tma_prefetch_l2_2d(&tm_do, rn.h * D + c * 64, rn.os0 + i2 * kTile);
                            }
                        }
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == 13) {
        // -------------------------------------------------- MMA issuer ---
        constexpr uint32_t idesc_sp = idesc_bf16(128, 128, false, false); // S^T, dP^T
        constexpr uint32_t idesc_kv = idesc_bf16(128, D, false, true);    // dV, dK (B MN-major)
        uint32_t it0 = 0, item_cnt = 0;
        TileRef r;
        bool ok = true;
        const uint32_t k_addr = smem_base + Lay::kK, v_addr = smem_base + Lay::kV;
        StaticItems items(p.tile_info, ntiles, p.heads, p.other_offsets);
        for (; ok && items.advance(r, sb.ring, abort, ok); ++item_cnt) {
            int ilo, ihi;
            query_tile_range<kCross>(r, B, W, ilo, ihi);
            const int nq = ihi - ilo + 1;
            // S^T = K Q^T of query tile m of this item; after the item's last one K is not read again
            auto issue_s = [&](int m) -> bool {
                const uint32_t it = it0 + m, qs = it % QS;
                if (!mbar_wait(&sb.q_full[qs], (it / QS) & 1, abort)) return false;
                tc_fence_after();
                {
                    const uint32_t q_addr = smem_base + Lay::kQ0 + qs * Lay::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32;
                        mma_ss(tmem + Lay::kColS, sdesc_sw128(k_addr + off, 16, 1024),
                               sdesc_sw128(q_addr + off, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&sb.s_full);
                    if (!kDq && m == nq - 1) tc_commit(&sb.k_empty); // the fused backward reads K again for dQ
                }
                __syncwarp();
                return true;
            };
            // dP^T = V dO^T of query tile m; after the item's last one V is not read again
            auto issue_dp = [&](int m) -> bool {
                const uint32_t it = it0 + m, os = it % OS;
                if (!mbar_wait(&sb.o_full[os], (it / OS) & 1, abort)) return false;
                if constexpr (kDq) {
                    // dP^T overwrites the previous item's dQ: the epilogue must have read it
                    if (m == 0 && !mbar_wait(&sb.dq_free, (item_cnt & 1) ^ 1, abort)) return false;
                }
                tc_fence_after();
                {
                    const uint32_t o_addr = smem_base + Lay::kO0 + os * Lay::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32;
                        mma_ss(tmem + Lay::kColDP, sdesc_sw128(v_addr + off, 16, 1024),
                               sdesc_sw128(o_addr + off, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&sb.dp_full);
                    if (m == nq - 1) tc_commit(&sb.v_empty);
                }
                __syncwarp();
                return true;
            };
            // dV += P^T dO (phase == 0) or dK += dS^T Q (phase == 1) of query tile m,
            // group by group as the compute warps finish; then release the operand's slot
            auto issue_acc = [&](int m, int phase) -> bool {
                const uint32_t it = it0 + m;
                const uint32_t slot = phase == 0 ? it % OS : it % QS;
                const uint32_t b_addr = smem_base + (phase == 0 ? Lay::kO0 + slot * Lay::kTileBytes
                                                                : Lay::kQ0 + slot * Lay::kTileBytes);
                for (int g = 0; g < 2; ++g) {
                    if (!mbar_wait(phase == 0 ? &sb.pa_done[g] : &sb.pb_done[g], it & 1, abort)) return false;
                    // the first product of an item overwrites the accumulator: the epilogue
                    // must have read the previous item's (dV and dK are released separately)
                    if (m == 0 && g == 0 &&
                        !mbar_wait(phase == 0 ? &sb.dv_free : &sb.dk_free, (item_cnt & 1) ^ 1, abort))
                        return false;
                    tc_fence_after();
                    {
                        const uint32_t acol = tmem + (phase == 0 ? Lay::kColS : Lay::kColDP) + 64 * g;
                        const uint32_t dcol = tmem + (phase == 0 ? Lay::kColDV : Lay::kColDK);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) // queries 64g + 16kk .. of the tile
                            mma_ts(dcol, acol + 8 * kk,
                                   sdesc_sw128(b_addr + (4 * g + kk) * 2048, Lay::kChunkBytes, 1024), idesc_kv,
                                   (m > 0 || g > 0 || kk > 0) ? 1u : 0u);
                        if (g == 1) tc_commit(phase == 0 ? &sb.o_empty[slot] : &sb.q_empty[slot]);
                    }
                    __syncwarp();
                }
                return true;
            };
            ok = mbar_wait(&sb.k_full, item_cnt & 1, abort);
            if (ok) tc_fence_after();
            ok = ok && issue_s(0) && mbar_wait(&sb.v_full, item_cnt & 1, abort);
            if (ok) tc_fence_after();
            ok = ok && issue_dp(0);
            for (int m = 0; ok && m < nq; ++m) {
                ok = issue_acc(m, 0) && (m + 1 >= nq || issue_s(m + 1)) && issue_acc(m, 1) &&
                     (m + 1 >= nq || issue_dp(m + 1));
            }
            if (!ok) break;
            if constexpr (kDq) {
                // dQ = dS K (scaled in the epilogue). A = dS from shared memory, written by the
                // compute warps before their phase-B arrivals (waited for in issue_acc), MN-major
                // with 16 keys (2 KB of rows) per step; B = K, MN-major. It accumulates over the
                // dS^T columns, which the dK product issued before it has read.
                constexpr uint32_t idesc_q = idesc_bf16(128, D, true, true);
                const uint32_t ds_addr = smem_base + Lay::kDS;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    mma_ss(tmem + Lay::kColDQ, sdesc_sw128(ds_addr + kk * 2048, Lay::kDSChunkBytes, 1024),
                           sdesc_sw128(k_addr + kk * 2048, Lay::kChunkBytes, 1024), idesc_q, kk > 0 ? 1u : 0u);
                tc_commit(&sb.k_empty);
            }
            tc_commit(&sb.dkv_full);
            __syncwarp();
            it0 += nq;
        }
    } else if (warp < 8) {
        // ----------------------------------------------------- compute ---
        const int g = warp >> 2;              // column group: queries [64g, 64g+64)
        const int row = threadIdx.x & 127;    // key row within the tile, TMEM lane
        const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
        const float scale_log2 = p.scale * 1.4426950408889634f;
        uint32_t it = 0;
        TileRef r;
        bool ok = true;
        StaticItems items(p.tile_info, ntiles, p.heads, p.other_offsets);
        while (ok && items.advance(r, sb.ring, abort, ok)) {
            int ilo, ihi;
            query_tile_range<kCross>(r, B, W, ilo, ihi);
            const int64_t k = int64_t(r.t) * kTile + row; // local key index
            const bool valid_k = k < r.L;
            // visible queries [qmin, qmax]: the block rule, or (cross-attention) the whole query set
            const int64_t qmax = valid_k ? (kCross ? int64_t(r.oL) - 1 : last_query_seeing(k, r.L, B, W)) : -1;
            const int64_t qmin = kCross ? 0 : k;
            for (int i = ilo; i <= ihi && ok; ++i, ++it) {
                const int qs = it % QS;
                const int64_t q0 = int64_t(i) * kTile + 64 * g;
                int64_t lo64 = qmin - q0, hi64 = qmax - q0;
                if (!valid_k) { lo64 = 1; hi64 = 0; }
                const int lo_c = int(lo64 < -1 ? -1 : (lo64 > 64 ? 64 : lo64));
                const int hi_c = int(hi64 < -1 ? -1 : (hi64 > 64 ? 64 : hi64));
                const bool full = __all_sync(0xffffffffu, lo_c <= 0 && hi_c >= 63);
                uint32_t vis[2] = {0u, 0u}; // visible columns [lo_c, hi_c] of the group's 64, as bits
                if (!full) {
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        const int lo = max(lo_c - 32 * w, 0), hi = min(hi_c - 32 * w, 31);
                        vis[w] = lo <= hi ? (0xffffffffu >> (31 - hi)) & (0xffffffffu << lo) : 0u;
                    }
                }
                // -lse (log2 units) and -Delta of this group's queries, staged with the Q tile
                // (complete once S^T is: the S^T product waited for the same barrier phase)
                if (!mbar_wait(&sb.q_full[qs], (it / QS) & 1, abort)) { ok = false; break; }
                const float4 *l2v = reinterpret_cast<const float4 *>(sb.stat[qs][0] + 64 * g);
                const float2 *dlv2 = reinterpret_cast<const float2 *>(sb.stat[qs][1] + 64 * g);
                // phase A: P^T from S^T, written (bf16) over the group's first 32 S^T columns
                if (!mbar_wait(&sb.s_full, it & 1, abort)) { ok = false; break; }
                tc_fence_after();
                // P^T of the group's 64 queries as bf16 pairs: the dV product reads the same
                // rounded values from TMEM, and phase B forms dS from them
                uint32_t pp[4][8];
                const float2 sc2 = make_float2(scale_log2, scale_log2);
                uint32_t sr[2][16];
                tmem_ld16(tmem + lane_base + Lay::kColS + 64 * g, sr[0]);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    // 16 queries at a time, the next 16 in flight; their P^T lands in 8
                    // columns this thread has already read
                    uint32_t(&cur)[16] = sr[q4 & 1];
                    reg_fence(cur);
                    if (q4 < 3) tmem_ld16(tmem + lane_base + Lay::kColS + 64 * g + 16 * (q4 + 1), sr[(q4 + 1) & 1]);
                    if constexpr (A == kSoftmax) {
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            const float4 l4 = l2v[4 * q4 + c4]; // -lse of 4 queries
                            const float2 x01 = ffma2(make_float2(__uint_as_float(cur[4 * c4]), __uint_as_float(cur[4 * c4 + 1])),
                                                     sc2, make_float2(l4.x, l4.y));
                            const float2 x23 = ffma2(make_float2(__uint_as_float(cur[4 * c4 + 2]), __uint_as_float(cur[4 * c4 + 3])),
                                                     sc2, make_float2(l4.z, l4.w));
                            // all on MUFU: these warps are bound by instruction issue (measured)
                            float ev[4] = {ex2_approx(x01.x), ex2_approx(x01.y), ex2_approx(x23.x), ex2_approx(x23.y)};
                            if (!full) {
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int cc = 16 * q4 + 4 * c4 + e;
                                    ev[e] = (vis[cc / 32] & (1u << (cc % 32))) ? ev[e] : 0.f;
                                }
                            }
                            pp[q4][2 * c4] = pack_bf16x2(ev[0], ev[1]);
                            pp[q4][2 * c4 + 1] = pack_bf16x2(ev[2], ev[3]);
                        }
                        tmem_st8(tmem + lane_base + Lay::kColS + 64 * g + 8 * q4, pp[q4]);
                    } else {
                        // generalized attention: act(S^T / sqrt(D)) goes to TMEM for dV; act' stays
                        // in registers for dS^T = act' dP^T (Delta is 0)
                        uint32_t pa[8];
#pragma unroll
                        for (int c2 = 0; c2 < 8; ++c2) {
                            float2 v0 = act_value_grad<A>(__uint_as_float(cur[2 * c2]) * p.scale);
                            float2 v1 = act_value_grad<A>(__uint_as_float(cur[2 * c2 + 1]) * p.scale);
                            if (!full) {
                                const int cc = 16 * q4 + 2 * c2;
                                if (!(vis[cc / 32] & (1u << (cc % 32)))) v0 = make_float2(0.f, 0.f);
                                if (!(vis[cc / 32] & (1u << (cc % 32 + 1)))) v1 = make_float2(0.f, 0.f);
                            }
                            pa[c2] = pack_bf16x2(v0.x, v1.x);
                            pp[q4][c2] = pack_bf16x2(v0.y, v1.y);
                        }
                        tmem_st8(tmem + lane_base + Lay::kColS + 64 * g + 8 * q4, pa);
                    }
                    if (q4 < 3) tmem_wait_ld();
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.pa_done[g]);
                // phase B: dS^T = P^T (dP^T - Delta), written (bf16) over the group's first 32 dP^T columns
                if (!mbar_wait(&sb.dp_full, it & 1, abort)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    // 32 queries at a time; their dS^T lands in 16 columns this thread has read
                    uint32_t dr[32];
                    tmem_ld32(tmem + lane_base + Lay::kColDP + 64 * g + 32 * h2, dr);
                    tmem_wait_ld();
                    reg_fence(dr);
                    uint32_t dk16[16];
#pragma unroll
                    for (int c2 = 0; c2 < 16; ++c2) {
                        const float2 d2 = A == kSoftmax ? dlv2[16 * h2 + c2] : make_float2(0.f, 0.f); // -Delta
                        const uint32_t pw = pp[2 * h2 + c2 / 8][c2 % 8];
                        const float2 p2 = make_float2(__uint_as_float(pw << 16), __uint_as_float(pw & 0xffff0000u));
                        const float2 ds = fmul2(p2, fadd2(make_float2(__uint_as_float(dr[2 * c2]),
                                                                      __uint_as_float(dr[2 * c2 + 1])), d2));
                        dk16[c2] = pack_bf16x2(ds.x, ds.y);
                    }
                    tmem_st16(tmem + lane_base + Lay::kColDP + 64 * g + 16 * h2, dk16);
                    if constexpr (kDq) {
                        // the same dS for dQ = dS K: row `row` (this key) of query chunk g, 16-byte
                        // units 4 h2 .. 4 h2 + 3; zero for a key past the example, whose dP^T row
                        // may hold a neighbour's non-finite values
                        uint8_t *drow = smem + Lay::kDS + g * Lay::kDSChunkBytes + row * 128;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4 *>(drow + (((4 * h2 + j) ^ (row & 7)) << 4)) =
                                valid_k ? make_uint4(dk16[4 * j], dk16[4 * j + 1], dk16[4 * j + 2], dk16[4 * j + 3])
                                        : make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                if constexpr (kDq) fence_proxy_async_smem(); // dS written for the tensor core
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.pb_done[g]);
            }
        }
    } else if (warp < 12) {
        // ---------------------------------------------------- epilogue ---
        // A full tile leaves through a 128-row x 64-column shared staging buffer and
        // TMA stores, so the rows are written as whole lines; the last tile of an
        // example (rows past its end belong to the next example) is stored row by row.
        const int row = threadIdx.x & 127;    // key row within the tile, TMEM lane
        const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
        const bool leader = threadIdx.x == 256;
        uint8_t *stage = smem + Lay::kStage;
        uint32_t item_cnt = 0, sync_phase = 0;
        bool ok = true;
        TileRef r;
        StaticItems items(p.tile_info, ntiles, p.heads, p.other_offsets);
        for (; ok && items.advance(r, sb.ring, abort, ok); ++item_cnt) {
            const int64_t k = int64_t(r.t) * kTile + row;
            const bool valid_k = k < r.L;
            const bool full_tile = int64_t(r.t) * kTile + kTile <= r.L;
            const int64_t grow = (int64_t(r.s0) + k) * p.heads + r.h;
            if (!mbar_wait(&sb.dkv_full, item_cnt & 1, abort)) break;
            tc_fence_after();
            if constexpr (kDq) {
                // dQ first (the tile's query rows are its key rows), 64 columns at a time, scaled
                // by 1/sqrt(D): reading it frees the columns the next item's dP^T writes
#pragma unroll 1
                for (int c = 0; c < Lay::kChunks; ++c) {
                    uint32_t rr[2][32], pk[32];
                    tmem_ld32(tmem + lane_base + Lay::kColDQ + 64 * c, rr[0]);
                    tmem_ld32(tmem + lane_base + Lay::kColDQ + 64 * c + 32, rr[1]);
                    tmem_wait_ld();
                    reg_fence(rr[0]);
                    reg_fence(rr[1]);
                    if (c == Lay::kChunks - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sb.dq_free);
                    }
#pragma unroll
                    for (int x = 0; x < 32; ++x)
                        pk[x] = pack_bf16x2(__uint_as_float(rr[x / 16][2 * (x % 16)]) * p.scale,
                                            __uint_as_float(rr[x / 16][2 * (x % 16) + 1]) * p.scale);
                    if (full_tile) {
                        if (leader) bulk_wait_group_read<0>();
                        if (!group_sync(&sb.epi_sync, sync_phase, abort)) { ok = false; break; }
                        uint8_t *srow = stage + row * 128;
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *reinterpret_cast<uint4 *>(srow + ((u ^ (row & 7)) << 4)) =
                                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                        fence_proxy_async_smem();
                        if (!group_sync(&sb.epi_sync, sync_phase, abort)) { ok = false; break; }
                        if (leader) {
                            tma_store_2d(&tm_dq, stage, r.h * D + 64 * c, r.s0 + r.t * kTile);
                            bulk_commit_group();
                        }
                    } else if (valid_k) {
                        uint4 *dst = reinterpret_cast<uint4 *>(dq + grow * D + 64 * c);
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                    }
                }
                if (!ok) break;
            }
            // 64 columns at a time: dV chunks, then dK chunks (scaled by 1/sqrt(D))
#pragma unroll 1
            for (int part = 0; part < 2 * Lay::kChunks; ++part) {
                const bool is_k = part >= Lay::kChunks;
                const int c = is_k ? part - Lay::kChunks : part;
                const float sc = is_k ? p.scale : 1.f;
                auto release = [&] {
                    if (c == Lay::kChunks - 1) { // all of dV (or dK) read: the next item may accumulate into it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(is_k ? &sb.dk_free : &sb.dv_free);
                    }
                };
                uint32_t pk[32];
                if (kRope && is_k) {
                    // rotary embedding: dK is the gradient of the rotated k; turn its pairs back
                    // (transposed rotation at this key row's position). One 32-column half at a
                    // time, read, turned and packed before the next, to stay within registers.
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t rh[32];
                        tmem_ld32(tmem + lane_base + Lay::kColDK + 64 * c + 32 * hh, rh);
                        tmem_wait_ld();
                        reg_fence(rh);
                        if (valid_k) rope_transpose_bits<4>(p, k, 32 * c + 16 * hh, rh);
#pragma unroll
                        for (int x = 0; x < 16; ++x)
                            pk[16 * hh + x] =
                                pack_bf16x2(__uint_as_float(rh[2 * x]) * sc, __uint_as_float(rh[2 * x + 1]) * sc);
                    }
                    release();
                } else {
                    uint32_t rr[2][32];
                    tmem_ld32(tmem + lane_base + (is_k ? Lay::kColDK : Lay::kColDV) + 64 * c, rr[0]);
                    tmem_ld32(tmem + lane_base + (is_k ? Lay::kColDK : Lay::kColDV) + 64 * c + 32, rr[1]);
                    tmem_wait_ld();
                    reg_fence(rr[0]);
                    reg_fence(rr[1]);
                    release();
#pragma unroll
                    for (int x = 0; x < 32; ++x)
                        pk[x] = pack_bf16x2(__uint_as_float(rr[x / 16][2 * (x % 16)]) * sc,
                                            __uint_as_float(rr[x / 16][2 * (x % 16) + 1]) * sc);
                }
                if (full_tile) {
                    if (leader) bulk_wait_group_read<0>(); // the previous store has left the buffer
                    if (!group_sync(&sb.epi_sync, sync_phase, abort)) { ok = false; break; }
                    uint8_t *srow = stage + row * 128;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        *reinterpret_cast<uint4 *>(srow + ((u ^ (row & 7)) << 4)) =
                            make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                    fence_proxy_async_smem();
                    if (!group_sync(&sb.epi_sync, sync_phase, abort)) { ok = false; break; }
                    if (leader) {
                        tma_store_2d(is_k ? &tm_dk : &tm_dv, stage, r.h * D + 64 * c, r.s0 + r.t * kTile);
                        bulk_commit_group();
                    }
                } else if (valid_k) {
                    uint4 *dst = reinterpret_cast<uint4 *>((is_k ? dk : dv) + grow * D + 64 * c);
#pragma unroll
                    for (int u = 0; u < 8; ++u) dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                }
            }
        }
        if (leader) bulk_wait_group<0>();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 13) tmem_dealloc(tmem, Lay::kTmemCols);
    if (threadIdx.x == 0 && sb.abort) atomicOr(p.status, kStatusTimeout);
}

template <int D, int A>
cudaError_t launch_bwd_dkdv_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const CUtensorMap &tdo, const CUtensorMap &tdk, const CUtensorMap &tdv,
                                  const CUtensorMap &tqt, const CUtensorMap &tdot, const Problem &p,
                                  const float *nlse2, const float *neg_delta, void *dk, void *dv, int num_sms,
                                  cudaStream_t stream)
{
    using Lay = DkvLayout<D>;
    // the rotary epilogue exists for block attention only, cross-attention for the generalized one
    auto kern = (A == kSoftmax && p.rope_cos)        ? bwd_dkdv_sm100_kernel<D, A == kSoftmax, A, false, false>
                : (A != kSoftmax && p.other_offsets) ? bwd_dkdv_sm100_kernel<D, false, A, A != kSoftmax, false>
                                                     : bwd_dkdv_sm100_kernel<D, false, A, false, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess) return e;
    // the last three arguments belong to the fused backward; valid maps stand in, unread
    kern<<<num_sms, Lay::kThreads, Lay::kAlloc, stream>>>(tq, tk, tv, tdo, tdk, tdv, tqt, tdot, p, nlse2, neg_delta,
                                                          static_cast<__nv_bfloat16 *>(dk),
                                                          static_cast<__nv_bfloat16 *>(dv), tk, tdk, nullptr);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_fused_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                   const CUtensorMap &tdo, const CUtensorMap &tdk, const CUtensorMap &tdv,
                                   const CUtensorMap &tqt, const CUtensorMap &tdot, const CUtensorMap &tkt,
                                   const CUtensorMap &tdq, const Problem &p, const float *nlse2,
                                   const float *neg_delta, void *dq, void *dk, void *dv, int num_sms,
                                   cudaStream_t stream)
{
    using Lay = DkvLayout<D, true>;
    auto kern = bwd_dkdv_sm100_kernel<D, false, kSoftmax, false, true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess) return e;
    kern<<<num_sms, Lay::kThreads, Lay::kAlloc, stream>>>(tq, tk, tv, tdo, tdk, tdv, tqt, tdot, p, nlse2, neg_delta,
                                                          static_cast<__nv_bfloat16 *>(dk),
                                                          static_cast<__nv_bfloat16 *>(dv), tkt, tdq,
                                                          static_cast<__nv_bfloat16 *>(dq));
    return cudaGetLastError();
}
template cudaError_t launch_bwd_fused_sm100<64>(const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                                                const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                                                const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                                                const CUtensorMap &, const Problem &, const float *, const float *,
                                                void *, void *, void *, int, cudaStream_t);
template cudaError_t launch_bwd_fused_sm100<128>(const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                                                 const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                                                 const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                                                 const CUtensorMap &, const Problem &, const float *, const float *,
                                                 void *, void *, void *, int, cudaStream_t);

#define BA_DKDV_INST(D, A)                                                                                   \
    template cudaError_t launch_bwd_dkdv_sm100<D, A>(const CUtensorMap &, const CUtensorMap &,                \
                                                     const CUtensorMap &, const CUtensorMap &, const CUtensorMap &, \
                                                     const CUtensorMap &, const CUtensorMap &, const CUtensorMap &, \
                                                     const Problem &, const float *,                            \
                                                     const float *, void *, void *, int, cudaStream_t);
BA_DKDV_INST(64, kSoftmax)
BA_DKDV_INST(128, kSoftmax)
BA_DKDV_INST(64, kGelu)
BA_DKDV_INST(128, kGelu)
BA_DKDV_INST(64, kSilu)
BA_DKDV_INST(128, kSilu)

} // namespace ba
