// Block attention backward, dQ pass (query-tile stationary), sm_100a.
//
// For one 128-query tile of one (example, head) this kernel recomputes the
// probabilities of every visible key tile from the forward's lse and forms
//   dS = P o (dO V^T - Delta),   dQ = (1/sqrt(D)) sum_j dS_j K_j,
// with Delta_i = dO_i . out_i computed here (and written out for the dK/dV
// pass). dQ is accumulated on chip and written once, in the input dtype: no
// atomics and no fp32 accumulator in global memory. The dK/dV pass
// (ba_bwd_dkdv_sm100.cu) recomputes P and dS per key tile; the two passes
// together are the exact gradient of the block attention forward ("GEM
// (Meta)", section "Custom kernels": the BlockAttention kernel trains, so it
// has a backward; the pages give no formulas).
//
// Tensor-core plan per key tile j (all tcgen05, fp32 accumulators in TMEM):
//   S  = Q K_j^T   A = Q from TMEM (copied there once per item), B = K_j smem
//   dP = dO V_j^T  A = dO from TMEM, B = V_j smem
//   dQ += dS K_j   A = dS from TMEM (bf16), B = K_j smem (MN-major)
// Keeping Q and dO in TMEM means every MMA streams only its B operand from
// shared memory, which keeps the tensor core ahead of shared-memory bandwidth.
//
// CTA roles (persistent, round-robin over (query tile, head) items):
//   warps 0-3 / 4-7  two compute warpgroups; thread t owns query row t (TMEM
//              lane t), group g the keys [64g, 64g+64) of each key tile.
//              Per item they copy Q (group 0) and dO (group 1) from the
//              staging tiles into TMEM and compute Delta; per key tile they
//              read S (then release it so the next S can be issued), form P,
//              read dP, form dS and write it as bf16 over their dP columns;
//              at the end they store dq.
//   warp 8     TMA producer: Q, dO, out tiles of the item into staging; K, V
//              per key tile into a ring.
//   warp 9     MMA issuer.
// TMEM columns: Q [0, D/2), dO [D/2, D), S [D, D+128), dP [D+128, D+256)
// (dS bf16 of group g over [D+128+64g, D+160+64g)), dQ [D+256, 2D+256).
#include "ba_common.cuh"
#include "ba_kernels.cuh"
#include "ba_ptx.cuh"
#include "ba_sched.cuh"

#include <cuda_bf16.h>

namespace ba {

namespace {

template <int D>
struct DqLayout {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr int kChunks = D / 64;              // 128-byte column chunks per row
    static constexpr int kChunkBytes = kTile * 128;     // one chunk of a 128-row tile
    static constexpr int kTileBytes = kTile * D * 2;
    static constexpr int kStages = D == 64 ? 3 : 2;     // K/V ring
    static constexpr int kKV0 = 0;                      // stage s: K at kKV0 + 2 s tile, V after it
    static constexpr int kStaging = 2 * kStages * kTileBytes; // Q, dO, out tiles of the next item
    static constexpr int kBytes = kStaging + 3 * kTileBytes;
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr int kThreads = 384;                 // three warpgroups
    // register budgets after the split; 2 * 128 * 216 + 128 * 72 = 384 * 168
    static constexpr uint32_t kRegsCompute = 216, kRegsOther = 72;
    static constexpr uint32_t kColQ = 0, kColDO = D / 2, kColS = D, kColDP = D + 128, kColDQ = D + 256;
    static constexpr uint32_t kTmemCols = 512;
};

struct DqBarriers {
    uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
    uint64_t st_full, st_empty, qt_ready;
    uint64_t s_full, s_free, dp_full, ds_full[2], dq_done, dq_free;
    uint64_t tail; // the TMA warp's own barrier for a K or V tile whose last rows it clears
    ItemRing ring; // items claimed by the TMA warp, read by the MMA and compute warps
    uint32_t tmem_base;
    int abort;
};

// Key-tile range [jlo, t] of query tile t.
__device__ __forceinline__ int first_key_tile(const TileRef &r, int64_t B, int64_t W)
{
    return int(window_start(int64_t(r.t) * kTile, B, W) / kTile);
}

} // namespace

template <int D, bool kRope, int A, bool kCross>
__global__ void __launch_bounds__(384, 1)
    bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_o, const Problem p, const float *__restrict__ lse,
                        float *__restrict__ neg_delta, float *__restrict__ nlse2, __nv_bfloat16 *__restrict__ dq)
{
    using Lay = DqLayout<D>;
    constexpr int S = Lay::kStages;
    extern __shared__ uint8_t smem_raw[];
    __shared__ DqBarriers sb;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&sb.k_full[i], 1);
            mbar_init(&sb.k_empty[i], 1);
            mbar_init(&sb.v_full[i], 1);
            mbar_init(&sb.v_empty[i], 1);
        }
        mbar_init(&sb.st_full, 1);
        mbar_init(&sb.st_empty, 8);
        mbar_init(&sb.qt_ready, 8);
        mbar_init(&sb.s_full, 1);
        mbar_init(&sb.s_free, 8);
        mbar_init(&sb.dp_full, 1);
        mbar_init(&sb.ds_full[0], 4);
        mbar_init(&sb.ds_full[1], 4);
        mbar_init(&sb.dq_done, 1);
        mbar_init(&sb.dq_free, 8);
        mbar_init(&sb.tail, 1);
        item_ring_init(sb.ring, 1 + 8); // MMA warp, compute warps
        sb.abort = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
        tma_prefetch_map(&tm_do);
        tma_prefetch_map(&tm_o);
    }
    if (warp == 9) {
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

    if (warp >= 8) {
        // warps 8-11 (one warpgroup: TMA, MMA, two idle) hand registers to the compute warpgroups
        warpgroup_regs_dec<Lay::kRegsOther>();
        if (warp == 8) {
            // ------------------------------------------------ TMA producer ---
            uint32_t kv_cnt = 0, item_cnt = 0, tail_phase = 0;
            TileRef r;
            bool ok = true;
            ItemSource items(p.tile_info, ntiles, p.heads, p.status + kCounterDq, p.other_offsets);
            for (; ok && items.advance(r, sb.ring, abort, ok); ++item_cnt) {
                // key tiles [jlo, jend]: the block rule, or (cross-attention) the example's whole key/value set
                const int jlo = kCross ? 0 : first_key_tile(r, B, W);
                const int jend = kCross ? (r.oL + kTile - 1) / kTile - 1 : r.t;
                if (!mbar_wait(&sb.st_empty, (item_cnt & 1) ^ 1, abort)) break;
                if (lane == 0) {
                    // Q, dO and (for Delta; the softmax only) out
                    uint8_t *st = smem + Lay::kStaging;
                    mbar_arrive_expect_tx(&sb.st_full, (A == kSoftmax ? 3 : 2) * Lay::kTileBytes);
                    for (int c = 0; c < Lay::kChunks; ++c) {
                        const int x = r.h * D + c * 64, y = r.s0 + r.t * kTile;
                        tma_load_2d(st + c * Lay::kChunkBytes, &tm_q, &sb.st_full, x, y);
                        tma_load_2d(st + Lay::kTileBytes + c * Lay::kChunkBytes, &tm_do, &sb.st_full, x, y);
                        if (A == kSoftmax)
                            tma_load_2d(st + 2 * Lay::kTileBytes + c * Lay::kChunkBytes, &tm_o, &sb.st_full, x, y);
                    }
                }
                __syncwarp();
                for (int j = jlo; j <= jend; ++j, ++kv_cnt) {
                    const int st = kv_cnt % S;
                    uint8_t *kdst = smem + Lay::kKV0 + 2 * st * Lay::kTileBytes;
                    // K is read until dQ, V only by dP: they are released and refilled separately
                    // the example's last K and V tiles: rows past the example are cleared, since
                    // dQ += dS K and the masked dS = P (dP - Delta) multiply them by zeros
                    const int valid = r.oL - j * kTile;
                    if (!mbar_wait(&sb.k_empty[st], ((kv_cnt / S) & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    if (valid >= kTile) {
                        if (lane == 0) {
                            mbar_arrive_expect_tx(&sb.k_full[st], Lay::kTileBytes);
                            for (int c = 0; c < Lay::kChunks; ++c)
                                tma_load_2d(kdst + c * Lay::kChunkBytes, &tm_k, &sb.k_full[st], r.h * D + c * 64,
                                            r.os0 + j * kTile);
                        }
                        __syncwarp();
                    } else {
                        if (!load_tail_tile(kdst, Lay::kChunks, &tm_k, &sb.k_full[st], &sb.tail, tail_phase, r.h * D,
                                            r.os0 + j * kTile, valid, abort)) {
                            ok = false;
                            break;
                        }
                        tail_phase ^= 1;
                    }
                    if (!mbar_wait(&sb.v_empty[st], ((kv_cnt / S) & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    if (valid >= kTile) {
                        if (lane == 0) {
                            mbar_arrive_expect_tx(&sb.v_full[st], Lay::kTileBytes);
                            for (int c = 0; c < Lay::kChunks; ++c)
                                tma_load_2d(kdst + Lay::kTileBytes + c * Lay::kChunkBytes, &tm_v, &sb.v_full[st],
                                            r.h * D + c * 64, r.os0 + j * kTile);
                        }
                        __syncwarp();
                    } else {
                        if (!load_tail_tile(kdst + Lay::kTileBytes, Lay::kChunks, &tm_v, &sb.v_full[st], &sb.tail,
                                            tail_phase, r.h * D, r.os0 + j * kTile, valid, abort)) {
                            ok = false;
                            break;
                        }
                        tail_phase ^= 1;
                    }
                }
            }
        } else if (warp == 9) {
            // -------------------------------------------------- MMA issuer ---
            constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false); // S, dP
            constexpr uint32_t idesc_q = idesc_bf16(128, D, false, true);    // dQ (B = K, MN-major)
            uint32_t kv_cnt = 0, s_cnt = 0, d_cnt = 0, item_cnt = 0;
            TileRef r;
            bool ok = true;
            // dQ += dS K for the key tile in ring stage `st` (m = its index in the item)
            auto issue_dq = [&](int m, int st) -> bool {
                if (!mbar_wait(&sb.ds_full[0], d_cnt & 1, abort)) return false;
                if (m == 0 && !mbar_wait(&sb.dq_free, (item_cnt & 1) ^ 1, abort)) return false;
                tc_fence_after();
                const uint32_t k_addr = smem_base + Lay::kKV0 + 2 * st * Lay::kTileBytes;
                {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tmem + Lay::kColDQ, tmem + Lay::kColDP + kk * 8,
                               sdesc_sw128(k_addr + kk * 2048, Lay::kChunkBytes, 1024), idesc_q,
                               (m > 0 || kk > 0) ? 1u : 0u);
                }
                __syncwarp();
                if (!mbar_wait(&sb.ds_full[1], d_cnt & 1, abort)) return false;
                tc_fence_after();
                {
#pragma unroll
                    for (int kk = 4; kk < 8; ++kk)
                        mma_ts(tmem + Lay::kColDQ, tmem + Lay::kColDP + 64 + (kk - 4) * 8,
                               sdesc_sw128(k_addr + kk * 2048, Lay::kChunkBytes, 1024), idesc_q, 1u);
                    tc_commit(&sb.k_empty[st]);
                }
                __syncwarp();
                ++d_cnt;
                return true;
            };
            ItemSink items;
            for (; ok && items.advance(r, sb.ring, abort, ok); ++item_cnt) {
                const int jlo = kCross ? 0 : first_key_tile(r, B, W);
                const int nkv = kCross ? (r.oL + kTile - 1) / kTile : r.t - jlo + 1;
                if (!mbar_wait(&sb.qt_ready, item_cnt & 1, abort)) break;
                tc_fence_after();
                for (int m = 0; m < nkv; ++m, ++kv_cnt, ++s_cnt) {
                    const int st = kv_cnt % S;
                    if (!mbar_wait(&sb.k_full[st], (kv_cnt / S) & 1, abort) ||
                        !mbar_wait(&sb.s_free, (s_cnt & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t k_addr = smem_base + Lay::kKV0 + 2 * st * Lay::kTileBytes;
                    const uint32_t v_addr = k_addr + Lay::kTileBytes;
                    {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            mma_ts(tmem + Lay::kColS, tmem + Lay::kColQ + kk * 8,
                                   sdesc_sw128(k_addr + (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32, 16, 1024),
                                   idesc_s, kk > 0 ? 1u : 0u);
                        tc_commit(&sb.s_full);
                    }
                    __syncwarp();
                    // dQ of the previous key tile: it reads dS from the dP columns,
                    // so it must be issued before this tile's dP overwrites them.
                    if (m > 0 && !issue_dq(m - 1, (kv_cnt - 1) % S)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&sb.v_full[st], (kv_cnt / S) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            mma_ts(tmem + Lay::kColDP, tmem + Lay::kColDO + kk * 8,
                                   sdesc_sw128(v_addr + (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32, 16, 1024),
                                   idesc_s, kk > 0 ? 1u : 0u);
                        tc_commit(&sb.dp_full);
                        tc_commit(&sb.v_empty[st]); // V of this tile has no other reader
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (!issue_dq(nkv - 1, (kv_cnt - 1) % S)) break;
                tc_commit(&sb.dq_done);
                __syncwarp();
            }
        }
    } else {
        warpgroup_regs_inc<Lay::kRegsCompute>();
        // ----------------------------------------------------- compute ---
        const int g = warp >> 2;              // column group: keys [64g, 64g+64)
        const int row = threadIdx.x & 127;    // query row within the tile, TMEM lane
        const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
        const float scale_log2 = p.scale * 1.4426950408889634f;
        const uint8_t *staging = smem + Lay::kStaging;
        uint32_t s_cnt = 0, item_cnt = 0;
        bool ok = true;

        // Copy this item's Q (group 0) or dO (group 1) row into TMEM and
        // compute Delta from the staged dO and out rows.
        auto fill = [&](const TileRef &rr, uint32_t cnt, float &delta_row, float lse_val) -> bool {
            if (!mbar_wait(&sb.st_full, cnt & 1, abort)) return false;
            const uint8_t *qsrc = staging;
            const uint8_t *dsrc = staging + Lay::kTileBytes;
            const uint8_t *osrc = staging + 2 * Lay::kTileBytes;
            const uint32_t col0 = g == 0 ? Lay::kColQ : Lay::kColDO;
            float2 dl2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < Lay::kChunks; ++c) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t w[16];
#pragma unroll
                    for (int u4 = 0; u4 < 4; ++u4) {
                        // 16-byte unit u of this row's 128-byte chunk c (128B-swizzled staging tile)
                        const int u = 4 * hh + u4;
                        const int off = c * Lay::kChunkBytes + row * 128 + ((u ^ (row & 7)) * 16);
                        const uint4 d4 = *reinterpret_cast<const uint4 *>(dsrc + off);
                        if constexpr (A == kSoftmax) {
                            const uint4 o4 = *reinterpret_cast<const uint4 *>(osrc + off);
                            const uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w}, ow[4] = {o4.x, o4.y, o4.z, o4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 df =
                                    __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&dw[e]));
                                const float2 of =
                                    __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ow[e]));
                                dl2 = ffma2(df, of, dl2);
                            }
                        }
                        const uint4 a = g == 0 ? *reinterpret_cast<const uint4 *>(qsrc + off) : d4;
                        w[4 * u4] = a.x;
                        w[4 * u4 + 1] = a.y;
                        w[4 * u4 + 2] = a.z;
                        w[4 * u4 + 3] = a.w;
                    }
                    // two bf16 per TMEM column: 32 values fill 16 columns
                    tmem_st16(tmem + lane_base + col0 + 32 * c + 16 * hh, w);
                }
            }
            const float dl = dl2.x + dl2.y;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sb.st_empty);
                mbar_arrive(&sb.qt_ready);
            }
            delta_row = dl;
            const int64_t i = int64_t(rr.t) * kTile + row;
            // for the dK/dV pass: -Delta (group 0) and -lse in log2 units (group 1)
            if (A == kSoftmax && i < rr.L) {
                if (g == 0) neg_delta[int64_t(rr.h) * T + rr.s0 + i] = -dl;
                else nlse2[int64_t(rr.h) * T + rr.s0 + i] = -lse_val * 1.4426950408889634f;
            }
            return true;
        };

        TileRef r;
        ItemSink items;
        bool have = items.advance(r, sb.ring, abort, ok);
        float delta_row = 0.f;
        // lse of this thread's query row (log2 units), loaded an item ahead
        auto load_l2 = [&](const TileRef &rr) -> float {
            const int64_t q = int64_t(rr.t) * kTile + row;
            if (A != kSoftmax) return 0.f;
            return q < rr.L ? lse[int64_t(rr.h) * T + rr.s0 + q] : INFINITY;
        };
        float lse_row = have ? load_l2(r) : 0.f;
        if (have) ok = fill(r, 0, delta_row, lse_row);
        while (have && ok) {
            const int jlo = kCross ? 0 : first_key_tile(r, B, W);
            const int nkv = kCross ? (r.oL + kTile - 1) / kTile : r.t - jlo + 1;
            const int64_t i = int64_t(r.t) * kTile + row;
            const bool valid = i < r.L;
            // visible keys [ws, last]: the block rule, or (cross-attention) the whole key/value set
            const int64_t ws = kCross ? 0 : window_start(i, B, W);
            const int64_t last = kCross ? int64_t(r.oL) - 1 : i;
            const float l2 = lse_row * 1.4426950408889634f;
            const float dl = delta_row;
            for (int m = 0; m < nkv; ++m, ++s_cnt) {
                const int64_t key0 = int64_t(jlo + m) * kTile + 64 * g;
                int64_t lo64 = ws - key0, hi64 = last - key0;
                if (!valid) { lo64 = 1; hi64 = 0; }
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
                // phase A: P from S
                if (!mbar_wait(&sb.s_full, s_cnt & 1, abort)) { ok = false; break; }
                tc_fence_after();
                // P of this group's 64 keys, kept in float32: phase B only needs it to form dS, so
                // it is never packed (packing and unpacking cost three instructions a pair)
                float2 pf[4][8];
                const float2 sc2 = make_float2(scale_log2, scale_log2), nl2 = make_float2(-l2, -l2);
                {
                    uint32_t sr[2][16];
                    tmem_ld16(tmem + lane_base + Lay::kColS + 64 * g, sr[0]);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        // 16 keys at a time, the next 16 in flight
                        uint32_t(&cur)[16] = sr[q4 & 1];
                        reg_fence(cur);
                        if (q4 < 3) tmem_ld16(tmem + lane_base + Lay::kColS + 64 * g + 16 * (q4 + 1), sr[(q4 + 1) & 1]);
                        else {
                            // all of S read: the next tile's S may overwrite it
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&sb.s_free);
                        }
#pragma unroll
                        for (int c2 = 0; c2 < 8; ++c2) {
                            const float2 x = ffma2(make_float2(__uint_as_float(cur[2 * c2]), __uint_as_float(cur[2 * c2 + 1])),
                                                   sc2, nl2);
                            float e0, e1;
                            if constexpr (A == kSoftmax) {
                                // all on MUFU: these warps are bound by instruction issue, and the
                                // FMA-pipe 2^x costs nine instructions to MUFU's one (measured)
                                e0 = ex2_approx(x.x);
                                e1 = ex2_approx(x.y);
                            } else {
                                // generalized attention: dS = act'(S / sqrt(D)) dP (Delta is 0)
                                e0 = act_grad<A>(__uint_as_float(cur[2 * c2]) * p.scale);
                                e1 = act_grad<A>(__uint_as_float(cur[2 * c2 + 1]) * p.scale);
                            }
                            if (!full) {
                                const int cc = 16 * q4 + 2 * c2;
                                e0 = (vis[cc / 32] & (1u << (cc % 32))) ? e0 : 0.f;
                                e1 = (vis[cc / 32] & (1u << (cc % 32 + 1))) ? e1 : 0.f;
                            }
                            pf[q4][c2] = make_float2(e0, e1);
                        }
                        if (q4 < 3) tmem_wait_ld();
                    }
                }
                // phase B: dS = P (dP - Delta), written as bf16 over this group's dP columns
                if (!mbar_wait(&sb.dp_full, s_cnt & 1, abort)) { ok = false; break; }
                tc_fence_after();
                const float2 ndl = make_float2(-dl, -dl);
                // both 32-key halves of dP in one round trip (one TMEM wait, not two)
                uint32_t drr[2][32];
                tmem_ld32(tmem + lane_base + Lay::kColDP + 64 * g, drr[0]);
                tmem_ld32(tmem + lane_base + Lay::kColDP + 64 * g + 32, drr[1]);
                tmem_wait_ld();
                reg_fence(drr[0]);
                reg_fence(drr[1]);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    // 32 keys at a time; their dS (16 columns) lands in [64g+16h2, +16),
                    // inside the dP columns this thread has already read
                    uint32_t(&dr)[32] = drr[h2];
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float2 ds = fmul2(pf[2 * h2 + c / 8][c % 8], fadd2(make_float2(__uint_as_float(dr[2 * c]),
                                                                      __uint_as_float(dr[2 * c + 1])), ndl));
                        pk[c] = pack_bf16x2(ds.x, ds.y);
                    }
                    tmem_st16(tmem + lane_base + Lay::kColDP + 64 * g + 16 * h2, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.ds_full[g]);
            }
            if (!ok) break;
            // rotary embedding: this row's cos / sin for the epilogue, read now so that they
            // arrive while the next item's Q / dO go into TMEM
            constexpr int kRopeVec = kRope ? D / 16 : 1; // float4s of the group's D / 4 pairs
            float4 rcos[kRopeVec], rsin[kRopeVec];
            const bool rope_in = !kRope || !valid || i < p.rope_rows;
            if constexpr (kRope) {
                if (valid && rope_in) {
                    const float4 *cs = reinterpret_cast<const float4 *>(p.rope_cos + i * (D / 2) + (D / 4) * g);
                    const float4 *sn = reinterpret_cast<const float4 *>(p.rope_sin + i * (D / 2) + (D / 4) * g);
#pragma unroll
                    for (int u = 0; u < kRopeVec; ++u) {
                        rcos[u] = ld_nc_early(cs + u);
                        rsin[u] = ld_nc_early(sn + u);
                    }
                }
            }
            // the next item's Q / dO go into TMEM now: this item's last S and dP have completed
            TileRef rn;
            const bool have_next = items.advance(rn, sb.ring, abort, ok);
            if (!ok) break;
            float delta_next = 0.f;
            const float lse_next = have_next ? load_l2(rn) : 0.f;
            if (have_next && !fill(rn, item_cnt + 1, delta_next, lse_next)) break;
            // epilogue: dq of this item
            if (!mbar_wait(&sb.dq_done, item_cnt & 1, abort)) break;
            tc_fence_after();
            {
                // dq rows start on 32-byte boundaries whenever dq itself does (a row is head_dim
                // bf16, 128 or 256 bytes); a 16-byte-aligned dq takes 16-byte stores
                const bool dq32 = (reinterpret_cast<uintptr_t>(dq) & 31) == 0;
                __nv_bfloat16 *qrow = dq + ((int64_t(r.s0) + i) * p.heads + r.h) * D + (D / 2) * g;
#pragma unroll 1
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t a[32];
                    tmem_ld32(tmem + lane_base + Lay::kColDQ + (D / 2) * g + 32 * c, a);
                    tmem_wait_ld();
                    reg_fence(a);
                    if (valid) {
                        // rotary embedding: the accumulator is the gradient of the rotated q; turn
                        // its 16 pairs back (transposed rotation at this row's position)
                        if constexpr (kRope) {
                            // this chunk's 16 pairs, picked with constant indices (the arrays stay in registers)
                            float4 cc[4], ss[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                cc[u] = rcos[u];
                                ss[u] = rsin[u];
#pragma unroll
                                for (int cq = 1; cq < D / 64; ++cq)
                                    if (c == cq) {
                                        cc[u] = rcos[4 * cq + u];
                                        ss[u] = rsin[4 * cq + u];
                                    }
                            }
                            if (rope_in) rope_transpose_loaded<4>(cc, ss, a);
                            else if (c == 0) atomicOr(p.status, kStatusRopeRange); // past the tables
                        }
                        uint32_t pk[16];
#pragma unroll
                        for (int x = 0; x < 16; ++x)
                            pk[x] = pack_bf16x2(__uint_as_float(a[2 * x]) * p.scale, __uint_as_float(a[2 * x + 1]) * p.scale);
                        if (dq32) { // 32-byte stores: half the store instructions, each writing whole sectors
                            st_global_32b(qrow + 32 * c, pk);
                            st_global_32b(qrow + 32 * c + 16, pk + 8);
                        } else {
                            uint4 *dst = reinterpret_cast<uint4 *>(qrow + 32 * c);
#pragma unroll
                            for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.dq_free);
            }
            ++item_cnt;
            r = rn;
            have = have_next;
            delta_row = delta_next;
            lse_row = lse_next;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, Lay::kTmemCols);
    if (threadIdx.x == 0 && sb.abort) atomicOr(p.status, kStatusTimeout);
}

template <int D, int A>
cudaError_t launch_bwd_dq_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                const CUtensorMap &tdo, const CUtensorMap &to, const Problem &p, const float *lse,
                                float *neg_delta, float *nlse2, void *dq, int num_sms, cudaStream_t stream)
{
    using Lay = DqLayout<D>;
    // the rotary epilogue exists for block attention only, cross-attention for the generalized one
    auto kern = (A == kSoftmax && p.rope_cos)        ? bwd_dq_sm100_kernel<D, A == kSoftmax, A, false>
                : (A != kSoftmax && p.other_offsets) ? bwd_dq_sm100_kernel<D, false, A, A != kSoftmax>
                                                     : bwd_dq_sm100_kernel<D, false, A, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess) return e;
    // the register split only works if the CTA is launched with at least the budgets' sum
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * Lay::kThreads < int(256 * Lay::kRegsCompute + 128 * Lay::kRegsOther))
        return cudaErrorInvalidConfiguration;
    kern<<<num_sms, Lay::kThreads, Lay::kAlloc, stream>>>(tq, tk, tv, tdo, to, p, lse, neg_delta, nlse2,
                                                          static_cast<__nv_bfloat16 *>(dq));
    return cudaGetLastError();
}

#define BA_DQ_INST(D, A)                                                                                   \
    template cudaError_t launch_bwd_dq_sm100<D, A>(const CUtensorMap &, const CUtensorMap &,                \
                                                   const CUtensorMap &, const CUtensorMap &, const CUtensorMap &, \
                                                   const Problem &, const float *, float *, float *, void *, int, \
                                                   cudaStream_t);
BA_DQ_INST(64, kSoftmax)
BA_DQ_INST(128, kSoftmax)
BA_DQ_INST(64, kGelu)
BA_DQ_INST(128, kGelu)
BA_DQ_INST(64, kSilu)
BA_DQ_INST(128, kSilu)

} // namespace ba
