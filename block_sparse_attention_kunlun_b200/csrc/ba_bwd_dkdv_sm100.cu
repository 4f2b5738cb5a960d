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
// CTA roles (persistent, round-robin over (key tile, head) items):
//   warps 0-3 / 4-7  two compute warpgroups; thread t owns key row t (TMEM
//              lane t), group g the queries [64g, 64g+64) of each query tile.
//              They read S^T (then release it, so the next tile's S^T can be
//              issued while they work), form P^T, read dP^T, form dS^T and
//              write P^T and dS^T as bf16 over their dP^T columns.
//   warps 8-11 epilogue: at the end of an item, move dV and dK from TMEM to
//              global memory while the compute warps start the next item.
//   warp 12    TMA producer: K, V per item (with an L2 prefetch of the next
//              item's); Q, dO per query tile into a ring.
//   warp 13    MMA issuer.
// TMEM columns: S^T [0,128), dP^T [128,256), dV [256, 256+D), dK [256+D,
// 256+2D). After the compute warps have read group g's dP^T columns
// [128+64g, 192+64g), each 16-query block b of the group holds P^T (bf16) in
// [128+64g+16b, +8) and dS^T in the next 8 columns.
#include "ba_common.cuh"
#include "ba_kernels.cuh"
#include "ba_ptx.cuh"

#include <cuda_bf16.h>

namespace ba {

namespace {

template <int D>
struct DkvLayout {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkBytes = kTile * 128;
    static constexpr int kTileBytes = kTile * D * 2;
    static constexpr int kStages = D == 64 ? 3 : 2;      // Q / dO ring
    static constexpr int kK = 0;
    static constexpr int kV = kTileBytes;
    static constexpr int kQ0 = 2 * kTileBytes;           // stage s: Q at kQ0 + 2 s tile, dO after it
    static constexpr int kBytes = kQ0 + 2 * kStages * kTileBytes;
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr int kThreads = 448;
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
    static constexpr uint32_t kTmemCols = 512;
};

struct DkvBarriers {
    uint64_t kv_full, kv_empty, dkv_full, dkv_free;
    uint64_t qo_full[3], qo_empty[3];
    uint64_t s_full, s_free, dp_full, ds_full[2];
    uint32_t tmem_base;
    int abort;
    __align__(16) float lse2[2][kTile];
    __align__(16) float delta[2][kTile];
};

__device__ __forceinline__ void query_tile_range(const TileRef &r, int64_t B, int64_t W, int &ilo, int &ihi)
{
    const int64_t kmax = (int64_t(r.t) * kTile + kTile < r.L ? int64_t(r.t) * kTile + kTile : r.L) - 1;
    ilo = r.t;
    ihi = int(last_query_seeing(kmax, r.L, B, W) / kTile);
}

} // namespace

template <int D>
__global__ void __launch_bounds__(448, 1)
    bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const Problem p, const float *__restrict__ lse, const float *__restrict__ delta,
                          __nv_bfloat16 *__restrict__ dk, __nv_bfloat16 *__restrict__ dv)
{
    using Lay = DkvLayout<D>;
    constexpr int S = Lay::kStages;
    extern __shared__ uint8_t smem_raw[];
    __shared__ DkvBarriers sb;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&sb.kv_full, 1);
        mbar_init(&sb.kv_empty, 1);
        mbar_init(&sb.dkv_full, 1);
        mbar_init(&sb.dkv_free, 4);
        for (int i = 0; i < S; ++i) {
            mbar_init(&sb.qo_full[i], 1);
            mbar_init(&sb.qo_empty[i], 1);
        }
        mbar_init(&sb.s_full, 1);
        mbar_init(&sb.s_free, 8);
        mbar_init(&sb.dp_full, 1);
        mbar_init(&sb.ds_full[0], 4);
        mbar_init(&sb.ds_full[1], 4);
        sb.abort = 0;
        fence_mbar_init();
    }
    if (warp == 12 && lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
        tma_prefetch_map(&tm_do);
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
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x, ++item_cnt) {
            int ilo, ihi;
            query_tile_range(r, B, W, ilo, ihi);
            if (!mbar_wait(&sb.kv_empty, (item_cnt & 1) ^ 1, abort)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&sb.kv_full, 2 * Lay::kTileBytes);
                for (int c = 0; c < Lay::kChunks; ++c) {
                    tma_load_2d(smem + Lay::kK + c * Lay::kChunkBytes, &tm_k, &sb.kv_full, r.h * D + c * 64,
                                r.s0 + r.t * kTile);
                    tma_load_2d(smem + Lay::kV + c * Lay::kChunkBytes, &tm_v, &sb.kv_full, r.h * D + c * 64,
                                r.s0 + r.t * kTile);
                }
                // warm L2 with the next item's K and V
                TileRef rn;
                if (decode_item(p, ntiles, n + gridDim.x, rn))
                    for (int c = 0; c < Lay::kChunks; ++c) {
                        tma_prefetch_l2_2d(&tm_k, rn.h * D + c * 64, rn.s0 + rn.t * kTile);
                        tma_prefetch_l2_2d(&tm_v, rn.h * D + c * 64, rn.s0 + rn.t * kTile);
                    }
            }
            __syncwarp();
            for (int i = ilo; i <= ihi; ++i, ++it) {
                const int st = it % S;
                if (!mbar_wait(&sb.qo_empty[st], ((it / S) & 1) ^ 1, abort)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t *qdst = smem + Lay::kQ0 + 2 * st * Lay::kTileBytes;
                    mbar_arrive_expect_tx(&sb.qo_full[st], 2 * Lay::kTileBytes);
                    for (int c = 0; c < Lay::kChunks; ++c) {
                        tma_load_2d(qdst + c * Lay::kChunkBytes, &tm_q, &sb.qo_full[st], r.h * D + c * 64,
                                    r.s0 + i * kTile);
                        tma_load_2d(qdst + Lay::kTileBytes + c * Lay::kChunkBytes, &tm_do, &sb.qo_full[st],
                                    r.h * D + c * 64, r.s0 + i * kTile);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == 13) {
        // -------------------------------------------------- MMA issuer ---
        constexpr uint32_t idesc_sp = idesc_bf16(128, 128, false, false); // S^T, dP^T
        constexpr uint32_t idesc_kv = idesc_bf16(128, D, false, true);    // dV, dK (B MN-major)
        uint32_t it = 0, s_cnt = 0, d_cnt = 0, item_cnt = 0;
        TileRef r;
        bool ok = true;
        const uint32_t k_addr = smem_base + Lay::kK, v_addr = smem_base + Lay::kV;
        // dV += P^T dO and dK += dS^T Q of the query tile in ring stage st (m = its index in the item)
        auto issue_dkv = [&](int m, int st) -> bool {
            const uint32_t q_addr = smem_base + Lay::kQ0 + 2 * st * Lay::kTileBytes;
            const uint32_t o_addr = q_addr + Lay::kTileBytes;
            for (int g = 0; g < 2; ++g) {
                if (!mbar_wait(&sb.ds_full[g], d_cnt & 1, abort)) return false;
                if (m == 0 && g == 0 && !mbar_wait(&sb.dkv_free, (item_cnt & 1) ^ 1, abort)) return false;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t pcol = tmem + Lay::kColDP + 64 * g;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t boff = (4 * g + kk) * 2048; // query rows 64g + 16kk ..
                        const uint32_t acc = (m > 0 || g > 0 || kk > 0) ? 1u : 0u;
                        // P^T of queries 64g + 16kk .. at column 16kk of the group, dS^T 8 columns later
                        const uint32_t acol = pcol + 16 * kk;
                        mma_ts(tmem + Lay::kColDV, acol, sdesc_sw128(o_addr + boff, Lay::kChunkBytes, 1024),
                               idesc_kv, acc);
                        mma_ts(tmem + Lay::kColDK, acol + 8, sdesc_sw128(q_addr + boff, Lay::kChunkBytes, 1024),
                               idesc_kv, acc);
                    }
                    if (g == 1) tc_commit(&sb.qo_empty[st]);
                }
                __syncwarp();
            }
            ++d_cnt;
            return true;
        };
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x, ++item_cnt) {
            int ilo, ihi;
            query_tile_range(r, B, W, ilo, ihi);
            if (!mbar_wait(&sb.kv_full, item_cnt & 1, abort)) break;
            tc_fence_after();
            const int nq = ihi - ilo + 1;
            for (int m = 0; m < nq; ++m, ++it, ++s_cnt) {
                const int st = it % S;
                const uint32_t q_addr = smem_base + Lay::kQ0 + 2 * st * Lay::kTileBytes;
                const uint32_t o_addr = q_addr + Lay::kTileBytes;
                if (!mbar_wait(&sb.qo_full[st], (it / S) & 1, abort) ||
                    !mbar_wait(&sb.s_free, (s_cnt & 1) ^ 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32;
                        mma_ss(tmem + Lay::kColS, sdesc_sw128(k_addr + off, 16, 1024),
                               sdesc_sw128(q_addr + off, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&sb.s_full);
                }
                __syncwarp();
                // dV / dK of the previous query tile read P^T / dS^T from the dP^T
                // columns, so they go before this tile's dP^T.
                if (m > 0 && !issue_dkv(m - 1, (it - 1) % S)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32;
                        mma_ss(tmem + Lay::kColDP, sdesc_sw128(v_addr + off, 16, 1024),
                               sdesc_sw128(o_addr + off, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&sb.dp_full);
                    if (m == nq - 1) tc_commit(&sb.kv_empty); // K and V are not read again
                }
                __syncwarp();
            }
            if (!ok) break;
            if (!issue_dkv(nq - 1, (it - 1) % S)) break;
            if (lane == 0) tc_commit(&sb.dkv_full);
            __syncwarp();
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
        // -lse (log2 units, group 0) or -Delta (group 1) of query row `row` of tile i
        auto load_row = [&](const TileRef &rr, int i) -> float {
            const int64_t q = int64_t(i) * kTile + row;
            if (q >= rr.L) return g == 0 ? -INFINITY : 0.f;
            const int64_t gi = int64_t(rr.h) * T + rr.s0 + q;
            return g == 0 ? -lse[gi] * 1.4426950408889634f : -delta[gi];
        };
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x) {
            int ilo, ihi;
            query_tile_range(r, B, W, ilo, ihi);
            const int64_t k = int64_t(r.t) * kTile + row; // local key index
            const bool valid_k = k < r.L;
            const int64_t qmax = valid_k ? last_query_seeing(k, r.L, B, W) : -1;
            float nxt = load_row(r, ilo);
            for (int i = ilo; i <= ihi && ok; ++i, ++it) {
                const int buf = it & 1;
                (g == 0 ? sb.lse2[buf] : sb.delta[buf])[row] = nxt;
                named_bar_sync(1, 256);
                if (i < ihi) nxt = load_row(r, i + 1);
                const int64_t q0 = int64_t(i) * kTile + 64 * g;
                int64_t lo64 = k - q0, hi64 = qmax - q0;
                if (!valid_k) { lo64 = 1; hi64 = 0; }
                const int lo_c = int(lo64 < -1 ? -1 : (lo64 > 64 ? 64 : lo64));
                const int hi_c = int(hi64 < -1 ? -1 : (hi64 > 64 ? 64 : hi64));
                const bool full = __all_sync(0xffffffffu, lo_c <= 0 && hi_c >= 63);
                // shared copies hold -lse (log2 units) and -Delta, so each use is one packed FMA/add
                const float4 *l2v = reinterpret_cast<const float4 *>(sb.lse2[buf] + 64 * g);
                const float4 *dlv = reinterpret_cast<const float4 *>(sb.delta[buf] + 64 * g);
                // phase A: P^T from S^T
                if (!mbar_wait(&sb.s_full, it & 1, abort)) { ok = false; break; }
                tc_fence_after();
                float pr[64];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t sr[32];
                    tmem_ld32(tmem + lane_base + Lay::kColS + 64 * g + 32 * h2, sr);
                    tmem_wait_ld();
                    reg_fence(sr);
                    if (h2 == 1) { // both halves read: the next tile's S^T may overwrite them
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sb.s_free);
                    }
                    const float2 sc2 = make_float2(scale_log2, scale_log2);
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 l4 = l2v[8 * h2 + c4]; // -lse of 4 queries
                        const float2 x01 = ffma2(make_float2(__uint_as_float(sr[4 * c4]), __uint_as_float(sr[4 * c4 + 1])),
                                                 sc2, make_float2(l4.x, l4.y));
                        const float2 x23 = ffma2(make_float2(__uint_as_float(sr[4 * c4 + 2]), __uint_as_float(sr[4 * c4 + 3])),
                                                 sc2, make_float2(l4.z, l4.w));
                        const float xv[4] = {x01.x, x01.y, x23.x, x23.y};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int cc = 32 * h2 + 4 * c4 + e;
                            const float x = ex2_approx(xv[e]);
                            pr[cc] = (full || (cc >= lo_c && cc <= hi_c)) ? x : 0.f;
                        }
                    }
                }
                // phase B: dS^T = P^T (dP^T - Delta); 16 queries at a time, P^T and dS^T (bf16)
                // written over exactly the 16 dP^T columns just read
                if (!mbar_wait(&sb.dp_full, it & 1, abort)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    uint32_t dr[16];
                    tmem_ld16(tmem + lane_base + Lay::kColDP + 64 * g + 16 * b, dr);
                    tmem_wait_ld();
                    reg_fence(dr);
                    uint32_t pk[8], dk8[8];
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const float4 d4 = dlv[4 * b + c4]; // -Delta of 4 queries
                        const int q = 16 * b + 4 * c4, j = 4 * c4;
                        const float2 ds01 = fmul2(make_float2(pr[q], pr[q + 1]),
                                                  fadd2(make_float2(__uint_as_float(dr[j]), __uint_as_float(dr[j + 1])),
                                                        make_float2(d4.x, d4.y)));
                        const float2 ds23 = fmul2(make_float2(pr[q + 2], pr[q + 3]),
                                                  fadd2(make_float2(__uint_as_float(dr[j + 2]), __uint_as_float(dr[j + 3])),
                                                        make_float2(d4.z, d4.w)));
                        pk[2 * c4] = pack_bf16x2(pr[q], pr[q + 1]);
                        pk[2 * c4 + 1] = pack_bf16x2(pr[q + 2], pr[q + 3]);
                        dk8[2 * c4] = pack_bf16x2(ds01.x, ds01.y);
                        dk8[2 * c4 + 1] = pack_bf16x2(ds23.x, ds23.y);
                    }
                    tmem_st8(tmem + lane_base + Lay::kColDP + 64 * g + 16 * b, pk);
                    tmem_st8(tmem + lane_base + Lay::kColDP + 64 * g + 16 * b + 8, dk8);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.ds_full[g]);
            }
        }
    } else if (warp < 12) {
        // ---------------------------------------------------- epilogue ---
        const int row = threadIdx.x & 127;    // key row within the tile, TMEM lane
        const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
        uint32_t item_cnt = 0;
        TileRef r;
        for (int64_t n = blockIdx.x; decode_item(p, ntiles, n, r); n += gridDim.x, ++item_cnt) {
            const int64_t k = int64_t(r.t) * kTile + row;
            const bool valid_k = k < r.L;
            const int64_t grow = (int64_t(r.s0) + k) * p.heads + r.h;
            if (!mbar_wait(&sb.dkv_full, item_cnt & 1, abort)) break;
            tc_fence_after();
            // dV: load and store chunk by chunk
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t rr[32];
                tmem_ld32(tmem + lane_base + Lay::kColDV + c * 32, rr);
                tmem_wait_ld();
                reg_fence(rr);
                if (valid_k) {
                    uint4 *dst = reinterpret_cast<uint4 *>(dv + grow * D + c * 32);
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        dst[x] = make_uint4(pack_bf16x2(__uint_as_float(rr[8 * x + 0]), __uint_as_float(rr[8 * x + 1])),
                                            pack_bf16x2(__uint_as_float(rr[8 * x + 2]), __uint_as_float(rr[8 * x + 3])),
                                            pack_bf16x2(__uint_as_float(rr[8 * x + 4]), __uint_as_float(rr[8 * x + 5])),
                                            pack_bf16x2(__uint_as_float(rr[8 * x + 6]), __uint_as_float(rr[8 * x + 7])));
                }
            }
            // dK: take it all out of TMEM, release the accumulators, then store
            uint32_t kp[D / 2];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t rr[32];
                tmem_ld32(tmem + lane_base + Lay::kColDK + c * 32, rr);
                tmem_wait_ld();
                reg_fence(rr);
#pragma unroll
                for (int x = 0; x < 16; ++x)
                    kp[16 * c + x] = pack_bf16x2(__uint_as_float(rr[2 * x]) * p.scale,
                                                 __uint_as_float(rr[2 * x + 1]) * p.scale);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.dkv_free);
            if (valid_k) {
                uint4 *dst = reinterpret_cast<uint4 *>(dk + grow * D);
#pragma unroll
                for (int x = 0; x < D / 8; ++x) dst[x] = make_uint4(kp[4 * x], kp[4 * x + 1], kp[4 * x + 2], kp[4 * x + 3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 13) tmem_dealloc(tmem, Lay::kTmemCols);
    if (threadIdx.x == 0 && sb.abort) atomicOr(p.status, kStatusTimeout);
}

template <int D>
cudaError_t launch_bwd_dkdv_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const CUtensorMap &tdo, const Problem &p, const float *lse, const float *delta,
                                  void *dk, void *dv, int num_sms, cudaStream_t stream)
{
    using Lay = DkvLayout<D>;
    auto kern = bwd_dkdv_sm100_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess) return e;
    kern<<<num_sms, Lay::kThreads, Lay::kAlloc, stream>>>(tq, tk, tv, tdo, p, lse, delta,
                                                          static_cast<__nv_bfloat16 *>(dk),
                                                          static_cast<__nv_bfloat16 *>(dv));
    return cudaGetLastError();
}

template cudaError_t launch_bwd_dkdv_sm100<64>(const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                                               const CUtensorMap &, const Problem &, const float *, const float *,
                                               void *, void *, int, cudaStream_t);
template cudaError_t launch_bwd_dkdv_sm100<128>(const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                                                const CUtensorMap &, const Problem &, const float *, const float *,
                                                void *, void *, int, cudaStream_t);

} // namespace ba
