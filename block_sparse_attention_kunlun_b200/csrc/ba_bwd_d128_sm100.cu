// Block attention backward on sm_100a for head_dim 128, key-tile stationary,
// query tiles processed in two 64-query halves.
//
// Same mathematics as the head_dim-64 kernel (ba_bwd_sm100.cu): with P
// recomputed from the forward's lse,
//   dV += P^T dO,  dP = dO V^T,  dS = P o (dP - Delta),
//   dK += dS^T Q / sqrt(D),  dQ += dS K / sqrt(D).
// One item = one 128-key tile of one (example, head); it visits the query
// tiles from the diagonal to the last query whose window reaches the tile.
//
// Splitting each 128-query tile into two halves lets the compute warps work
// on one half while the tensor core runs the other half's MMAs, and lets dQ
// be produced transposed: dQ^T = K^T dS^T lands in TMEM with one head_dim
// column per lane, so each warp's reduction into the fp32 dq accumulator is a
// single coalesced 128-byte red.global.add per query.
//
// CTA roles (persistent, round-robin over items):
//   warps 0-3  compute: thread t owns key row t (TMEM lane t); per half reads
//              S^T and dP^T (64 columns each, 32 at a time), writes P^T and
//              dS^T as bf16 (A operands of the dV / dK MMAs) and dS into
//              shared memory (B operand of the dQ^T MMA); stores dK, dV at
//              the end of the item.
//   warps 4-7  dQ: thread t owns head_dim column 32(w-4)+lane; reads dQ^T of
//              a half (64 query columns) and reduce-adds it to dq_acc.
//   warp 8     TMA producer: K, V per item; Q, dO per query tile (2 stages).
//   warp 9     MMA issuer.
// TMEM columns per half h: S^T at [64h, 64h+64), dP^T at [128+64h, ...+64).
// Once the compute warps have read a half, P^T (bf16) occupies the first 32
// columns of its S^T block and dS^T (bf16) the first 32 of its dP^T block;
// dQ^T of queries 0-31 of the half goes to the last 32 columns of the S^T
// block and of queries 32-63 to the last 32 of the dP^T block.
// dV [256,384); dK [384,512).
#include "ba_common.cuh"
#include "ba_kernels.cuh"
#include "ba_ptx.cuh"

#include <cuda_bf16.h>

namespace ba {

namespace {

struct Bwd128Layout {
    static constexpr int D = 128;
    static constexpr int kStages = 2;
    static constexpr int kChunkBytes = kTile * 128;      // 64 columns of a 128-row tile
    static constexpr int kTileBytes = kTile * D * 2;     // 32 KB
    static constexpr int kHalfRows = 64;
    static constexpr int kK = 0;
    static constexpr int kV = kTileBytes;
    static constexpr int kQ0 = 2 * kTileBytes;           // stage s: Q at kQ0 + 2 s tile, dO after it
    static constexpr int kDS = kQ0 + 2 * kStages * kTileBytes;
    static constexpr int kDSHalf = kTile * 128;          // 128 keys x 64 queries bf16
    static constexpr int kBytes = kDS + 2 * kDSHalf;
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr int kThreads = 320;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColDP = 128, kColDV = 256, kColDK = 384;
};

struct Bwd128Barriers {
    uint64_t kv_full, kv_empty, dkv_full, dkv_free;
    uint64_t qo_full[2], qo_empty[2];
    uint64_t sp_full[2], ds_full[2], ds_free[2], dq_full[2], dq_free[2];
    uint32_t tmem_base;
    int abort;
    float lse2[kTile];
    float delta[kTile];
};

__device__ __forceinline__ void q_tile_range(const TileRef &r, int64_t B, int64_t W, int &ilo, int &ihi)
{
    const int64_t kmax = (int64_t(r.t) * kTile + kTile < r.L ? int64_t(r.t) * kTile + kTile : r.L) - 1;
    ilo = r.t;
    ihi = int(last_query_seeing(kmax, r.L, B, W) / kTile);
}

} // namespace

__global__ void __launch_bounds__(320, 1)
    bwd_d128_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const Problem p, const float *__restrict__ lse, const float *__restrict__ delta,
                          float *__restrict__ dq_acc, __nv_bfloat16 *__restrict__ dk,
                          __nv_bfloat16 *__restrict__ dv)
{
    using Lay = Bwd128Layout;
    constexpr int D = Lay::D;
    constexpr int S = Lay::kStages;
    extern __shared__ uint8_t smem_raw[];
    __shared__ Bwd128Barriers sb;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&sb.kv_full, 1);
        mbar_init(&sb.kv_empty, 1);
        mbar_init(&sb.dkv_full, 1);
        mbar_init(&sb.dkv_free, 4);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sb.qo_full[i], 1);
            mbar_init(&sb.qo_empty[i], 1);
            mbar_init(&sb.sp_full[i], 1);
            mbar_init(&sb.ds_full[i], 4);
            mbar_init(&sb.ds_free[i], 1);
            mbar_init(&sb.dq_full[i], 1);
            mbar_init(&sb.dq_free[i], 4);
        }
        sb.abort = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
        tma_prefetch_map(&tm_do);
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

    if (warp == 8) {
        // ------------------------------------------------ TMA producer ---
        uint32_t it = 0, item_cnt = 0;
        TileRef r;
        const int32_t ntiles = live_tile_count(p);
        bool ok = true;
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x, ++item_cnt) {
            int ilo, ihi;
            q_tile_range(r, B, W, ilo, ihi);
            if (!mbar_wait(&sb.kv_empty, (item_cnt & 1) ^ 1, abort)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&sb.kv_full, 2 * Lay::kTileBytes);
                for (int c = 0; c < 2; ++c) {
                    tma_load_2d(smem + Lay::kK + c * Lay::kChunkBytes, &tm_k, &sb.kv_full, r.h * D + c * 64,
                                r.s0 + r.t * kTile);
                    tma_load_2d(smem + Lay::kV + c * Lay::kChunkBytes, &tm_v, &sb.kv_full, r.h * D + c * 64,
                                r.s0 + r.t * kTile);
                }
            }
            __syncwarp();
            {
                // warm L2 with the next item's K and V: their loads wait for this item to finish
                TileRef rn;
                if (lane == 0 && decode_item(p, ntiles, n + gridDim.x, rn))
                    for (int c = 0; c < 2; ++c) {
                        tma_prefetch_l2_2d(&tm_k, rn.h * D + c * 64, rn.s0 + rn.t * kTile);
                        tma_prefetch_l2_2d(&tm_v, rn.h * D + c * 64, rn.s0 + rn.t * kTile);
                    }
                __syncwarp();
            }
            for (int i = ilo; i <= ihi; ++i, ++it) {
                const int st = it % S;
                if (!mbar_wait(&sb.qo_empty[st], ((it / S) & 1) ^ 1, abort)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t *qdst = smem + Lay::kQ0 + 2 * st * Lay::kTileBytes;
                    uint8_t *odst = qdst + Lay::kTileBytes;
                    mbar_arrive_expect_tx(&sb.qo_full[st], 2 * Lay::kTileBytes);
                    for (int c = 0; c < 2; ++c) {
                        tma_load_2d(qdst + c * Lay::kChunkBytes, &tm_q, &sb.qo_full[st], r.h * D + c * 64,
                                    r.s0 + i * kTile);
                        tma_load_2d(odst + c * Lay::kChunkBytes, &tm_do, &sb.qo_full[st], r.h * D + c * 64,
                                    r.s0 + i * kTile);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == 9) {
        // -------------------------------------------------- MMA issuer ---
        constexpr uint32_t idesc_sp = idesc_bf16(128, 64, false, false);  // S^T, dP^T halves
        constexpr uint32_t idesc_kv = idesc_bf16(128, D, false, true);    // dV, dK (B MN-major)
        constexpr uint32_t idesc_dq = idesc_bf16(128, 32, true, true);    // dQ^T quarter (A, B MN-major)
        uint32_t it = 0, item_cnt = 0;
        TileRef r;
        const int32_t ntiles = live_tile_count(p);
        bool ok = true;
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x, ++item_cnt) {
            int ilo, ihi;
            q_tile_range(r, B, W, ilo, ihi);
            if (!mbar_wait(&sb.kv_full, item_cnt & 1, abort)) break;
            tc_fence_after();
            const uint32_t k_addr = smem_base + Lay::kK, v_addr = smem_base + Lay::kV;
            for (int i = ilo; i <= ihi && ok; ++i, ++it) {
                const int st = it % S;
                const uint32_t q_addr = smem_base + Lay::kQ0 + 2 * st * Lay::kTileBytes;
                const uint32_t o_addr = q_addr + Lay::kTileBytes;
                if (!mbar_wait(&sb.qo_full[st], (it / S) & 1, abort)) {
                    ok = false;
                    break;
                }
                // S^T and dP^T for both halves
                for (int h = 0; h < 2; ++h) {
                    if (!mbar_wait(&sb.dq_free[h], (it & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t hoff = h * (Lay::kHalfRows * 128);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32;
                            mma_ss(tmem + 64 * h, sdesc_sw128(k_addr + off, 16, 1024),
                                   sdesc_sw128(q_addr + off + hoff, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
                        }
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32;
                            mma_ss(tmem + Lay::kColDP + 64 * h, sdesc_sw128(v_addr + off, 16, 1024),
                                   sdesc_sw128(o_addr + off + hoff, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
                        }
                        tc_commit(&sb.sp_full[h]);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                // dV, dK, dQ^T per half once its P^T / dS^T are ready
                for (int h = 0; h < 2; ++h) {
                    if (!mbar_wait(&sb.ds_full[h], it & 1, abort) ||
                        (i == ilo && h == 0 && !mbar_wait(&sb.dkv_free, (item_cnt & 1) ^ 1, abort))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t hoff = h * (Lay::kHalfRows * 128);
                        const uint32_t scol = tmem + 64 * h, pcol = tmem + Lay::kColDP + 64 * h;
                        const bool first = (i == ilo && h == 0);
#pragma unroll
                        for (int kk = 0; kk < Lay::kHalfRows / 16; ++kk)
                            mma_ts(tmem + Lay::kColDV, scol + kk * 8,
                                   sdesc_sw128(o_addr + hoff + kk * 2048, Lay::kChunkBytes, 1024), idesc_kv,
                                   (!first || kk > 0) ? 1u : 0u);
#pragma unroll
                        for (int kk = 0; kk < Lay::kHalfRows / 16; ++kk)
                            mma_ts(tmem + Lay::kColDK, pcol + kk * 8,
                                   sdesc_sw128(q_addr + hoff + kk * 2048, Lay::kChunkBytes, 1024), idesc_kv,
                                   (!first || kk > 0) ? 1u : 0u);
                        const uint32_t ds_addr = smem_base + Lay::kDS + h * Lay::kDSHalf;
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk) {
                            const uint64_t adesc = sdesc_sw128(k_addr + kk * 2048, Lay::kChunkBytes, 1024);
                            // queries 0-31 of the half start at byte 0 of each dS row, 32-63 at byte 64
                            mma_ss(scol + 32, adesc, sdesc_sw128(ds_addr + kk * 2048, Lay::kChunkBytes, 1024),
                                   idesc_dq, kk > 0 ? 1u : 0u);
                            mma_ss(pcol + 32, adesc, sdesc_sw128(ds_addr + 64 + kk * 2048, Lay::kChunkBytes, 1024),
                                   idesc_dq, kk > 0 ? 1u : 0u);
                        }
                        tc_commit(&sb.ds_free[h]);
                        tc_commit(&sb.dq_full[h]);
                        if (h == 1) {
                            tc_commit(&sb.qo_empty[st]);
                            if (i == ihi) {
                                tc_commit(&sb.dkv_full);
                                tc_commit(&sb.kv_empty);
                            }
                        }
                    }
                    __syncwarp();
                }
            }
        }
    } else if (warp < 4) {
        // ----------------------------------------------------- compute ---
        const int row = threadIdx.x; // key row within the tile, TMEM lane
        const uint32_t lane_base = uint32_t(warp * 32) << 16;
        const float scale_log2 = p.scale * 1.4426950408889634f;
        uint32_t it = 0, item_cnt = 0;
        TileRef r;
        const int32_t ntiles = live_tile_count(p);
        bool ok = true;
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x, ++item_cnt) {
            int ilo, ihi;
            q_tile_range(r, B, W, ilo, ihi);
            const int64_t k = int64_t(r.t) * kTile + row; // local key index
            const bool valid_k = k < r.L;
            const int64_t qmax = valid_k ? last_query_seeing(k, r.L, B, W) : -1;
            // lse (log2 units) and Delta of query row `row` of tile i; loaded one tile ahead
            auto load_row = [&](int i, float &l2, float &dl) {
                const int64_t q = int64_t(i) * kTile + row;
                l2 = INFINITY;
                dl = 0.f;
                if (q < r.L) {
                    const int64_t g = int64_t(r.h) * T + r.s0 + q;
                    l2 = lse[g] * 1.4426950408889634f;
                    dl = delta[g];
                }
            };
            float nl2, ndl;
            load_row(ilo, nl2, ndl);
            for (int i = ilo; i <= ihi && ok; ++i, ++it) {
                named_bar_sync(1, 128); // everyone is done with the previous tile's lse / Delta
                sb.lse2[row] = nl2;
                sb.delta[row] = ndl;
                named_bar_sync(1, 128);
                if (i < ihi) load_row(i + 1, nl2, ndl);
                for (int h = 0; h < 2; ++h) {
                    if (!mbar_wait(&sb.sp_full[h], it & 1, abort) ||
                        !mbar_wait(&sb.ds_free[h], (it & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int64_t q0 = int64_t(i) * kTile + 64 * h;
                    int64_t lo64 = k - q0, hi64 = qmax - q0;
                    if (!valid_k) { lo64 = 1; hi64 = 0; }
                    const int lo_c = int(lo64 < -1 ? -1 : (lo64 > 64 ? 64 : lo64));
                    const int hi_c = int(hi64 < -1 ? -1 : (hi64 > 64 ? 64 : hi64));
                    const float *l2s = sb.lse2 + 64 * h;
                    const float *dls = sb.delta + 64 * h;
                    const uint32_t s_addr = tmem + lane_base + 64 * h;
                    const uint32_t p_addr = tmem + lane_base + Lay::kColDP + 64 * h;
                    uint8_t *ds_row = smem + Lay::kDS + h * Lay::kDSHalf + row * 128;
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        uint32_t sr[32], pr[32];
                        tmem_ld32(s_addr + 32 * c2, sr);
                        tmem_ld32(p_addr + 32 * c2, pr);
                        tmem_wait_ld();
                        reg_fence(sr);
                        reg_fence(pr);
                        uint32_t pk[16], dk16[16];
#pragma unroll
                        for (int x = 0; x < 16; ++x) {
                            float pv[2], dsv[2];
#pragma unroll
                            for (int y = 0; y < 2; ++y) {
                                const int col = 32 * c2 + 2 * x + y;
                                const bool vis = col >= lo_c && col <= hi_c;
                                const float pe =
                                    ex2_approx(__uint_as_float(sr[2 * x + y]) * scale_log2 - l2s[col]);
                                pv[y] = vis ? pe : 0.f;
                                dsv[y] = vis ? pe * (__uint_as_float(pr[2 * x + y]) - dls[col]) : 0.f;
                            }
                            pk[x] = pack_bf16x2(pv[0], pv[1]);
                            dk16[x] = pack_bf16x2(dsv[0], dsv[1]);
                        }
                        // P^T and dS^T overwrite columns this thread has already read
                        tmem_st16(s_addr + 16 * c2, pk);
                        tmem_st16(p_addr + 16 * c2, dk16);
                        // dS of this key row, queries 32 c2 .. 32 c2 + 31 of the half (128B-swizzled row)
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            *reinterpret_cast<uint4 *>(ds_row + (((4 * c2 + u) ^ (row & 7)) * 16)) =
                                make_uint4(dk16[4 * u], dk16[4 * u + 1], dk16[4 * u + 2], dk16[4 * u + 3]);
                    }
                    tmem_wait_st();
                    fence_proxy_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sb.ds_full[h]);
                }
            }
            if (!ok) break;
            // epilogue: dV, dK of this key tile
            if (!mbar_wait(&sb.dkv_full, item_cnt & 1, abort)) break;
            tc_fence_after();
            const int64_t grow = (int64_t(r.s0) + k) * p.heads + r.h;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t col0 = which == 0 ? Lay::kColDV : Lay::kColDK;
                const float mul = which == 0 ? 1.f : p.scale;
                __nv_bfloat16 *dst_row = (which == 0 ? dv : dk) + grow * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t rr[32];
                    tmem_ld32(tmem + lane_base + col0 + c * 32, rr);
                    tmem_wait_ld();
                    reg_fence(rr);
                    if (valid_k) {
                        uint4 *dst = reinterpret_cast<uint4 *>(dst_row + c * 32);
#pragma unroll
                        for (int x = 0; x < 4; ++x)
                            dst[x] = make_uint4(
                                pack_bf16x2(__uint_as_float(rr[8 * x + 0]) * mul, __uint_as_float(rr[8 * x + 1]) * mul),
                                pack_bf16x2(__uint_as_float(rr[8 * x + 2]) * mul, __uint_as_float(rr[8 * x + 3]) * mul),
                                pack_bf16x2(__uint_as_float(rr[8 * x + 4]) * mul, __uint_as_float(rr[8 * x + 5]) * mul),
                                pack_bf16x2(__uint_as_float(rr[8 * x + 6]) * mul, __uint_as_float(rr[8 * x + 7]) * mul));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.dkv_free);
        }
    } else {
        // ---------------------------------------------------------- dQ ---
        const int d = (warp - 4) * 32 + lane; // head_dim column owned by this thread (TMEM lane)
        const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
        uint32_t it = 0;
        TileRef r;
        const int32_t ntiles = live_tile_count(p);
        bool ok = true;
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x) {
            int ilo, ihi;
            q_tile_range(r, B, W, ilo, ihi);
            float *acc_h = dq_acc + (int64_t(r.h) * T + r.s0) * D + d;
            for (int i = ilo; i <= ihi && ok; ++i, ++it) {
                for (int h = 0; h < 2; ++h) {
                    if (!mbar_wait(&sb.dq_full[h], it & 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint32_t a[64];
                    tmem_ld32(tmem + lane_base + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
                    tmem_ld32(tmem + lane_base + Lay::kColDP + 64 * h + 32,
                              *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
                    tmem_wait_ld();
                    reg_fence(a);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sb.dq_free[h]);
                    const int64_t q0 = int64_t(i) * kTile + 64 * h;
                    const int nq = int(r.L - q0 < 64 ? r.L - q0 : 64);
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c < nq) atomicAdd(acc_h + (q0 + c) * D, __uint_as_float(a[c]));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, Lay::kTmemCols);
    if (threadIdx.x == 0 && sb.abort) atomicOr(p.status, kStatusTimeout);
}

cudaError_t launch_bwd_d128_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const CUtensorMap &tdo, const Problem &p, const float *lse, const float *delta,
                                  float *dq_acc, void *dk, void *dv, int num_sms, cudaStream_t stream)
{
    using Lay = Bwd128Layout;
    cudaError_t e =
        cudaFuncSetAttribute(bwd_d128_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess) return e;
    bwd_d128_sm100_kernel<<<num_sms, Lay::kThreads, Lay::kAlloc, stream>>>(
        tq, tk, tv, tdo, p, lse, delta, dq_acc, static_cast<__nv_bfloat16 *>(dk), static_cast<__nv_bfloat16 *>(dv));
    return cudaGetLastError();
}

} // namespace ba
