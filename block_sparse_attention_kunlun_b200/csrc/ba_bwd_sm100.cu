// Block attention backward on sm_100a, key-tile stationary (head_dim 64;
// head_dim 128 has its own kernel in ba_bwd_d128_sm100.cu).
//
// Gradients of out = softmax(q k^T / sqrt(D)) v over the visible keys
// (visibility rule in ba_common.cuh), with the probabilities recomputed from
// the forward's lse so that nothing else is kept between the passes:
//   P = exp(S / sqrt(D) - lse),  dV += P^T dO,  dP = dO V^T,
//   dS = P o (dP - Delta),  dK += dS^T Q / sqrt(D),  dQ += dS K / sqrt(D),
// with Delta_i = dO_i . out_i from the pre-pass. ("GEM (Meta)", section
// "Custom kernels", BlockAttention: the page's kernel trains, so it has a
// backward; it gives no formulas -- these are the exact gradients.)
//
// One item = one 128-key tile of one (example, head). It visits only the
// query tiles that can see the key tile: from the diagonal up to the last
// query whose window still reaches the tile.
//
// CTA roles (persistent, round-robin over items):
//   warps 0-3  compute: thread t owns key row t (TMEM lane t). Reads S^T and
//              dP^T from TMEM, writes P^T and dS^T back as bf16 (A operands
//              of the dV / dK MMAs) and dS to shared memory (A operand of the
//              dQ MMA); at the end of the item stores dK and dV.
//   warps 4-7  dQ: thread t owns query row t of the dQ tile; moves it from
//              TMEM to the fp32 dq accumulator with vector atomic adds.
//   warp 8     TMA producer: K, V once per item; Q, dO per query tile.
//   warp 9     MMA issuer.
// TMEM columns: S^T [0,128) -> P^T bf16 [0,64); dP^T [128,256) -> dS^T bf16
// [128,192); dQ halves at [64,128) and [192,256) (free once P^T and dS^T are
// packed); dV [256, 256+D); dK [256+D, 256+2D).
#include "ba_common.cuh"
#include "ba_kernels.cuh"
#include "ba_ptx.cuh"

#include <cuda_bf16.h>

namespace ba {

namespace {

template <int D>
struct BwdLayout {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr int kStages = D == 64 ? 2 : 1;
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkBytes = kTile * 128;
    static constexpr int kTileBytes = kTile * D * 2;
    static constexpr int kK = 0;
    static constexpr int kV = kTileBytes;
    static constexpr int kQ0 = 2 * kTileBytes;            // stage s: Q at kQ0 + 2 s tile, dO after it
    static constexpr int kDS = kQ0 + 2 * kStages * kTileBytes;
    static constexpr int kDSBytes = kTile * kTile * 2;    // 128 keys x 128 queries bf16
    static constexpr int kBytes = kDS + kDSBytes;
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr int kThreads = 320;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColDP = 128, kColDV = 256, kColDK = 256 + D;
};

struct BwdBarriers {
    uint64_t kv_full, kv_empty, sp_full, ds_full, ds_free, dq_full, dq_free, dkv_full, dkv_free;
    uint64_t qo_full[2], qo_empty[2];
    uint32_t tmem_base;
    int abort;
    float lse2[2][kTile];
    float delta[2][kTile];
};

__device__ __forceinline__ void last_q_tile(const TileRef &r, int64_t B, int64_t W, int &ilo, int &ihi)
{
    const int64_t kmax = (int64_t(r.t) * kTile + kTile < r.L ? int64_t(r.t) * kTile + kTile : r.L) - 1;
    ilo = r.t;
    ihi = int(last_query_seeing(kmax, r.L, B, W) / kTile);
}

} // namespace

template <int D>
__global__ void __launch_bounds__(320, 1)
    bwd_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_do, const Problem p,
                          const float *__restrict__ lse, const float *__restrict__ delta,
                          float *__restrict__ dq_acc, __nv_bfloat16 *__restrict__ dk,
                          __nv_bfloat16 *__restrict__ dv)
{
    using Lay = BwdLayout<D>;
    constexpr int S = Lay::kStages;
    extern __shared__ uint8_t smem_raw[];
    __shared__ BwdBarriers sb;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&sb.kv_full, 1);
        mbar_init(&sb.kv_empty, 1);
        mbar_init(&sb.sp_full, 1);
        mbar_init(&sb.ds_full, 4);
        mbar_init(&sb.ds_free, 1);
        mbar_init(&sb.dq_full, 1);
        mbar_init(&sb.dq_free, 4);
        mbar_init(&sb.dkv_full, 1);
        mbar_init(&sb.dkv_free, 4);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sb.qo_full[i], 1);
            mbar_init(&sb.qo_empty[i], 1);
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
            last_q_tile(r, B, W, ilo, ihi);
            if (!mbar_wait(&sb.kv_empty, (item_cnt & 1) ^ 1, abort)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&sb.kv_full, 2 * Lay::kTileBytes);
                for (int c = 0; c < Lay::kChunks; ++c) {
                    tma_load_2d(smem + Lay::kK + c * Lay::kChunkBytes, &tm_k, &sb.kv_full,
                                r.h * D + c * 64, r.s0 + r.t * kTile);
                    tma_load_2d(smem + Lay::kV + c * Lay::kChunkBytes, &tm_v, &sb.kv_full,
                                r.h * D + c * 64, r.s0 + r.t * kTile);
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
                    uint8_t *odst = qdst + Lay::kTileBytes;
                    mbar_arrive_expect_tx(&sb.qo_full[st], 2 * Lay::kTileBytes);
                    for (int c = 0; c < Lay::kChunks; ++c) {
                        tma_load_2d(qdst + c * Lay::kChunkBytes, &tm_q, &sb.qo_full[st],
                                    r.h * D + c * 64, r.s0 + i * kTile);
                        tma_load_2d(odst + c * Lay::kChunkBytes, &tm_do, &sb.qo_full[st],
                                    r.h * D + c * 64, r.s0 + i * kTile);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == 9) {
        // -------------------------------------------------- MMA issuer ---
        constexpr uint32_t idesc_sp = idesc_bf16(128, 128, false, false);  // S^T, dP^T
        constexpr uint32_t idesc_kv = idesc_bf16(128, D, false, true);      // dV, dK (B MN-major)
        constexpr uint32_t idesc_dq = idesc_bf16(128, 64, true, true);      // dQ halves (A, B MN-major)
        uint32_t it = 0, item_cnt = 0;
        TileRef r;
        const int32_t ntiles = live_tile_count(p);
        bool ok = true;
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x, ++item_cnt) {
            int ilo, ihi;
            last_q_tile(r, B, W, ilo, ihi);
            if (!mbar_wait(&sb.kv_full, item_cnt & 1, abort)) break;
            tc_fence_after();
            const uint32_t k_addr = smem_base + Lay::kK, v_addr = smem_base + Lay::kV;
            const uint32_t ds_addr = smem_base + Lay::kDS;
            for (int i = ilo; i <= ihi; ++i, ++it) {
                const int st = it % S;
                const uint32_t q_addr = smem_base + Lay::kQ0 + 2 * st * Lay::kTileBytes;
                const uint32_t o_addr = q_addr + Lay::kTileBytes;
                if (!mbar_wait(&sb.qo_full[st], (it / S) & 1, abort) ||
                    !mbar_wait(&sb.dq_free, (it & 1) ^ 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32;
                        mma_ss(tmem, sdesc_sw128(k_addr + off, 16, 1024),
                               sdesc_sw128(q_addr + off, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32;
                        mma_ss(tmem + Lay::kColDP, sdesc_sw128(v_addr + off, 16, 1024),
                               sdesc_sw128(o_addr + off, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&sb.sp_full);
                }
                __syncwarp();
                if (!mbar_wait(&sb.ds_full, it & 1, abort) ||
                    (i == ilo && !mbar_wait(&sb.dkv_free, (item_cnt & 1) ^ 1, abort))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t acc0 = i > ilo ? 1u : 0u;
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        // dV += P^T dO : A = P^T (TMEM), B = dO (N = D, K = queries; MN-major)
                        mma_ts(tmem + Lay::kColDV, tmem + kk * 8,
                               sdesc_sw128(o_addr + kk * 2048, Lay::kChunkBytes, 1024), idesc_kv,
                               (acc0 || kk > 0) ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        // dK += dS^T Q : A = dS^T (TMEM), B = Q (MN-major)
                        mma_ts(tmem + Lay::kColDK, tmem + Lay::kColDP + kk * 8,
                               sdesc_sw128(q_addr + kk * 2048, Lay::kChunkBytes, 1024), idesc_kv,
                               (acc0 || kk > 0) ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        // dQ = dS K : A = dS (M = queries, K = keys; MN-major in smem),
                        // B = K (N = D, K = keys; MN-major), N split into 64-column halves.
                        const uint64_t adesc = sdesc_sw128(ds_addr + kk * 2048, Lay::kChunkBytes, 1024);
                        mma_ss(tmem + 64, adesc, sdesc_sw128(k_addr + kk * 2048, Lay::kChunkBytes, 1024),
                               idesc_dq, kk > 0 ? 1u : 0u);
                        if (D == 128)
                            mma_ss(tmem + 192, adesc,
                                   sdesc_sw128(k_addr + Lay::kChunkBytes + kk * 2048, Lay::kChunkBytes, 1024),
                                   idesc_dq, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&sb.qo_empty[st]);
                    tc_commit(&sb.ds_free);
                    tc_commit(&sb.dq_full);
                    if (i == ihi) {
                        tc_commit(&sb.dkv_full);
                        tc_commit(&sb.kv_empty);
                    }
                }
                __syncwarp();
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
            last_q_tile(r, B, W, ilo, ihi);
            const int64_t k = int64_t(r.t) * kTile + row; // local key index
            const bool valid_k = k < r.L;
            const int64_t qmax = valid_k ? last_query_seeing(k, r.L, B, W) : -1;
            for (int i = ilo; i <= ihi; ++i, ++it) {
                // lse (log2 units) and Delta of the 128 queries of this tile
                {
                    const int64_t q = int64_t(i) * kTile + row;
                    float l2 = INFINITY, dl = 0.f;
                    if (q < r.L) {
                        const int64_t g = int64_t(r.h) * T + r.s0 + q;
                        l2 = lse[g] * 1.4426950408889634f;
                        dl = delta[g];
                    }
                    sb.lse2[it & 1][row] = l2;
                    sb.delta[it & 1][row] = dl;
                }
                named_bar_sync(1, 128);
                if (!mbar_wait(&sb.sp_full, it & 1, abort) ||
                    !mbar_wait(&sb.ds_free, (it & 1) ^ 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int64_t q0 = int64_t(i) * kTile;
                int64_t lo64 = k - q0, hi64 = qmax - q0;
                if (!valid_k) { lo64 = 1; hi64 = 0; }
                const int lo_c = int(lo64 < -1 ? -1 : (lo64 > 128 ? 128 : lo64));
                const int hi_c = int(hi64 < -1 ? -1 : (hi64 > 128 ? 128 : hi64));
                const float *l2s = sb.lse2[it & 1];
                const float *dls = sb.delta[it & 1];
                uint8_t *ds_row = smem + Lay::kDS + row * 128;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t sr[32], pr[32];
                    tmem_ld32(tmem + lane_base + c * 32, sr);
                    tmem_ld32(tmem + lane_base + Lay::kColDP + c * 32, pr);
                    tmem_wait_ld();
                    reg_fence(sr);
                    reg_fence(pr);
                    uint32_t pk[16], dk16[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        float pv[2], dsv[2];
#pragma unroll
                        for (int y = 0; y < 2; ++y) {
                            const int col = c * 32 + 2 * x + y;
                            const bool vis = col >= lo_c && col <= hi_c;
                            const float pe = ex2_approx(__uint_as_float(sr[2 * x + y]) * scale_log2 - l2s[col]);
                            pv[y] = vis ? pe : 0.f;
                            dsv[y] = vis ? pe * (__uint_as_float(pr[2 * x + y]) - dls[col]) : 0.f;
                        }
                        pk[x] = pack_bf16x2(pv[0], pv[1]);
                        dk16[x] = pack_bf16x2(dsv[0], dsv[1]);
                    }
                    tmem_st16(tmem + lane_base + c * 16, pk);
                    tmem_st16(tmem + lane_base + Lay::kColDP + c * 16, dk16);
                    // dS row (this key) into the 128B-swizzled [keys x queries] tile
                    uint8_t *chunk = ds_row + (c >> 1) * Lay::kChunkBytes;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int unit = ((c & 1) * 4 + u) ^ (row & 7);
                        *reinterpret_cast<uint4 *>(chunk + unit * 16) =
                            make_uint4(dk16[4 * u], dk16[4 * u + 1], dk16[4 * u + 2], dk16[4 * u + 3]);
                    }
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.ds_full);
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
        const int row = threadIdx.x - 128; // query row within the tile, TMEM lane
        const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
        uint32_t it = 0;
        TileRef r;
        const int32_t ntiles = live_tile_count(p);
        bool ok = true;
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x) {
            int ilo, ihi;
            last_q_tile(r, B, W, ilo, ihi);
            for (int i = ilo; i <= ihi; ++i, ++it) {
                if (!mbar_wait(&sb.dq_full, it & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t a[D];
                tmem_ld32(tmem + lane_base + 64, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
                tmem_ld32(tmem + lane_base + 96, *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
                if (D == 128) {
                    tmem_ld32(tmem + lane_base + 192, *reinterpret_cast<uint32_t(*)[32]>(&a[D == 128 ? 64 : 0]));
                    tmem_ld32(tmem + lane_base + 224, *reinterpret_cast<uint32_t(*)[32]>(&a[D == 128 ? 96 : 0]));
                }
                tmem_wait_ld();
                reg_fence(a);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.dq_free);
                const int64_t q = int64_t(i) * kTile + row;
                if (q < r.L) {
                    float4 *dst = reinterpret_cast<float4 *>(
                        dq_acc + ((int64_t(r.h) * T + r.s0 + q) * D));
#pragma unroll
                    for (int x = 0; x < D / 4; ++x)
                        atomicAdd(dst + x, make_float4(__uint_as_float(a[4 * x]), __uint_as_float(a[4 * x + 1]),
                                                       __uint_as_float(a[4 * x + 2]), __uint_as_float(a[4 * x + 3])));
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

template <int D>
cudaError_t launch_bwd_bf16_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const CUtensorMap &tdo, const Problem &p, const float *lse,
                                  const float *delta, float *dq_acc, void *dk, void *dv, int num_sms,
                                  cudaStream_t stream)
{
    using Lay = BwdLayout<D>;
    auto kern = bwd_bf16_sm100_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess) return e;
    kern<<<num_sms, Lay::kThreads, Lay::kAlloc, stream>>>(tq, tk, tv, tdo, p, lse, delta, dq_acc,
                                                          static_cast<__nv_bfloat16 *>(dk),
                                                          static_cast<__nv_bfloat16 *>(dv));
    return cudaGetLastError();
}

template cudaError_t launch_bwd_bf16_sm100<64>(const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                                               const CUtensorMap &, const Problem &, const float *,
                                               const float *, float *, void *, void *, int, cudaStream_t);

} // namespace ba
