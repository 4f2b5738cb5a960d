// Block attention forward on sm_100a: TMA-staged Q/K/V tiles, tcgen05 MMAs
// with fp32 accumulators in TMEM, online softmax on the CUDA cores.
//
// What it computes ("Meta Scales GEM Ads Model Across Platforms and Thousands
// of GPUs", section "Kunlun changes how GEM scales"; "GEM (Meta)", section
// "Custom kernels", BlockAttention): for each query row i of each example and
// head, out_i = softmax over the visible keys j of (q_i . k_j / sqrt(D))
// applied to v_j, and lse_i = log of that softmax's normaliser. The work is
// tiled 128 queries x 128 keys; a query tile only visits the key tiles from
// its first row's window start up to the diagonal (block skipping), so the
// cost is linear in the example length for a fixed window.
//
// CTA roles (persistent: one CTA per SM, static round-robin over the
// (query tile, head) items):
//   warps 0-3  softmax: thread t owns TMEM lane t = query row t of the tile;
//              reads S, masks, keeps the running max/sum, writes P (bf16) back
//              into TMEM over S, rescales O when the max grows by > 2^8, and
//              stores out and lse at the end of the item;
//   warp 4     TMA producer: Q once per item (two buffers, so the next item's
//              Q arrives while this one runs), K and V per key tile into a ring;
//   warp 5     MMA issuer: S = Q K^T into one of two TMEM S buffers, then
//              O += P V with P read straight from TMEM (no shared-memory trip).
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D).
#include "ba_common.cuh"
#include "ba_kernels.cuh"
#include "ba_ptx.cuh"

#include <cuda_bf16.h>

namespace ba {

namespace {

template <int D>
struct FwdLayout {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr int kStages = D == 64 ? 4 : 2;
    static constexpr int kChunks = D / 64;               // 128-byte column chunks per row
    static constexpr int kChunkBytes = kTile * 128;      // one chunk of a 128-row tile
    static constexpr int kTileBytes = kTile * D * 2;     // one 128 x D bf16 tile
    static constexpr int kQ = 0;                         // two Q buffers (consecutive items)
    static constexpr int kK0 = 2 * kTileBytes;           // stage s: K at kK0 + 2 s tile, V after it
    static constexpr int kBytes = kTileBytes * (2 + 2 * kStages);
    static constexpr int kAlloc = kBytes + 1024;         // slack to align the base to 1024 B
    static constexpr int kThreads = 192;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColO = 256;
};

struct FwdBarriers {
    uint64_t q_full[2], q_empty[2], o_done, o_free;
    uint64_t s_full[2], p_full[2];
    uint64_t kv_full[4], kv_empty[4];
    uint32_t tmem_base;
    int abort;
};

} // namespace

template <int D>
__global__ void __launch_bounds__(192, 1)
    fwd_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const Problem p,
                          __nv_bfloat16 *__restrict__ out, float *__restrict__ lse)
{
    using Lay = FwdLayout<D>;
    constexpr int S = Lay::kStages;
    extern __shared__ uint8_t smem_raw[];
    __shared__ FwdBarriers sb;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&sb.q_full[0], 1);
        mbar_init(&sb.q_full[1], 1);
        mbar_init(&sb.q_empty[0], 1);
        mbar_init(&sb.q_empty[1], 1);
        mbar_init(&sb.o_done, 1);
        mbar_init(&sb.o_free, 4);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sb.s_full[i], 1);
            mbar_init(&sb.p_full[i], 4);
        }
        for (int i = 0; i < S; ++i) {
            mbar_init(&sb.kv_full[i], 1);
            mbar_init(&sb.kv_empty[i], 1);
        }
        sb.abort = 0;
        fence_mbar_init();
    }
    if (warp == 4 && lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
    }
    if (warp == 5) {
        tmem_alloc(&sb.tmem_base, Lay::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sb.tmem_base;
    volatile int *abort = &sb.abort;
    const int64_t B = p.block, W = p.window;

    if (warp == 4) {
        // ------------------------------------------------ TMA producer ---
        uint32_t kv_cnt = 0, item_cnt = 0;
        TileRef r;
        const int32_t ntiles = live_tile_count(p);
        for (int64_t n = blockIdx.x; decode_item(p, ntiles, n, r); n += gridDim.x, ++item_cnt) {
            const int jlo = int(window_start(int64_t(r.t) * kTile, B, W) / kTile);
            const int qb = item_cnt & 1;
            if (!mbar_wait(&sb.q_empty[qb], ((item_cnt >> 1) & 1) ^ 1, abort)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&sb.q_full[qb], Lay::kTileBytes);
                for (int c = 0; c < Lay::kChunks; ++c)
                    tma_load_2d(smem + Lay::kQ + qb * Lay::kTileBytes + c * Lay::kChunkBytes, &tm_q,
                                &sb.q_full[qb], r.h * D + c * 64, r.s0 + r.t * kTile);
            }
            __syncwarp();
            bool ok = true;
            for (int j = jlo; j <= r.t; ++j, ++kv_cnt) {
                const int st = kv_cnt % S;
                if (!mbar_wait(&sb.kv_empty[st], ((kv_cnt / S) & 1) ^ 1, abort)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t *kdst = smem + Lay::kK0 + 2 * st * Lay::kTileBytes;
                    uint8_t *vdst = kdst + Lay::kTileBytes;
                    mbar_arrive_expect_tx(&sb.kv_full[st], 2 * Lay::kTileBytes);
                    for (int c = 0; c < Lay::kChunks; ++c) {
                        tma_load_2d(kdst + c * Lay::kChunkBytes, &tm_k, &sb.kv_full[st],
                                    r.h * D + c * 64, r.s0 + j * kTile);
                        tma_load_2d(vdst + c * Lay::kChunkBytes, &tm_v, &sb.kv_full[st],
                                    r.h * D + c * 64, r.s0 + j * kTile);
                    }
                }
                __syncwarp();
            }
            if (!ok) break;
        }
    } else if (warp == 5) {
        // -------------------------------------------------- MMA issuer ---
        constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);
        constexpr uint32_t idesc_o = idesc_bf16(128, D, false, true);
        uint32_t kv_cnt = 0, s_cnt = 0, item_cnt = 0;
        TileRef r;
        const int32_t ntiles = live_tile_count(p);
        bool ok = true;
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x, ++item_cnt) {
            const int jlo = int(window_start(int64_t(r.t) * kTile, B, W) / kTile);
            const int nkv = r.t - jlo + 1;
            const int qb = item_cnt & 1;
            if (!mbar_wait(&sb.q_full[qb], (item_cnt >> 1) & 1, abort)) break;
            tc_fence_after();
            // O += P_m V_m for the key tile issued m-th in this item.
            auto issue_pv = [&](int m, uint32_t s_idx, uint32_t kv_idx) -> bool {
                if (!mbar_wait(&sb.p_full[s_idx & 1], (s_idx >> 1) & 1, abort)) return false;
                if (m == 0 && !mbar_wait(&sb.o_free, (item_cnt & 1) ^ 1, abort)) return false;
                tc_fence_after();
                if (lane == 0) {
                    const int st = kv_idx % S;
                    const uint32_t v_addr = smem_base + Lay::kK0 + (2 * st + 1) * Lay::kTileBytes;
                    const uint32_t a_tmem = tmem + (s_idx & 1) * 128;
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        const uint64_t bdesc = sdesc_sw128(v_addr + kk * 2048, Lay::kChunkBytes, 1024);
                        mma_ts(tmem + Lay::kColO, a_tmem + kk * 8, bdesc, idesc_o,
                               (m > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(&sb.kv_empty[st]);
                    tc_commit(&sb.o_done);
                }
                __syncwarp();
                return true;
            };
            for (int m = 0; m < nkv; ++m, ++s_cnt, ++kv_cnt) {
                const int st = kv_cnt % S;
                if (!mbar_wait(&sb.kv_full[st], (kv_cnt / S) & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t q_addr = smem_base + Lay::kQ + qb * Lay::kTileBytes;
                    const uint32_t k_addr = smem_base + Lay::kK0 + 2 * st * Lay::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32;
                        mma_ss(tmem + (s_cnt & 1) * 128, sdesc_sw128(q_addr + off, 16, 1024),
                               sdesc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&sb.s_full[s_cnt & 1]);
                    if (m == nkv - 1) tc_commit(&sb.q_empty[qb]);
                }
                __syncwarp();
                if (m > 0 && !issue_pv(m - 1, s_cnt - 1, kv_cnt - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok && !issue_pv(nkv - 1, s_cnt - 1, kv_cnt - 1)) ok = false;
        }
    } else {
        // ----------------------------------------------------- softmax ---
        const int row = threadIdx.x; // 0..127
        const uint32_t lane_base = uint32_t(warp * 32) << 16;
        const float scale_log2 = p.scale * 1.4426950408889634f;
        uint32_t s_cnt = 0, pv_cnt = 0;
        TileRef r;
        const int32_t ntiles = live_tile_count(p);
        bool ok = true;
        for (int64_t n = blockIdx.x; ok && decode_item(p, ntiles, n, r); n += gridDim.x) {
            const int64_t i = int64_t(r.t) * kTile + row;
            const bool valid = i < r.L;
            const int64_t ws = window_start(i, B, W);
            const int jlo = int(window_start(int64_t(r.t) * kTile, B, W) / kTile);
            const int nkv = r.t - jlo + 1;
            float m_ref = -INFINITY, l = 0.f;
            for (int m = 0; m < nkv; ++m, ++s_cnt) {
                const int64_t key0 = int64_t(jlo + m) * kTile;
                const uint32_t s_addr = tmem + lane_base + (s_cnt & 1) * 128;
                if (!mbar_wait(&sb.s_full[s_cnt & 1], (s_cnt >> 1) & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t sr[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, sr[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) reg_fence(sr[c]);
                // visible columns of this row: lo_c <= c <= hi_c
                int64_t lo64 = ws - key0, hi64 = i - key0;
                if (!valid) { lo64 = 1; hi64 = 0; }
                const int lo_c = int(lo64 < -1 ? -1 : (lo64 > 128 ? 128 : lo64));
                const int hi_c = int(hi64 < -1 ? -1 : (hi64 > 128 ? 128 : hi64));
                float x[128];
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                    const bool vis = c >= lo_c && c <= hi_c;
                    x[c] = vis ? __uint_as_float(sr[c / 32][c % 32]) * scale_log2 : -INFINITY;
                    mx = fmaxf(mx, x[c]);
                }
                const float m_new = fmaxf(m_ref, mx);
                const bool grow = m_new > m_ref + 8.0f;
                float alpha = 1.f;
                if (grow) {
                    alpha = ex2_approx(m_ref - m_new);
                    m_ref = m_new;
                }
                const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
                float rs = 0.f;
                uint32_t pk[4][16];
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float p0 = ex2_approx(x[2 * c] - m_use);
                    const float p1 = ex2_approx(x[2 * c + 1] - m_use);
                    rs += p0 + p1;
                    pk[c / 16][c % 16] = pack_bf16x2(p0, p1);
                }
                l = l * alpha + rs;
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_st16(s_addr + c * 16, pk[c]);
                tmem_wait_st();
                if (m > 0) {
                    // O must hold P_{m-1} V_{m-1} before it is rescaled.
                    if (!mbar_wait(&sb.o_done, pv_cnt & 1, abort)) {
                        ok = false;
                        break;
                    }
                    ++pv_cnt;
                    tc_fence_after();
                    if (__any_sync(0xffffffffu, grow)) {
                        const uint32_t o_addr = tmem + lane_base + Lay::kColO;
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t orr[32];
                            tmem_ld32(o_addr + c * 32, orr);
                            tmem_wait_ld();
                            reg_fence(orr);
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                orr[k] = __float_as_uint(__uint_as_float(orr[k]) * alpha);
                            tmem_st32(o_addr + c * 32, orr);
                        }
                        tmem_wait_st();
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.p_full[s_cnt & 1]);
            }
            if (!ok) break;
            // epilogue: wait for the last P V, normalise, store.
            if (!mbar_wait(&sb.o_done, pv_cnt & 1, abort)) break;
            ++pv_cnt;
            tc_fence_after();
            const uint32_t o_addr = tmem + lane_base + Lay::kColO;
            const float inv_l = valid ? 1.f / l : 0.f;
            __nv_bfloat16 *orow = out + ((int64_t(r.s0) + i) * p.heads + r.h) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t orr[32];
                tmem_ld32(o_addr + c * 32, orr);
                tmem_wait_ld();
                reg_fence(orr);
                if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint4 v4;
                        v4.x = pack_bf16x2(__uint_as_float(orr[8 * k + 0]) * inv_l,
                                           __uint_as_float(orr[8 * k + 1]) * inv_l);
                        v4.y = pack_bf16x2(__uint_as_float(orr[8 * k + 2]) * inv_l,
                                           __uint_as_float(orr[8 * k + 3]) * inv_l);
                        v4.z = pack_bf16x2(__uint_as_float(orr[8 * k + 4]) * inv_l,
                                           __uint_as_float(orr[8 * k + 5]) * inv_l);
                        v4.w = pack_bf16x2(__uint_as_float(orr[8 * k + 6]) * inv_l,
                                           __uint_as_float(orr[8 * k + 7]) * inv_l);
                        dst[k] = v4;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.o_free);
            if (valid)
                lse[int64_t(r.h) * p.total_tokens + r.s0 + i] =
                    (m_ref + log2f(l)) * 0.6931471805599453f;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, Lay::kTmemCols);
    if (threadIdx.x == 0 && sb.abort) atomicOr(p.status, kStatusTimeout);
}

template <int D>
cudaError_t launch_fwd_bf16_sm100(const CUtensorMap &tq, const CUtensorMap &tk,
                                  const CUtensorMap &tv, const Problem &p, void *out, float *lse,
                                  int num_sms, cudaStream_t stream)
{
    using Lay = FwdLayout<D>;
    auto kern = fwd_bf16_sm100_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess) return e;
    kern<<<num_sms, Lay::kThreads, Lay::kAlloc, stream>>>(tq, tk, tv, p,
                                                          static_cast<__nv_bfloat16 *>(out), lse);
    return cudaGetLastError();
}

template cudaError_t launch_fwd_bf16_sm100<64>(const CUtensorMap &, const CUtensorMap &,
                                               const CUtensorMap &, const Problem &, void *,
                                               float *, int, cudaStream_t);
template cudaError_t launch_fwd_bf16_sm100<128>(const CUtensorMap &, const CUtensorMap &,
                                                const CUtensorMap &, const Problem &, void *,
                                                float *, int, cudaStream_t);

} // namespace ba
