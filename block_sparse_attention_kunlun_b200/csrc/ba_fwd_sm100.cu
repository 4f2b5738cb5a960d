// Block attention forward on sm_100a: TMA-staged Q/K/V tiles, tcgen05 MMAs
// with fp32 accumulators in TMEM, online softmax on the CUDA cores.
//
// What it computes ("Meta Scales GEM Ads Model Across Platforms and Thousands
// of GPUs", section "Kunlun changes how GEM scales"; "GEM (Meta)", section
// "Custom kernels", BlockAttention): for each query row i of each example and
// head, out_i = softmax over the visible keys j of (q_i . k_j / sqrt(D))
// applied to v_j, and lse_i = log of that softmax's normaliser. Work is tiled
// 128 queries x 128 keys; a query tile only visits the key tiles from its
// first row's window start up to the diagonal (block skipping), so the cost
// is linear in the example length for a fixed window.
//
// One item = two consecutive query tiles (t, t+1) of one (example, head).
// Their key-tile ranges overlap almost entirely, so each K/V tile is loaded
// once and used by both. Two softmax warpgroups own one query tile each; the
// MMA warp interleaves their work as
//   ... PV0(j-1) S0(j) | PV1(j-1) S1(j) | PV0(j) S0(j+1) | ...
// so that one group's softmax runs while the tensor core serves the other.
//
// CTA roles (persistent, round-robin over items):
//   warps 0-3 / 4-7  softmax group w: thread t owns TMEM lane t = query row t
//              of tile t+w. Reads S, masks, keeps the running max/sum (O is
//              rescaled only when the max grows by more than 2^8), writes P
//              (bf16) back over S for the P V MMA, stores out and lse.
//   warp 8     TMA producer: both Q tiles per item, K and V per key tile
//              into a ring shared by the two groups.
//   warp 9     MMA issuer.
// TMEM columns: S of group w at [128w, 128w+128) (P bf16 in its first 64),
// O of group w at [256 + D w, 256 + D w + D).
#include "ba_common.cuh"
#include "ba_kernels.cuh"
#include "ba_ptx.cuh"
#include "ba_sched.cuh"

#include <cuda_bf16.h>
#include <type_traits>

namespace ba {

namespace {

template <int D>
struct FwdLayout {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr int kStages = D == 64 ? 4 : 2;
    static constexpr int kChunks = D / 64;               // 128-byte column chunks per row
    static constexpr int kChunkBytes = kTile * 128;      // one chunk of a 128-row tile
    static constexpr int kTileBytes = kTile * D * 2;     // one 128 x D bf16 tile
    static constexpr int kQ = 0;                         // Q tile of group w at kQ + w tile
    static constexpr int kK0 = 2 * kTileBytes;           // stage s: K at kK0 + 2 s tile, V after it
    static constexpr int kStage = kTileBytes * (2 + 2 * kStages); // epilogue staging of group w at
                                                                  // kStage + w chunk (128 x 64 bf16)
    static constexpr int kBytes = kStage + 2 * kChunkBytes;
    static constexpr int kAlloc = kBytes + 1024;         // slack to align the base to 1024 B
    static constexpr int kThreads = 512;                 // four warpgroups
    // register budgets after the split: softmax warpgroups, epilogue warpgroup,
    // TMA / MMA warpgroup; 2 * 128 * compute + 128 * epi + 128 * other = 512 * 128
    static constexpr uint32_t kRegsCompute = D == 64 ? 168 : 184, kRegsEpi = 64, kRegsOther = D == 64 ? 112 : 80;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColO = 256;
};

// MXFP8 mode of the head_dim-128 layout (one softmax group, single query
// tiles): Q and K are E4M3 (one 16 KB chunk per 128 x 128 tile, in the bf16
// slots); the Q tile's scale words (a 128-row x 16-byte box: four heads' words
// per row) sit in group 1's Q slot, the K stages' boxes after it; the scale
// factors go to TMEM columns that group 1's S would use: A (the Q tile's) at
// 128..131, B (the K tile's) at 132..135.
struct FwdMx {
    static constexpr int kQScale = FwdLayout<128>::kQ + FwdLayout<128>::kTileBytes;
    static constexpr int kScaleBox = kTile * 16;
    static constexpr int kFp8TileBytes = kTile * 128;
    static constexpr uint32_t kColSFA = 128, kColSFB = 132;
};

struct FwdBarriers {
    uint64_t q_full[2], q_empty[2]; // query tile of group w, released after its last S
    uint64_t s_full[2], p_full[2], o_final[2], o_free[2];
    uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
    // group w's softmax is done with its item: inv_l[w] holds 1 / l. A group may finish its next
    // item (whose S needs nothing from the epilogue) before the epilogue has taken this one, so it
    // writes inv_l[w] and arrives on o_ready[w] only once the epilogue has read the previous value
    // (l_free[w]); o_ready[w] is then never two phases ahead of the epilogue's wait.
    uint64_t o_ready[2], l_free[2];
    uint32_t handed[8]; // per softmax warp: items handed to the epilogue (kept here, not in registers)
    uint64_t epi_sync;   // group barrier of the epilogue warpgroup
    uint64_t tail;       // the TMA warp's own barrier for a V tile whose last rows it clears
    uint64_t sf_ready;   // MXFP8: the item's scale factors (Q tile and first K tile) are in TMEM
    ItemRing ring;       // unused: this kernel deals its items statically (StaticItems)
    float inv_l[2][kTile];
    uint32_t tmem_base;
    int abort;
};

// Key-tile range of query tile t: [first_key_tile, t].
__device__ __forceinline__ int first_key_tile(int t, int64_t B, int64_t W)
{
    return int(window_start(int64_t(t) * kTile, B, W) / kTile);
}

} // namespace

// kFmaExp: one exponential pair in eight goes through the FMA pipe (the
// launcher's choice for long items; short ones keep every exponential on MUFU)
template <int D, int A, bool kCross, bool kMx, bool kFmaExp = true>
__global__ void __launch_bounds__(512, 1)
    fwd_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                          const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_ks,
                          const Problem p,
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
        mbar_init(&sb.q_empty[0], 1);
        mbar_init(&sb.q_full[1], 1);
        mbar_init(&sb.q_empty[1], 1);
        for (int w = 0; w < 2; ++w) {
            mbar_init(&sb.s_full[w], 1);
            mbar_init(&sb.p_full[w], 4);
            mbar_init(&sb.o_final[w], 1);
            mbar_init(&sb.o_free[w], 4);
            mbar_init(&sb.o_ready[w], 4);
            mbar_init(&sb.l_free[w], 4);
        }
        for (int i = 0; i < S; ++i) {
            mbar_init(&sb.k_full[i], 1);
            mbar_init(&sb.k_empty[i], 1);
            mbar_init(&sb.v_full[i], 1);
            mbar_init(&sb.v_empty[i], 1);
        }
        mbar_init(&sb.epi_sync, 128);
        mbar_init(&sb.tail, 1);
        mbar_init(&sb.sf_ready, 4);
        for (int i = 0; i < 8; ++i) sb.handed[i] = 0;
        sb.abort = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
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
    // MXFP8 mode walks single query tiles (one softmax group), the others pairs of them
    const int32_t nitems = kMx ? live_tile_count(p) : live_pair_count(p);
    const int4 *item_table = kMx ? p.tile_info : p.pair_info;
    static_assert(!kMx || (D == 128 && A == kSoftmax && !kCross), "MXFP8 mode: head_dim 128, softmax, self-attention");

    if (warp >= 8 && warp < 12) {
        // warps 8-11 (one warpgroup: TMA, MMA, two idle) hand registers to the softmax warpgroups
        warpgroup_regs_dec<Lay::kRegsOther>();
        if (warp == 8) {
            // ------------------------------------------------ TMA producer ---
            uint32_t kv_cnt = 0, item_cnt = 0, tail_phase = 0;
            uint32_t qcnt[2] = {0, 0}; // query tiles loaded per group
            TileRef r;
            bool second;
            bool ok = true;
            StaticItems items(item_table, nitems, p.heads, p.other_offsets);
            for (; ok && items.advance(r, sb.ring, abort, ok); ++item_cnt) {
                second = !kMx && pair_has_second(r);
                // cross-attention: every key tile of the example's own key/value set
                const int jlo = kCross ? 0 : first_key_tile(r.t, B, W);
                const int jhi = kCross ? (r.oL + kTile - 1) / kTile - 1 : r.t + (second ? 1 : 0);
                // each group's query tile as soon as that group's previous one is done with
                for (int w = 0; w < (second ? 2 : 1) && ok; ++w) {
                    if (!mbar_wait(&sb.q_empty[w], (qcnt[w] & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        if constexpr (kMx) { // E4M3 tile (128 bytes a row) and its rows' scale words
                            mbar_arrive_expect_tx(&sb.q_full[w], FwdMx::kFp8TileBytes + FwdMx::kScaleBox);
                            tma_load_2d(smem + Lay::kQ, &tm_q, &sb.q_full[w], r.h * D, r.s0 + r.t * kTile);
                            tma_load_2d(smem + FwdMx::kQScale, &tm_qs, &sb.q_full[w], (r.h / 4) * 16, r.s0 + r.t * kTile);
                        } else {
                            mbar_arrive_expect_tx(&sb.q_full[w], Lay::kTileBytes);
                            for (int c = 0; c < Lay::kChunks; ++c)
                                tma_load_2d(smem + Lay::kQ + w * Lay::kTileBytes + c * Lay::kChunkBytes, &tm_q,
                                            &sb.q_full[w], r.h * D + c * 64, r.s0 + (r.t + w) * kTile);
                        }
                    }
                    __syncwarp();
                    ++qcnt[w];
                }
                if (!ok) break;
                if (lane == 0) {
                    // warm L2 with the next item's query tiles
                    TileRef rn;
                    if (items.peek(rn)) {
                        const bool sn = !kMx && pair_has_second(rn);
                        for (int w = 0; w < (sn ? 2 : 1); ++w)
                            for (int c = 0; c < Lay::kChunks; ++c)
                                tma_prefetch_l2_2d(&tm_q, rn.h * D + c * 64, rn.s0 + (rn.t + w) * kTile);
                    }
                }
                __syncwarp();
                for (int j = jlo; j <= jhi; ++j, ++kv_cnt) {
                    const int st = kv_cnt % S;
                    uint8_t *kdst = smem + Lay::kK0 + 2 * st * Lay::kTileBytes;
                    // K and V of a stage are released separately (K after the tile's S products,
                    // V after its P V products), so each is refilled as soon as it is free
                    if (!mbar_wait(&sb.k_empty[st], ((kv_cnt / S) & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        if constexpr (kMx) {
                            mbar_arrive_expect_tx(&sb.k_full[st], FwdMx::kFp8TileBytes + FwdMx::kScaleBox);
                            tma_load_2d(kdst, &tm_k, &sb.k_full[st], r.h * D, r.os0 + j * kTile);
                            tma_load_2d(smem + FwdMx::kQScale + (1 + st) * FwdMx::kScaleBox, &tm_ks, &sb.k_full[st],
                                        (r.h / 4) * 16, r.os0 + j * kTile);
                        } else {
                            mbar_arrive_expect_tx(&sb.k_full[st], Lay::kTileBytes);
                            for (int c = 0; c < Lay::kChunks; ++c)
                                tma_load_2d(kdst + c * Lay::kChunkBytes, &tm_k, &sb.k_full[st], r.h * D + c * 64,
                                            r.os0 + j * kTile);
                        }
                    }
                    __syncwarp();
                    if (!mbar_wait(&sb.v_empty[st], ((kv_cnt / S) & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    // the example's last V tile: its rows past the example are cleared, since
                    // P V multiplies them by zero probabilities (K needs nothing: masked scores
                    // are replaced, not multiplied)
                    const int valid = r.oL - j * kTile;
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
            constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idesc_o = idesc_bf16(128, D, false, true);
            uint32_t kv_cnt = 0, item_cnt = 0;
            uint32_t pcnt[2] = {0, 0}; // P tiles consumed so far by each group
            uint32_t qf[2] = {0, 0};   // query tiles used up so far by each group
            uint32_t icnt[2] = {0, 0}; // items each group has finished (group 1 skips single-tile items)
            TileRef r;
            bool second;
            bool ok = true;
            StaticItems items(item_table, nitems, p.heads, p.other_offsets);
            for (; ok && items.advance(r, sb.ring, abort, ok); ++item_cnt) {
                second = !kMx && pair_has_second(r);
                const int nkt = (r.oL + kTile - 1) / kTile; // cross-attention: key tiles of the example
                const int lo[2] = {kCross ? 0 : first_key_tile(r.t, B, W),
                                   second ? (kCross ? 0 : first_key_tile(r.t + 1, B, W)) : 1};
                const int hi[2] = {kCross ? nkt - 1 : r.t, second ? (kCross ? nkt - 1 : r.t + 1) : 0};
                const int jlo = lo[0], jhi = second ? hi[1] : hi[0];
                // O_w += P_w V for key tile j of group w (V from ring stage st)
                auto issue_pv = [&](int w, int j, int st) -> bool {
                    if (!mbar_wait(&sb.p_full[w], pcnt[w] & 1, abort)) return false;
                    const bool first = (j == lo[w]);
                    if (first && !mbar_wait(&sb.o_free[w], (icnt[w] & 1) ^ 1, abort)) return false;
                    tc_fence_after();
                    {
                        const uint32_t v_addr = smem_base + Lay::kK0 + (2 * st + 1) * Lay::kTileBytes;
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_ts(tmem + Lay::kColO + D * w, tmem + 128 * w + kk * 8,
                                   sdesc_sw128(v_addr + kk * 2048, Lay::kChunkBytes, 1024), idesc_o,
                                   (!first || kk > 0) ? 1u : 0u);
                        if (j == hi[w]) tc_commit(&sb.o_final[w]);
                    }
                    __syncwarp();
                    ++pcnt[w];
                    return true;
                };
                auto issue_s = [&](int w, int j, int st) -> bool {
                    if (j == lo[w]) { // this group's query tile of the item
                        if (!mbar_wait(&sb.q_full[w], qf[w] & 1, abort)) return false;
                        // MXFP8: the softmax warps have put the item's scale factors in TMEM
                        if (kMx && !mbar_wait(&sb.sf_ready, qf[w] & 1, abort)) return false;
                        tc_fence_after();
                    }
                    {
                        const uint32_t q_addr = smem_base + Lay::kQ + w * Lay::kTileBytes;
                        const uint32_t k_addr = smem_base + Lay::kK0 + 2 * st * Lay::kTileBytes;
                        if constexpr (kMx) {
                            // four K = 32 products along head_dim, k-block kk scaled by byte kk of
                            // each row's scale word
#pragma unroll
                            for (uint32_t kk = 0; kk < 4; ++kk)
                                mma_mx_ss(tmem, sdesc_sw128(q_addr + kk * 32, 16, 1024),
                                          sdesc_sw128(k_addr + kk * 32, 16, 1024), idesc_mx_e4m3(128, 128, kk, kk),
                                          (tmem + FwdMx::kColSFA) | (kk << 30), (tmem + FwdMx::kColSFB) | (kk << 30),
                                          kk > 0 ? 1u : 0u);
                        } else {
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t off = (kk / 4) * Lay::kChunkBytes + (kk % 4) * 32;
                                mma_ss(tmem + 128 * w, sdesc_sw128(q_addr + off, 16, 1024),
                                       sdesc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                            }
                        }
                        tc_commit(&sb.s_full[w]);
                        if (j == hi[w]) tc_commit(&sb.q_empty[w]); // its last S: the tile may be replaced
                    }
                    __syncwarp();
                    if (j == hi[w]) ++qf[w];
                    return true;
                };
                // V of the previous key tile (ring position kv_cnt - 1) before its first P V
                auto wait_v_prev = [&]() -> bool {
                    const uint32_t pc = kv_cnt - 1;
                    if (!mbar_wait(&sb.v_full[pc % S], (pc / S) & 1, abort)) return false;
                    tc_fence_after();
                    return true;
                };
                for (int j = jlo; j <= jhi && ok; ++j, ++kv_cnt) {
                    const int st = kv_cnt % S;
                    if (!mbar_wait(&sb.k_full[st], (kv_cnt / S) & 1, abort) || (j > jlo && !wait_v_prev())) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int w = 0; w < 2 && ok; ++w) {
                        // the previous tile's P V of this group reads P from the S buffer: issue it first
                        if (j - 1 >= lo[w] && j - 1 <= hi[w] && !issue_pv(w, j - 1, (kv_cnt - 1) % S)) ok = false;
                        if (ok && j >= lo[w] && j <= hi[w] && !issue_s(w, j, st)) ok = false;
                    }
                    if (!ok) break;
                    {
                        tc_commit(&sb.k_empty[st]);                            // K of tile j: S products issued
                        if (j > jlo) tc_commit(&sb.v_empty[(kv_cnt - 1) % S]); // V of tile j-1: P V issued
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (!wait_v_prev()) break;
                for (int w = 0; w < 2 && ok; ++w)
                    if (jhi >= lo[w] && jhi <= hi[w] && !issue_pv(w, jhi, (kv_cnt - 1) % S)) ok = false;
                if (!ok) break;
                tc_commit(&sb.v_empty[(kv_cnt - 1) % S]);
                __syncwarp();
                ++icnt[0];
                if (second) ++icnt[1];
            }
        }
    } else if (warp < 8) {
        warpgroup_regs_inc<Lay::kRegsCompute>();
        // ----------------------------------------------------- softmax ---
        const int w = warp >> 2;              // group: query tile t + w
        const int row = threadIdx.x & 127;    // query row within the tile, TMEM lane
        const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
        const uint32_t s_addr = tmem + lane_base + 128 * w;
        const uint32_t o_addr = tmem + lane_base + Lay::kColO + D * w;
        const float scale_log2 = p.scale * 1.4426950408889634f;
        uint32_t cnt = 0; // tiles this group has processed
        uint32_t mx_items = 0;
        TileRef r;
        bool second;
        bool ok = true;
        // MXFP8: move the scale words of 128 rows (a TMA box of 16 bytes a row, this head's word
        // at 4 (h % 4)) into TMEM columns col .. col + 3 in the block-scaled MMA's layout: lane
        // l of every lane quarter holds, in column m, the word of row l + 32 m (byte k: k-block k)
        auto put_scales = [&](const uint8_t *box, uint32_t col, int head) {
            uint32_t wd[4];
#pragma unroll
            for (int m = 0; m < 4; ++m)
                wd[m] = *reinterpret_cast<const uint32_t *>(box + (lane + 32 * m) * 16 + (head % 4) * 4);
            tmem_st4(tmem + lane_base + col, wd);
        };
        StaticItems items(item_table, nitems, p.heads, p.other_offsets);
        while (ok && items.advance(r, sb.ring, abort, ok)) {
            second = !kMx && pair_has_second(r);
            if (w == 1 && !second) continue;
            if constexpr (kMx) {
                // the Q tile's and the first K tile's scale factors, before the item's first S
                const uint32_t st0 = cnt % S;
                if (!mbar_wait(&sb.q_full[0], mx_items & 1, abort) ||
                    !mbar_wait(&sb.k_full[st0], (cnt / S) & 1, abort)) {
                    ok = false;
                    break;
                }
                put_scales(smem + FwdMx::kQScale, FwdMx::kColSFA, r.h);
                put_scales(smem + FwdMx::kQScale + (1 + st0) * FwdMx::kScaleBox, FwdMx::kColSFB, r.h);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.sf_ready);
                ++mx_items;
            }
            const int t = r.t + w;
            const int jlo = kCross ? 0 : first_key_tile(t, B, W);
            const int jend = kCross ? (r.oL + kTile - 1) / kTile - 1 : t;
            const int64_t i = int64_t(t) * kTile + row;
            const bool valid = i < r.L;
            // visible keys [ws, last]: the block rule, or (cross-attention) the whole key/value set
            const int64_t ws = kCross ? 0 : window_start(i, B, W);
            const int64_t last = kCross ? int64_t(r.oL) - 1 : i;
            float m_ref = -INFINITY, l = 0.f;
            for (int j = jlo; j <= jend; ++j, ++cnt) {
                const int64_t key0 = int64_t(j) * kTile;
                int64_t lo64 = ws - key0, hi64 = last - key0;
                if (!valid) { lo64 = 1; hi64 = 0; }
                const int lo_c = int(lo64 < -1 ? -1 : (lo64 > 128 ? 128 : lo64));
                const int hi_c = int(hi64 < -1 ? -1 : (hi64 > 128 ? 128 : hi64));
                const bool full = __all_sync(0xffffffffu, lo_c <= 0 && hi_c >= 127);
                if (!mbar_wait(&sb.s_full[w], cnt & 1, abort)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, sr[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) reg_fence(sr[c]);
                // One pass for the row maximum of the visible raw scores (the scale is
                // positive), one for P; a tile visible to the whole warp skips masking.
                float alpha = 1.f, rs = 0.f;
                bool grow = false;
                // this row's visible columns [lo_c, hi_c] as four 32-bit masks (partial tiles only),
                // so that each column's test is one bit test
                uint32_t vis[4] = {0u, 0u, 0u, 0u};
                if (!full) {
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int lo = max(lo_c - 32 * w, 0), hi = min(hi_c - 32 * w, 31);
                        vis[w] = lo <= hi ? (0xffffffffu >> (31 - hi)) & (0xffffffffu << lo) : 0u;
                    }
                }
                auto softmax_tile = [&](auto full_t) {
                    constexpr bool FULL = decltype(full_t)::value;
                    float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < 128; c += 2) {
                        float a = __uint_as_float(sr[c / 32][c % 32]), b = __uint_as_float(sr[c / 32][c % 32 + 1]);
                        if (!FULL) {
                            a = (vis[c / 32] & (1u << (c % 32))) ? a : -INFINITY;
                            b = (vis[c / 32] & (1u << (c % 32 + 1))) ? b : -INFINITY;
                            sr[c / 32][c % 32] = __float_as_uint(a);
                            sr[c / 32][c % 32 + 1] = __float_as_uint(b);
                        }
                        mp[(c / 2) % 4] = fmax3(mp[(c / 2) % 4], a, b);
                    }
                    const float mx = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
                    const float m_new = mx * scale_log2;
                    grow = m_new > m_ref + 8.0f;
                    if (grow) {
                        alpha = ex2_approx(m_ref - m_new);
                        m_ref = m_new;
                    }
                    const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
                    const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(neg_m, neg_m);
                    float2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
                    // P in two 64-column halves, each stored (packed bf16) over S columns
                    // this thread has already read
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t pk[32];
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int c0 = 64 * hh + 2 * c;
                            const float2 x = ffma2(make_float2(__uint_as_float(sr[c0 / 32][c0 % 32]),
                                                               __uint_as_float(sr[c0 / 32][c0 % 32 + 1])),
                                                   sc2, nm2);
                            // with kFmaExp one pair in eight goes through the FMA pipe to offload MUFU
                            float p0 = (kFmaExp && c % 8 == 7) ? exp2_fma(x.x) : ex2_approx(x.x);
                            float p1 = (kFmaExp && c % 8 == 7) ? exp2_fma(x.y) : ex2_approx(x.y);
                            // masked scores are -inf here and ex2.approx(-inf) is 0; only the
                            // FMA-pipe form (which floors x at -125) needs them zeroed again
                            if (!FULL && kFmaExp && c % 8 == 7) {
                                p0 = x.x > -INFINITY ? p0 : 0.f;
                                p1 = x.y > -INFINITY ? p1 : 0.f;
                            }
                            acc[c % 4] = fadd2(acc[c % 4], make_float2(p0, p1));
                            pk[c] = pack_bf16x2(p0, p1);
                        }
                        tmem_st32(s_addr + 32 * hh, pk);
                    }
                    const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
                    const float2 a = fadd2(a01, a23);
                    rs = a.x + a.y;
                };
                // generalized attention: P = act(S / sqrt(D)) on the visible keys, nothing to normalise
                auto activation_tile = [&](auto full_t) {
                    constexpr bool FULL = decltype(full_t)::value;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t pk[32];
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int c0 = 64 * hh + 2 * c;
                            float p0 = 0.f, p1 = 0.f;
                            if constexpr (A != kSoftmax) {
                                p0 = act_value<A>(__uint_as_float(sr[c0 / 32][c0 % 32]) * p.scale);
                                p1 = act_value<A>(__uint_as_float(sr[c0 / 32][c0 % 32 + 1]) * p.scale);
                            }
                            if (!FULL) {
                                p0 = (vis[c0 / 32] & (1u << (c0 % 32))) ? p0 : 0.f;
                                p1 = (vis[c0 / 32] & (1u << (c0 % 32 + 1))) ? p1 : 0.f;
                            }
                            pk[c] = pack_bf16x2(p0, p1);
                        }
                        tmem_st32(s_addr + 32 * hh, pk);
                    }
                };
                if constexpr (A != kSoftmax) {
                    if (full) activation_tile(std::true_type{});
                    else activation_tile(std::false_type{});
                } else if (full) softmax_tile(std::true_type{});
                else softmax_tile(std::false_type{});
                l = l * alpha + rs;
                tmem_wait_st();
                // O holds the earlier tiles' P V (complete: this S was issued after it).
                if (A == kSoftmax && j > jlo && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t orr[32];
                        tmem_ld32(o_addr + c * 32, orr);
                        tmem_wait_ld();
                        reg_fence(orr);
#pragma unroll
                        for (int k = 0; k < 32; ++k) orr[k] = __float_as_uint(__uint_as_float(orr[k]) * alpha);
                        tmem_st32(o_addr + c * 32, orr);
                    }
                    tmem_wait_st();
                }
                if constexpr (kMx) {
                    // the next K tile's scale factors go to TMEM before P is released: the MMA warp
                    // issues that tile's S right after this tile's P V
                    if (j < jend) {
                        const uint32_t st1 = (cnt + 1) % S;
                        if (!mbar_wait(&sb.k_full[st1], ((cnt + 1) / S) & 1, abort)) { ok = false; break; }
                        put_scales(smem + FwdMx::kQScale + (1 + st1) * FwdMx::kScaleBox, FwdMx::kColSFB, r.h);
                        tmem_wait_st();
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.p_full[w]);
            }
            if (!ok) break;
            // hand 1 / l to the epilogue warps (once they have read the previous item's), write lse,
            // and go on with the next item
            const uint32_t gi = sb.handed[warp];
            if (!mbar_wait(&sb.l_free[w], (gi & 1) ^ 1, abort)) { ok = false; break; }
            if constexpr (A == kSoftmax) {
                sb.inv_l[w][row] = valid ? 1.f / l : 0.f;
                if (valid)
                    lse[int64_t(r.h) * p.total_tokens + r.s0 + i] = (m_ref + log2f(l)) * 0.6931471805599453f;
            } else {
                sb.inv_l[w][row] = valid ? 1.f : 0.f;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sb.o_ready[w]);
                sb.handed[warp] = gi + 1;
            }
        }
    } else {
        warpgroup_regs_dec<Lay::kRegsEpi>();
        // ---------------------------------------------------- epilogue ---
        // Per item and group: wait for the softmax (1 / l) and the last P V, then
        // normalise O and store it. A tile whose rows all belong to the example
        // leaves through the two staging buffers (alternating) and TMA stores; the
        // example's last tile is stored row by row.
        const int row = threadIdx.x & 127;    // query row within the tile, TMEM lane
        const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
        const bool leader = threadIdx.x == 384;
        uint32_t done[2] = {0, 0}, sync_phase = 0, nstored = 0;
        TileRef r;
        bool ok = true;
        StaticItems items(item_table, nitems, p.heads, p.other_offsets);
        while (ok && items.advance(r, sb.ring, abort, ok)) {
            const bool second = !kMx && pair_has_second(r);
            for (int w = 0; w < (second ? 2 : 1) && ok; ++w) {
                // 1 / l first, released at once so the softmax may write the next item's, then
                // the item's last P V
                if (!mbar_wait(&sb.o_ready[w], done[w] & 1, abort)) {
                    ok = false;
                    break;
                }
                const float inv_l = sb.inv_l[w][row];
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.l_free[w]);
                if (!mbar_wait(&sb.o_final[w], done[w] & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                ++done[w];
                const int t = r.t + w;
                const int64_t i = int64_t(t) * kTile + row;
                const bool valid = i < r.L;
                const bool full_tile = int64_t(t) * kTile + kTile <= r.L;
                const uint32_t o_addr = tmem + lane_base + Lay::kColO + D * w;
                __nv_bfloat16 *orow = out + ((int64_t(r.s0) + i) * p.heads + r.h) * D;
#pragma unroll 1
                for (int c = 0; c < D / 64; ++c) {
                    uint8_t *stage = smem + Lay::kStage + (nstored & 1) * Lay::kChunkBytes;
                    if (full_tile) {
                        if (leader) bulk_wait_group_read<1>(); // this buffer's previous store has left it
                        if (!group_sync(&sb.epi_sync, sync_phase, abort)) { ok = false; break; }
                    }
                    // 32 columns at a time: normalise, pack, and put them in the staging row
                    // (or straight into the output row for the example's last tile)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t orr[32];
                        tmem_ld32(o_addr + 64 * c + 32 * hh, orr);
                        tmem_wait_ld();
                        reg_fence(orr);
                        if (c == D / 64 - 1 && hh == 1) { // all of O read: the next item's P V may overwrite it
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&sb.o_free[w]);
                        }
                        uint32_t pk[16];
#pragma unroll
                        for (int x = 0; x < 16; ++x)
                            pk[x] = pack_bf16x2(__uint_as_float(orr[2 * x]) * inv_l,
                                                __uint_as_float(orr[2 * x + 1]) * inv_l);
                        if (full_tile) {
                            uint8_t *srow = stage + row * 128;
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                *reinterpret_cast<uint4 *>(srow + (((4 * hh + u) ^ (row & 7)) << 4)) =
                                    make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                        } else if (valid) {
                            uint4 *dst = reinterpret_cast<uint4 *>(orow + 64 * c + 32 * hh);
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                        }
                    }
                    if (full_tile) {
                        fence_proxy_async_smem();
                        if (!group_sync(&sb.epi_sync, sync_phase, abort)) { ok = false; break; }
                        if (leader) {
                            tma_store_2d(&tm_o, stage, r.h * D + 64 * c, r.s0 + t * kTile);
                            bulk_commit_group();
                        }
                        ++nstored;
                    }
                }
            }
        }
        if (leader) bulk_wait_group<0>();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, Lay::kTmemCols);
    if (threadIdx.x == 0 && sb.abort) atomicOr(p.status, kStatusTimeout);
}

template <int D, int A>
cudaError_t launch_fwd_bf16_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const CUtensorMap &to, const Problem &p, void *out, float *lse, int num_sms,
                                  cudaStream_t stream, const CUtensorMap *tqs, const CUtensorMap *tks)
{
    using Lay = FwdLayout<D>;
    // cross-attention exists for the generalized attention only, the MXFP8 mode (scale maps
    // given) for block attention at head_dim 128
    constexpr bool kCanMx = D == 128 && A == kSoftmax;
    const bool mx = kCanMx && tqs && tks;
    if (!kCanMx && (tqs || tks)) return cudaErrorInvalidValue;
    auto kern = mx ? fwd_bf16_sm100_kernel<D, A, false, kCanMx>
                   : (A != kSoftmax && p.other_offsets) ? fwd_bf16_sm100_kernel<D, A, A != kSoftmax, false>
                                                        : fwd_bf16_sm100_kernel<D, A, false, false>;
    if constexpr (A == kSoftmax) {
        // Items that see fewer than 1024 keys (block x window) are short: their softmax warps are
        // bound by instruction issue, and MUFU's one-instruction 2^x beats the FMA-pipe form's nine
        // (measured: config-3 forward 4% faster; with 16-tile items the 1-in-8 mix is 3% faster).
        if (!mx && int64_t(p.block) * p.window < 1024) kern = fwd_bf16_sm100_kernel<D, A, false, false, false>;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess) return e;
    // the register split only works if the CTA is launched with at least the budgets' sum
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * Lay::kThreads < int(256 * Lay::kRegsCompute + 128 * Lay::kRegsEpi + 128 * Lay::kRegsOther))
        return cudaErrorInvalidConfiguration;
    kern<<<num_sms, Lay::kThreads, Lay::kAlloc, stream>>>(tq, tk, tv, to, mx ? *tqs : tq, mx ? *tks : tk, p,
                                                          static_cast<__nv_bfloat16 *>(out), lse);
    return cudaGetLastError();
}

#define BA_FWD_INST(D, A)                                                                                  \
    template cudaError_t launch_fwd_bf16_sm100<D, A>(const CUtensorMap &, const CUtensorMap &,              \
                                                     const CUtensorMap &, const CUtensorMap &, const Problem &, \
                                                     void *, float *, int, cudaStream_t, const CUtensorMap *,   \
                                                     const CUtensorMap *);
BA_FWD_INST(64, kSoftmax)
BA_FWD_INST(128, kSoftmax)
BA_FWD_INST(64, kGelu)
BA_FWD_INST(128, kGelu)
BA_FWD_INST(64, kSilu)
BA_FWD_INST(128, kSilu)

} // namespace ba
