// Small memory-bound kernels around the attention kernels:
//   worklist_kernel   the persistent kernels' work list: every live 128-row
//                     tile (and pair of tiles), examples longest first; resets
//                     the status word
//   stage_query_tails_kernel  the last, partial query tile of each example
//                     (q and dout), zero-padded, for the dK/dV pass
//   bwd_pre_kernel    Delta = rowsum(dout * out) in fp32 (the fp32 path; the
//                     bf16 dQ pass computes Delta itself)
//   bwd_stats_kernel  -Delta and -lse log2(e) per row for the fused bf16
//                     backward (masks whose query tiles see only their own
//                     key tile), which has no dQ pass
//   wait_selftest_kernel  one warp waits on a barrier nothing completes, with a
//                     short limit, through the same bounded wait the attention
//                     kernels use, and reports the timeout in the status word
//   exp2_selftest_kernel  the forward's FMA-pipe 2^x on a caller's array
//                     (its accuracy is tested against 2^x computed on the host)
//   activation_selftest_kernel  the generalized attention's GELU / SiLU and
//                     their derivatives on a caller's array (tested likewise)
//   skip_*_kernel     component skip: flagged examples pass v through
//                     ("Meta Scales GEM Ads Model Across Platforms and
//                     Thousands of GPUs", section "Kunlun changes how GEM
//                     scales": sequence modules bypassed selectively)
#include "ba_common.cuh"
#include "ba_kernels.cuh"
#include "ba_ptx.cuh"
#include "ba_sched.cuh"

#include <cuda_bf16.h>

namespace ba {

namespace {

// Live 128-row tiles of example b: none if it is skipped, or (cross-attention)
// if its other side is empty.
__device__ __forceinline__ int32_t live_tiles(const int32_t *offs, const uint8_t *skip, const int32_t *other,
                                              int32_t b)
{
    if (skip && skip[b]) return 0;
    if (other && other[b + 1] == other[b]) return 0;
    const int32_t L = offs[b + 1] - offs[b];
    return L > 0 ? (L + kTile - 1) / kTile : 0;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

} // namespace

// Exclusive block-wide scan of one value per thread; returns the prefix and
// stores the total in *total (read after the call's final barrier).
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t local, int32_t *warp_tot, int32_t &total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int32_t incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += y;
    }
    __syncthreads();
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int32_t w = warp_tot[lane];
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, w, d);
            if (lane >= d) w += y;
        }
        warp_tot[lane] = w; // inclusive over warps
    }
    __syncthreads();
    total = warp_tot[kWorklistThreads / 32 - 1];
    return incl - local + (wid > 0 ? warp_tot[wid - 1] : 0);
}

// The persistent kernels deal their work items out round-robin (item n to CTA
// n mod grid) in table order. The table lists examples longest first, each
// example's tiles together and in order: the long examples' items, which see
// the most key tiles, go out first and the short examples' cheap ones fill in
// at the end, so the CTAs finish close together (longest-processing-time-first
// dealing), while the tiles of one example, which share K/V tiles, still run
// at about the same time. Examples are bucketed by their live tile count
// (counts of kSortBuckets - 1 and more share the first bucket); the order
// inside a bucket is whatever order the examples claim their slots in.
constexpr int kSortBuckets = kWorklistThreads;

// Per live example: its 128-row tiles, and pairs of consecutive tiles (the
// forward processes two query tiles of one example together).
__global__ void __launch_bounds__(kWorklistThreads)
    worklist_kernel(const int32_t *__restrict__ offs, const uint8_t *__restrict__ skip,
                    const int32_t *__restrict__ other, int32_t batch, int32_t *__restrict__ tile_prefix,
                    int4 *__restrict__ tile_info, int32_t *__restrict__ pair_prefix, int4 *__restrict__ pair_info,
                    int *__restrict__ status, int reset_status)
{
    __shared__ int32_t warp_tot[kWorklistThreads / 32];
    __shared__ int32_t bucket_tiles[kSortBuckets], bucket_pairs[kSortBuckets];
    const int tid = threadIdx.x;
    auto bucket = [](int32_t nt) { return kSortBuckets - 1 - (nt < kSortBuckets - 1 ? nt : kSortBuckets - 1); };
    bucket_tiles[tid] = 0;
    bucket_pairs[tid] = 0;
    __syncthreads();
    for (int b = tid; b < batch; b += kWorklistThreads) {
        const int32_t nt = live_tiles(offs, skip, other, b);
        if (nt == 0) continue;
        atomicAdd(&bucket_tiles[bucket(nt)], nt);
        atomicAdd(&bucket_pairs[bucket(nt)], (nt + 1) / 2);
    }
    __syncthreads();
    int32_t ttot, ptot;
    const int32_t tstart = block_exclusive_scan(bucket_tiles[tid], warp_tot, ttot);
    const int32_t pstart = block_exclusive_scan(bucket_pairs[tid], warp_tot, ptot);
    bucket_tiles[tid] = tstart; // every thread read its bucket before the scans' barriers
    bucket_pairs[tid] = pstart;
    __syncthreads();
    for (int b = tid; b < batch; b += kWorklistThreads) {
        const int32_t nt = live_tiles(offs, skip, other, b);
        const int32_t s0 = offs[b], L = offs[b + 1] - s0;
        int32_t t0 = ttot, p0 = ptot; // an example without live tiles owns no slots
        if (nt > 0) {
            t0 = atomicAdd(&bucket_tiles[bucket(nt)], nt);
            p0 = atomicAdd(&bucket_pairs[bucket(nt)], (nt + 1) / 2);
        }
        tile_prefix[b] = t0;
        pair_prefix[b] = p0;
        for (int32_t t = 0; t < nt; ++t) tile_info[t0 + t] = make_int4(s0, L, t, b);
        for (int32_t t = 0; t < nt; t += 2) pair_info[p0 + t / 2] = make_int4(s0, L, t, b);
    }
    if (tid == kWorklistThreads - 1) {
        tile_prefix[batch] = ttot;
        pair_prefix[batch] = ptot;
        if (reset_status) *status = 0;
        // the attention kernels' item counters (one per kernel of a call)
        for (int c = kCounterFwd; c <= kCounterDkdv; ++c) status[c] = 0;
    }
}

// One warp per (token, head) row.
template <typename T, int D>
__global__ void __launch_bounds__(256)
    bwd_pre_kernel(const T *__restrict__ out, const T *__restrict__ dout, int32_t total_tokens,
                   int32_t heads, float *__restrict__ delta)
{
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t nrows = int64_t(total_tokens) * heads;
    const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t rw = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); rw < nrows; rw += wstride) {
        const int64_t t = rw / heads, h = rw % heads;
        const T *o = out + rw * D + lane * PER;
        const T *g = dout + rw * D + lane * PER;
        float acc = 0.f;
#pragma unroll
        for (int x = 0; x < PER; ++x) acc += to_f32(o[x]) * to_f32(g[x]);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, d);
        const int64_t hr = h * total_tokens + t;
        if (lane == 0) delta[hr] = acc;
    }
}

// Forward skip: out = v and lse = 0 for flagged examples. grid.x = example,
// grid.y splits the example's contiguous rows.
__global__ void __launch_bounds__(256)
    skip_fwd_kernel(const int32_t *__restrict__ offs, const uint8_t *__restrict__ skip, int32_t heads,
                    int32_t total_tokens, int64_t row_bytes, const uint8_t *__restrict__ v,
                    uint8_t *__restrict__ out, float *__restrict__ lse)
{
    const int b = blockIdx.x;
    if (!skip[b]) return;
    const int64_t s0 = offs[b], L = offs[b + 1] - s0;
    if (L <= 0) return;
    const int64_t nvec = L * row_bytes / 16; // rows are whole multiples of 16 bytes
    const uint4 *src = reinterpret_cast<const uint4 *>(v + s0 * row_bytes);
    uint4 *dst = reinterpret_cast<uint4 *>(out + s0 * row_bytes);
    const int64_t stride = int64_t(gridDim.y) * blockDim.x;
    for (int64_t x = int64_t(blockIdx.y) * blockDim.x + threadIdx.x; x < nvec; x += stride) dst[x] = src[x];
    for (int64_t x = int64_t(blockIdx.y) * blockDim.x + threadIdx.x; x < L * heads; x += stride)
        lse[(x / L) * total_tokens + s0 + x % L] = 0.f;
}

// Backward skip: dk = 0 and dv = dout for flagged examples; dq = 0 too when
// `dq` is given (the bf16 path instead gets 0 from its zeroed accumulator,
// since no tile of a flagged example is scheduled).
__global__ void __launch_bounds__(256)
    skip_bwd_kernel(const int32_t *__restrict__ offs, const uint8_t *__restrict__ skip, int64_t row_bytes,
                    const uint8_t *__restrict__ dout, uint8_t *__restrict__ dq, uint8_t *__restrict__ dk,
                    uint8_t *__restrict__ dv)
{
    const int b = blockIdx.x;
    if (!skip[b]) return;
    const int64_t s0 = offs[b], L = offs[b + 1] - s0;
    if (L <= 0) return;
    const int64_t nvec = L * row_bytes / 16;
    const uint4 *src = reinterpret_cast<const uint4 *>(dout + s0 * row_bytes);
    uint4 *dvv = reinterpret_cast<uint4 *>(dv + s0 * row_bytes);
    uint4 *dkv = reinterpret_cast<uint4 *>(dk + s0 * row_bytes);
    const int64_t stride = int64_t(gridDim.y) * blockDim.x;
    uint4 *dqv = dq ? reinterpret_cast<uint4 *>(dq + s0 * row_bytes) : nullptr;
    for (int64_t x = int64_t(blockIdx.y) * blockDim.x + threadIdx.x; x < nvec; x += stride) {
        dvv[x] = src[x];
        dkv[x] = make_uint4(0, 0, 0, 0);
        if (dqv) dqv[x] = make_uint4(0, 0, 0, 0);
    }
}

// ---------------------------------------------------------------- launchers

cudaError_t launch_worklist(const Problem &p, cudaStream_t stream, bool reset_status)
{
    worklist_kernel<<<1, kWorklistThreads, 0, stream>>>(
        p.seq_offsets, p.skip, p.other_offsets, p.batch, const_cast<int32_t *>(p.tile_prefix),
        const_cast<int4 *>(p.tile_info), const_cast<int32_t *>(p.pair_prefix), const_cast<int4 *>(p.pair_info),
        p.status, reset_status ? 1 : 0);
    return cudaGetLastError();
}

// Cross-attention: rows of examples whose other side is empty get zeros (an
// empty sum) in a and, when given, b. grid.x = example.
__global__ void __launch_bounds__(256)
    zero_unpaired_rows_kernel(const int32_t *__restrict__ offs, const int32_t *__restrict__ other, int64_t row_bytes,
                              uint8_t *__restrict__ a, uint8_t *__restrict__ b)
{
    const int e = blockIdx.x;
    if (other[e + 1] != other[e]) return;
    const int64_t s0 = offs[e], L = offs[e + 1] - s0;
    const int64_t nvec = L * row_bytes / 16;
    uint4 *av = reinterpret_cast<uint4 *>(a + s0 * row_bytes);
    uint4 *bv = b ? reinterpret_cast<uint4 *>(b + s0 * row_bytes) : nullptr;
    const int64_t stride = int64_t(gridDim.y) * blockDim.x;
    for (int64_t x = int64_t(blockIdx.y) * blockDim.x + threadIdx.x; x < nvec; x += stride) {
        av[x] = make_uint4(0, 0, 0, 0);
        if (bv) bv[x] = make_uint4(0, 0, 0, 0);
    }
}

cudaError_t launch_zero_unpaired_rows(const int32_t *offs, const int32_t *other, int32_t batch, size_t row_bytes,
                                      void *a, void *b, cudaStream_t stream)
{
    if (batch == 0) return cudaSuccess;
    zero_unpaired_rows_kernel<<<dim3(batch, 8), 256, 0, stream>>>(offs, other, int64_t(row_bytes),
                                                                 static_cast<uint8_t *>(a), static_cast<uint8_t *>(b));
    return cudaGetLastError();
}

// The dK/dV pass's partial query tiles: example b's last query tile, when it
// has fewer than 128 rows, is copied from a (q) and b (dout) to rows
// [128 b, 128 b + 128) of ta and tb with zeros in the rows past the example,
// so that the pass never multiplies a neighbour's rows, finite or not, by its
// zero probabilities. The fused backward also stages c (k) into tc, since its
// dQ = dS K sums over the partial key tile's rows. Examples whose length is a
// multiple of 128 (or zero) or that are skipped are left alone. grid =
// (example, 8 slices of 16 rows).
__global__ void __launch_bounds__(256)
    stage_query_tails_kernel(const int32_t *__restrict__ offs, const uint8_t *__restrict__ skip, int64_t row_bytes,
                             const uint8_t *__restrict__ a, const uint8_t *__restrict__ b,
                             const uint8_t *__restrict__ c, uint8_t *__restrict__ ta, uint8_t *__restrict__ tb,
                             uint8_t *__restrict__ tc)
{
    const int e = blockIdx.x;
    if (skip && skip[e]) return;
    const int64_t L = offs[e + 1] - offs[e];
    const int64_t valid = L % kTile;
    if (valid == 0) return;
    const int64_t first = offs[e] + (L - valid); // first row of the partial tile
    const int64_t units = row_bytes / 16;        // 16-byte units per row
    const int64_t r0 = int64_t(blockIdx.y) * (kTile / 8);
    for (int64_t x = threadIdx.x; x < (kTile / 8) * units; x += blockDim.x) {
        const int64_t r = r0 + x / units, u = x % units;
        const int64_t dst = (int64_t(e) * kTile + r) * units + u;
        uint4 va = make_uint4(0, 0, 0, 0), vb = va, vc = va;
        if (r < valid) {
            va = reinterpret_cast<const uint4 *>(a)[(first + r) * units + u];
            vb = reinterpret_cast<const uint4 *>(b)[(first + r) * units + u];
            if (c) vc = reinterpret_cast<const uint4 *>(c)[(first + r) * units + u];
        }
        reinterpret_cast<uint4 *>(ta)[dst] = va;
        reinterpret_cast<uint4 *>(tb)[dst] = vb;
        if (c) reinterpret_cast<uint4 *>(tc)[dst] = vc;
    }
}

cudaError_t launch_stage_query_tails(const int32_t *offs, const uint8_t *skip, int32_t batch, size_t row_bytes,
                                     const void *a, const void *b, void *ta, void *tb, cudaStream_t stream,
                                     const void *c, void *tc)
{
    if (batch == 0) return cudaSuccess;
    if ((c == nullptr) != (tc == nullptr)) return cudaErrorInvalidValue;
    stage_query_tails_kernel<<<dim3(batch, 8), 256, 0, stream>>>(
        offs, skip, int64_t(row_bytes), static_cast<const uint8_t *>(a), static_cast<const uint8_t *>(b),
        static_cast<const uint8_t *>(c), static_cast<uint8_t *>(ta), static_cast<uint8_t *>(tb),
        static_cast<uint8_t *>(tc));
    return cudaGetLastError();
}

// The fused backward's per-row statistics, which the dQ pass computes
// otherwise: -Delta = -(dout . out) and -lse log2(e) of every (token, head)
// row, written [heads, total_tokens]. One warp per (head, 32 consecutive
// tokens): D / 8 lanes per token row, one 16-byte vector of each operand per
// lane, and each output written as one 128-byte line. Rows of skipped
// examples are computed too (nothing reads them).
__device__ __forceinline__ float bf16x8_dot(const uint4 a, const uint4 b)
{
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&aw[e]));
        const float2 bf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&bw[e]));
        acc.x = fmaf(af.x, bf.x, acc.x);
        acc.y = fmaf(af.y, bf.y, acc.y);
    }
    return acc.x + acc.y;
}

template <int D>
__global__ void __launch_bounds__(256)
    bwd_stats_kernel(const __nv_bfloat16 *__restrict__ out, const __nv_bfloat16 *__restrict__ dout,
                     const float *__restrict__ lse, int32_t total_tokens, int32_t heads,
                     float *__restrict__ neg_delta, float *__restrict__ nlse2)
{
    constexpr int LPR = D / 8;      // lanes per row: one 16-byte vector each
    constexpr int RPS = 32 / LPR;   // rows per load step
    constexpr int STEPS = 32 / RPS; // load steps per task of 32 tokens
    const int lane = threadIdx.x & 31, u = lane % LPR, sub = lane / LPR;
    const int64_t T = total_tokens;
    const int64_t ntasks = (T + 31) / 32 * heads;
    const int64_t rs = int64_t(heads) * D; // elements from one token's row of a head to the next token's
    // task = (32-token block, head), heads fastest: the warps of one token block read whole token rows
    for (int64_t task = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); task < ntasks;
         task += int64_t(gridDim.x) * (blockDim.x >> 5)) {
        const int64_t tb = task / heads, h = task - tb * heads, t0 = tb * 32;
        float mine = 0.f; // lane j ends with token t0 + j's dout . out
#pragma unroll 4
        for (int k = 0; k < STEPS; ++k) {
            const int64_t t = t0 + k * RPS + sub;
            float sum = 0.f;
            if (t < T) {
                const uint4 o4 = __ldg(reinterpret_cast<const uint4 *>(out + t * rs + h * D) + u);
                const uint4 g4 = __ldg(reinterpret_cast<const uint4 *>(dout + t * rs + h * D) + u);
                sum = bf16x8_dot(o4, g4);
            }
#pragma unroll
            for (int d = LPR / 2; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
            // token t0 + j was row j % RPS of step j / RPS, whose sum sits in lanes (j % RPS) * LPR ..
            const float b = __shfl_sync(0xffffffffu, sum, (lane % RPS) * LPR);
            if (lane / RPS == k) mine = b;
        }
        const int64_t t = t0 + lane;
        if (t < T) {
            const int64_t hr = h * T + t;
            neg_delta[hr] = -mine;
            nlse2[hr] = -lse[hr] * 1.4426950408889634f;
        }
    }
}

static int grid_for_rows(int64_t nrows, int num_sms)
{
    const int64_t warps = 8; // per 256-thread block
    int64_t g = (nrows + warps - 1) / warps;
    const int64_t cap = int64_t(num_sms) * 16;
    if (g > cap) g = cap;
    return int(g < 1 ? 1 : g);
}

cudaError_t launch_bwd_stats(const Problem &p, const void *out, const void *dout, const float *lse,
                             float *neg_delta, float *nlse2, int num_sms, cudaStream_t stream)
{
    const int64_t ntasks = (int64_t(p.total_tokens) + 31) / 32 * p.heads; // warps' tasks
    if (ntasks == 0) return cudaSuccess;
    const int g = grid_for_rows(ntasks, num_sms); // one task per warp, 8 warps per block, capped
    const auto *o = static_cast<const __nv_bfloat16 *>(out), *d = static_cast<const __nv_bfloat16 *>(dout);
    switch (p.head_dim) {
    case 64:
        bwd_stats_kernel<64><<<g, 256, 0, stream>>>(o, d, lse, p.total_tokens, p.heads, neg_delta, nlse2);
        break;
    case 128:
        bwd_stats_kernel<128><<<g, 256, 0, stream>>>(o, d, lse, p.total_tokens, p.heads, neg_delta, nlse2);
        break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd_pre(const Problem &p, const void *out, const void *dout, float *delta, int num_sms,
                           cudaStream_t stream)
{
    const int64_t nrows = int64_t(p.total_tokens) * p.heads;
    if (nrows == 0) return cudaSuccess;
    const int g = grid_for_rows(nrows, num_sms);
    const T *o = static_cast<const T *>(out), *d = static_cast<const T *>(dout);
    switch (p.head_dim) {
    case 32: bwd_pre_kernel<T, 32><<<g, 256, 0, stream>>>(o, d, p.total_tokens, p.heads, delta); break;
    case 64: bwd_pre_kernel<T, 64><<<g, 256, 0, stream>>>(o, d, p.total_tokens, p.heads, delta); break;
    case 128: bwd_pre_kernel<T, 128><<<g, 256, 0, stream>>>(o, d, p.total_tokens, p.heads, delta); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_skip_fwd(const Problem &p, size_t elem_bytes, const void *v, void *out, float *lse,
                            cudaStream_t stream)
{
    if (!p.skip || p.batch == 0) return cudaSuccess;
    const int64_t row_bytes = int64_t(p.heads) * p.head_dim * elem_bytes;
    skip_fwd_kernel<<<dim3(p.batch, 8), 256, 0, stream>>>(p.seq_offsets, p.skip, p.heads, p.total_tokens,
                                                         row_bytes, static_cast<const uint8_t *>(v),
                                                         static_cast<uint8_t *>(out), lse);
    return cudaGetLastError();
}

cudaError_t launch_skip_bwd(const Problem &p, size_t elem_bytes, const void *dout, void *dq, void *dk,
                            void *dv, cudaStream_t stream)
{
    if (!p.skip || p.batch == 0) return cudaSuccess;
    const int64_t row_bytes = int64_t(p.heads) * p.head_dim * elem_bytes;
    skip_bwd_kernel<<<dim3(p.batch, 8), 256, 0, stream>>>(p.seq_offsets, p.skip, row_bytes,
                                                         static_cast<const uint8_t *>(dout),
                                                         static_cast<uint8_t *>(dq), static_cast<uint8_t *>(dk),
                                                         static_cast<uint8_t *>(dv));
    return cudaGetLastError();
}

__global__ void __launch_bounds__(32) wait_selftest_kernel(int *status, uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort = 0;
        fence_mbar_init();
    }
    __syncwarp();
    // nothing ever arrives on `bar`
    if (!mbar_wait(&bar, 0, &abort, limit_ns) && threadIdx.x == 0) atomicOr(status, kStatusTimeout);
}

cudaError_t launch_wait_selftest(int *status, uint64_t limit_ns, cudaStream_t stream)
{
    wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256) exp2_selftest_kernel(const float *__restrict__ x, float *__restrict__ y, int64_t n)
{
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
        y[i] = exp2_fma(x[i]);
}

cudaError_t launch_exp2_selftest(const float *x, float *y, int64_t n, cudaStream_t stream)
{
    if (n == 0) return cudaSuccess;
    const int64_t g = (n + 255) / 256;
    exp2_selftest_kernel<<<int(g < 4096 ? g : 4096), 256, 0, stream>>>(x, y, n);
    return cudaGetLastError();
}

// The generalized attention's activation A on a caller's array: y = act(x)
// and dy = act'(x) through the same device functions the kernels use.
template <int A>
__global__ void __launch_bounds__(256)
    activation_selftest_kernel(const float *__restrict__ x, float *__restrict__ y, float *__restrict__ dy, int64_t n)
{
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        const float2 vg = act_value_grad<A>(x[i]);
        // the kernels call all three forms; they must agree bit for bit
        const bool same = __float_as_uint(vg.x) == __float_as_uint(act_value<A>(x[i])) &&
                          __float_as_uint(vg.y) == __float_as_uint(act_grad<A>(x[i]));
        y[i] = vg.x;
        dy[i] = same ? vg.y : __int_as_float(0x7fc00000); // a disagreement shows as NaN
    }
}

cudaError_t launch_activation_selftest(int act, const float *x, float *y, float *dy, int64_t n, cudaStream_t stream)
{
    if (n == 0) return cudaSuccess;
    const int64_t g = (n + 255) / 256;
    const int grid = int(g < 4096 ? g : 4096);
    if (act == kGelu) activation_selftest_kernel<kGelu><<<grid, 256, 0, stream>>>(x, y, dy, n);
    else activation_selftest_kernel<kSilu><<<grid, 256, 0, stream>>>(x, y, dy, n);
    return cudaGetLastError();
}

template cudaError_t launch_bwd_pre<float>(const Problem &, const void *, const void *, float *, int, cudaStream_t);
template cudaError_t launch_bwd_pre<__nv_bfloat16>(const Problem &, const void *, const void *, float *, int,
                                                   cudaStream_t);

} // namespace ba
