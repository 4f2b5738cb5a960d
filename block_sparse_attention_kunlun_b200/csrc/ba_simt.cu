// Block attention in fp32 on the CUDA cores (FFMA only, no TF32), forward
// and backward. Same definition and visibility rule as the tensor-core path
// (ba_common.cuh); kept simple: one thread per query row (forward, dq) or per
// key row (dk, dv), keys or queries staged through shared memory in chunks of
// 32, softmax with expf/logf.
#include "ba_common.cuh"
#include "ba_kernels.cuh"

namespace ba {

namespace {
constexpr int kChunk = 32;
}

template <int D>
__global__ void __launch_bounds__(128)
    fwd_f32_kernel(const Problem p, const float *__restrict__ q, const float *__restrict__ k,
                   const float *__restrict__ v, float *__restrict__ out, float *__restrict__ lse)
{
    __shared__ float ks[kChunk][D], vs[kChunk][D];
    const int64_t B = p.block, W = p.window, H = p.heads;
    TileRef r;
    const int32_t ntiles = live_tile_count(p);
    for (int64_t n = blockIdx.x; decode_item(p, ntiles, n, r); n += gridDim.x) {
        const int64_t i = int64_t(r.t) * kTile + threadIdx.x;
        const bool valid = i < r.L;
        const int64_t ws = window_start(i, B, W);
        const int64_t klo = window_start(int64_t(r.t) * kTile, B, W);
        const int64_t khi = (int64_t(r.t) * kTile + kTile < r.L ? int64_t(r.t) * kTile + kTile : r.L) - 1;
        float qr[D], o[D];
        const float *qrow = q + ((r.s0 + i) * H + r.h) * D;
#pragma unroll
        for (int d = 0; d < D; ++d) {
            qr[d] = valid ? qrow[d] * p.scale : 0.f;
            o[d] = 0.f;
        }
        float m = -INFINITY, l = 0.f;
        for (int64_t c0 = klo; c0 <= khi; c0 += kChunk) {
            __syncthreads();
            for (int x = threadIdx.x; x < kChunk * D; x += blockDim.x) {
                const int kk = x / D, d = x % D;
                const int64_t key = c0 + kk;
                const int64_t g = ((r.s0 + key) * H + r.h) * D + d;
                ks[kk][d] = key <= khi ? k[g] : 0.f;
                vs[kk][d] = key <= khi ? v[g] : 0.f;
            }
            __syncthreads();
            if (!valid) continue;
            for (int kk = 0; kk < kChunk; ++kk) {
                const int64_t key = c0 + kk;
                if (key > i || key < ws) continue;
                float s = 0.f;
#pragma unroll
                for (int d = 0; d < D; ++d) s = fmaf(qr[d], ks[kk][d], s);
                if (s > m) {
                    const float corr = expf(m - s);
                    l *= corr;
#pragma unroll
                    for (int d = 0; d < D; ++d) o[d] *= corr;
                    m = s;
                }
                const float e = expf(s - m);
                l += e;
#pragma unroll
                for (int d = 0; d < D; ++d) o[d] = fmaf(e, vs[kk][d], o[d]);
            }
        }
        if (valid) {
            float *orow = out + ((r.s0 + i) * H + r.h) * D;
            const float inv = 1.f / l;
#pragma unroll
            for (int d = 0; d < D; ++d) orow[d] = o[d] * inv;
            lse[int64_t(r.h) * p.total_tokens + r.s0 + i] = m + logf(l);
        }
    }
}

// dq_i = scale * sum_j p_ij (dp_ij - Delta_i) k_j, one thread per query row.
template <int D>
__global__ void __launch_bounds__(128)
    bwd_dq_f32_kernel(const Problem p, const float *__restrict__ q, const float *__restrict__ k,
                      const float *__restrict__ v, const float *__restrict__ dout, const float *__restrict__ lse,
                      const float *__restrict__ delta, float *__restrict__ dq)
{
    __shared__ float ks[kChunk][D], vs[kChunk][D];
    const int64_t B = p.block, W = p.window, H = p.heads, T = p.total_tokens;
    TileRef r;
    const int32_t ntiles = live_tile_count(p);
    for (int64_t n = blockIdx.x; decode_item(p, ntiles, n, r); n += gridDim.x) {
        const int64_t i = int64_t(r.t) * kTile + threadIdx.x;
        const bool valid = i < r.L;
        const int64_t ws = window_start(i, B, W);
        const int64_t klo = window_start(int64_t(r.t) * kTile, B, W);
        const int64_t khi = (int64_t(r.t) * kTile + kTile < r.L ? int64_t(r.t) * kTile + kTile : r.L) - 1;
        const int64_t row = ((r.s0 + i) * H + r.h) * D;
        float qr[D], gr[D], acc[D];
#pragma unroll
        for (int d = 0; d < D; ++d) {
            qr[d] = valid ? q[row + d] * p.scale : 0.f;
            gr[d] = valid ? dout[row + d] : 0.f;
            acc[d] = 0.f;
        }
        const float li = valid ? lse[r.h * T + r.s0 + i] : 0.f;
        const float di = valid ? delta[r.h * T + r.s0 + i] : 0.f;
        for (int64_t c0 = klo; c0 <= khi; c0 += kChunk) {
            __syncthreads();
            for (int x = threadIdx.x; x < kChunk * D; x += blockDim.x) {
                const int kk = x / D, d = x % D;
                const int64_t key = c0 + kk;
                const int64_t g = ((r.s0 + key) * H + r.h) * D + d;
                ks[kk][d] = key <= khi ? k[g] : 0.f;
                vs[kk][d] = key <= khi ? v[g] : 0.f;
            }
            __syncthreads();
            if (!valid) continue;
            for (int kk = 0; kk < kChunk; ++kk) {
                const int64_t key = c0 + kk;
                if (key > i || key < ws) continue;
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int d = 0; d < D; ++d) {
                    s = fmaf(qr[d], ks[kk][d], s);
                    dp = fmaf(gr[d], vs[kk][d], dp);
                }
                const float ds = expf(s - li) * (dp - di);
#pragma unroll
                for (int d = 0; d < D; ++d) acc[d] = fmaf(ds, ks[kk][d], acc[d]);
            }
        }
        if (valid) {
#pragma unroll
            for (int d = 0; d < D; ++d) dq[row + d] = acc[d] * p.scale;
        }
    }
}

// dk_j = scale * sum_i ds_ij q_i, dv_j = sum_i p_ij dO_i, one thread per key row.
template <int D>
__global__ void __launch_bounds__(128)
    bwd_dkdv_f32_kernel(const Problem p, const float *__restrict__ q, const float *__restrict__ k,
                        const float *__restrict__ v, const float *__restrict__ dout,
                        const float *__restrict__ lse, const float *__restrict__ delta, float *__restrict__ dk,
                        float *__restrict__ dv)
{
    __shared__ float qs[kChunk][D], gs[kChunk][D], ls[kChunk], dls[kChunk];
    const int64_t B = p.block, W = p.window, H = p.heads, T = p.total_tokens;
    TileRef r;
    const int32_t ntiles = live_tile_count(p);
    for (int64_t n = blockIdx.x; decode_item(p, ntiles, n, r); n += gridDim.x) {
        const int64_t j = int64_t(r.t) * kTile + threadIdx.x;
        const bool valid = j < r.L;
        const int64_t jmax = (int64_t(r.t) * kTile + kTile < r.L ? int64_t(r.t) * kTile + kTile : r.L) - 1;
        const int64_t qlo = int64_t(r.t) * kTile;
        const int64_t qhi = last_query_seeing(jmax, r.L, B, W);
        const int64_t my_qhi = valid ? last_query_seeing(j, r.L, B, W) : -1;
        const int64_t row = ((r.s0 + j) * H + r.h) * D;
        float kr[D], vr[D], adk[D], adv[D];
#pragma unroll
        for (int d = 0; d < D; ++d) {
            kr[d] = valid ? k[row + d] * p.scale : 0.f;
            vr[d] = valid ? v[row + d] : 0.f;
            adk[d] = 0.f;
            adv[d] = 0.f;
        }
        for (int64_t c0 = qlo; c0 <= qhi; c0 += kChunk) {
            __syncthreads();
            for (int x = threadIdx.x; x < kChunk * D; x += blockDim.x) {
                const int qq = x / D, d = x % D;
                const int64_t qi = c0 + qq;
                const int64_t g = ((r.s0 + qi) * H + r.h) * D + d;
                qs[qq][d] = qi <= qhi ? q[g] : 0.f;
                gs[qq][d] = qi <= qhi ? dout[g] : 0.f;
            }
            if (threadIdx.x < kChunk) {
                const int64_t qi = c0 + threadIdx.x;
                ls[threadIdx.x] = qi <= qhi ? lse[r.h * T + r.s0 + qi] : 0.f;
                dls[threadIdx.x] = qi <= qhi ? delta[r.h * T + r.s0 + qi] : 0.f;
            }
            __syncthreads();
            if (!valid) continue;
            for (int qq = 0; qq < kChunk; ++qq) {
                const int64_t qi = c0 + qq;
                if (qi < j || qi > my_qhi) continue;
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int d = 0; d < D; ++d) {
                    s = fmaf(kr[d], qs[qq][d], s);
                    dp = fmaf(vr[d], gs[qq][d], dp);
                }
                const float pr = expf(s - ls[qq]);
                const float ds = pr * (dp - dls[qq]);
#pragma unroll
                for (int d = 0; d < D; ++d) {
                    adk[d] = fmaf(ds, qs[qq][d], adk[d]);
                    adv[d] = fmaf(pr, gs[qq][d], adv[d]);
                }
            }
        }
        if (valid) {
#pragma unroll
            for (int d = 0; d < D; ++d) {
                dk[row + d] = adk[d] * p.scale;
                dv[row + d] = adv[d];
            }
        }
    }
}

static int simt_grid(int num_sms) { return num_sms * 8; }

cudaError_t launch_fwd_f32(const Problem &p, const float *q, const float *k, const float *v, float *out, float *lse,
                           int num_sms, cudaStream_t stream)
{
    switch (p.head_dim) {
    case 32: fwd_f32_kernel<32><<<simt_grid(num_sms), 128, 0, stream>>>(p, q, k, v, out, lse); break;
    case 64: fwd_f32_kernel<64><<<simt_grid(num_sms), 128, 0, stream>>>(p, q, k, v, out, lse); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_bwd_f32(const Problem &p, const float *q, const float *k, const float *v, const float *dout,
                           const float *lse, const float *delta, float *dq, float *dk, float *dv, int num_sms,
                           cudaStream_t stream)
{
    switch (p.head_dim) {
    case 32:
        bwd_dq_f32_kernel<32><<<simt_grid(num_sms), 128, 0, stream>>>(p, q, k, v, dout, lse, delta, dq);
        bwd_dkdv_f32_kernel<32><<<simt_grid(num_sms), 128, 0, stream>>>(p, q, k, v, dout, lse, delta, dk, dv);
        break;
    case 64:
        bwd_dq_f32_kernel<64><<<simt_grid(num_sms), 128, 0, stream>>>(p, q, k, v, dout, lse, delta, dq);
        bwd_dkdv_f32_kernel<64><<<simt_grid(num_sms), 128, 0, stream>>>(p, q, k, v, dout, lse, delta, dk, dv);
        break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

} // namespace ba
