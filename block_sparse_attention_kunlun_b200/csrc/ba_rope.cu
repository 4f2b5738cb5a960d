// Rotary position embedding as a pass over whole rows ("GEM (Meta)", section
// "Custom kernels": the production block-attention kernel carries a fused
// rotary embedding). RoFormer's rotation of adjacent pairs; the row's
// position is its index within its example.
//
//   forward (q, k -> rotated copies the attention kernels read):
//       a_out = R(pos) a_in,   b_out = R(pos) b_in
//   transposed, in place (the fp32 backward's dq, dk; the bf16 backward
//   applies R(pos)^T inside the dQ and dK/dV epilogues instead):
//       a = R(pos)^T a,        b = R(pos)^T b
//
// HBM-bound: per row and head it reads 2 x head_dim elements and writes as
// many; the cos/sin tables ([rows, head_dim / 2] float32) stay in L2. Every
// row of the batch is rotated, skipped examples' too: the attention kernels
// load whole 128-row tiles, so a tile at the end of one example also reads
// the next example's rows (masked, but multiplied by a zero probability,
// which must not meet a NaN). A CTA takes 128 consecutive rows, finds each
// row's example by binary search over seq_offsets, then moves 16-byte
// vectors, four per thread at a time, loading all four before storing any
// (the in-place form reads and writes the same vectors).
#include "ba_common.cuh"
#include "ba_kernels.cuh"

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace ba {
namespace {

constexpr int kRopeThreads = 256;
constexpr int kRopeUnroll = 4;

// 16 bytes of T as float pairs and back.
template <typename T> struct Pairs;

template <> struct Pairs<__nv_bfloat16> {
    static constexpr int kPairs = 4;
    static __device__ __forceinline__ void unpack(const uint4 &u, float (&x)[8])
    {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
        }
    }
    static __device__ __forceinline__ uint4 pack(const float (&x)[8])
    {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&b);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <> struct Pairs<float> {
    static constexpr int kPairs = 2;
    static __device__ __forceinline__ void unpack(const uint4 &u, float (&x)[4])
    {
        x[0] = __uint_as_float(u.x);
        x[1] = __uint_as_float(u.y);
        x[2] = __uint_as_float(u.z);
        x[3] = __uint_as_float(u.w);
    }
    static __device__ __forceinline__ uint4 pack(const float (&x)[4])
    {
        return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
    }
};

// NP consecutive table entries (16-byte aligned for NP = 4, 8-byte for NP = 2).
template <int NP> __device__ __forceinline__ void load_table(const float *t, float (&x)[NP]);
template <> __device__ __forceinline__ void load_table<4>(const float *t, float (&x)[4])
{
    const float4 f = __ldg(reinterpret_cast<const float4 *>(t));
    x[0] = f.x;
    x[1] = f.y;
    x[2] = f.z;
    x[3] = f.w;
}
template <> __device__ __forceinline__ void load_table<2>(const float *t, float (&x)[2])
{
    const float2 f = __ldg(reinterpret_cast<const float2 *>(t));
    x[0] = f.x;
    x[1] = f.y;
}

template <typename T, bool kTranspose>
__global__ void __launch_bounds__(kRopeThreads)
    rope_rows_kernel(const Problem p, const T *a_in, const T *b_in, T *a_out, T *b_out)
{
    using V = Pairs<T>;
    constexpr int NP = V::kPairs;                      // pairs per 16-byte vector
    __shared__ int32_t s_pos[kTile];                   // position of each row of the chunk in its example
    const int32_t nchunks = (p.total_tokens + kTile - 1) / kTile;
    const int32_t head_vecs = p.head_dim / (2 * NP);   // vectors per head row (a power of two)
    const int32_t row_vecs = p.heads * head_vecs;      // vectors per token row
    const int32_t half = p.head_dim / 2;
    const uint4 *ain = reinterpret_cast<const uint4 *>(a_in);
    const uint4 *bin = reinterpret_cast<const uint4 *>(b_in);
    uint4 *aout = reinterpret_cast<uint4 *>(a_out);
    uint4 *bout = reinterpret_cast<uint4 *>(b_out);
    for (int32_t chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
        const int32_t r0 = chunk * kTile; // first row of the chunk (global)
        const int32_t rows = min(kTile, p.total_tokens - r0);
        __syncthreads(); // the previous chunk's positions are no longer read
        if (int(threadIdx.x) < rows) {
            // the example holding this row: the last e with seq_offsets[e] <= row
            // (seq_offsets[batch] = total_tokens > row, so e < batch and the search is bounded)
            const int32_t row = r0 + int32_t(threadIdx.x);
            int32_t lo = 1, hi = p.batch;
            while (lo < hi) {
                const int32_t mid = (lo + hi) >> 1;
                if (__ldg(p.seq_offsets + mid) > row) hi = mid;
                else lo = mid + 1;
            }
            s_pos[threadIdx.x] = row - __ldg(p.seq_offsets + lo - 1);
        }
        __syncthreads();
        const int64_t base = int64_t(r0) * row_vecs; // first vector of the chunk
        const int32_t nvec = rows * row_vecs;        // < 2^31: heads * head_dim <= 2^24
        for (int32_t v0 = threadIdx.x; v0 < nvec; v0 += kRopeUnroll * kRopeThreads) {
            uint4 xa[kRopeUnroll], xb[kRopeUnroll];
            float cs[kRopeUnroll][NP], sn[kRopeUnroll][NP];
#pragma unroll
            for (int u = 0; u < kRopeUnroll; ++u) {
                const int32_t v = v0 + u * kRopeThreads;
                if (v >= nvec) break;
                const int32_t pos = s_pos[v / row_vecs];
                const int32_t k0 = (v & (head_vecs - 1)) * NP; // first pair of the vector
                xa[u] = ain[base + v];
                xb[u] = bin[base + v];
                if (pos >= 0 && pos < p.rope_rows) {
                    load_table<NP>(p.rope_cos + int64_t(pos) * half + k0, cs[u]);
                    load_table<NP>(p.rope_sin + int64_t(pos) * half + k0, sn[u]);
                } else {
                    atomicOr(p.status, kStatusRopeRange);
#pragma unroll
                    for (int e = 0; e < NP; ++e) {
                        cs[u][e] = 1.f;
                        sn[u][e] = 0.f;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kRopeUnroll; ++u) {
                const int32_t v = v0 + u * kRopeThreads;
                if (v >= nvec) break;
                float a[2 * NP], b[2 * NP];
                V::unpack(xa[u], a);
                V::unpack(xb[u], b);
#pragma unroll
                for (int e = 0; e < NP; ++e) {
                    const float2 ra = kTranspose ? rope_pair_t(a[2 * e], a[2 * e + 1], cs[u][e], sn[u][e])
                                                 : rope_pair(a[2 * e], a[2 * e + 1], cs[u][e], sn[u][e]);
                    const float2 rb = kTranspose ? rope_pair_t(b[2 * e], b[2 * e + 1], cs[u][e], sn[u][e])
                                                 : rope_pair(b[2 * e], b[2 * e + 1], cs[u][e], sn[u][e]);
                    a[2 * e] = ra.x;
                    a[2 * e + 1] = ra.y;
                    b[2 * e] = rb.x;
                    b[2 * e + 1] = rb.y;
                }
                aout[base + v] = V::pack(a);
                bout[base + v] = V::pack(b);
            }
        }
    }
}

template <typename T>
cudaError_t launch_rope_typed(const Problem &p, bool transpose, const void *a_in, const void *b_in, void *a_out,
                              void *b_out, int num_sms, cudaStream_t stream)
{
    const int64_t chunks = (int64_t(p.total_tokens) + kTile - 1) / kTile;
    const int grid = int(chunks < int64_t(num_sms) * 8 ? chunks : int64_t(num_sms) * 8);
    if (grid <= 0) return cudaSuccess;
    const T *ai = static_cast<const T *>(a_in), *bi = static_cast<const T *>(b_in);
    T *ao = static_cast<T *>(a_out), *bo = static_cast<T *>(b_out);
    if (transpose) rope_rows_kernel<T, true><<<grid, kRopeThreads, 0, stream>>>(p, ai, bi, ao, bo);
    else rope_rows_kernel<T, false><<<grid, kRopeThreads, 0, stream>>>(p, ai, bi, ao, bo);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_rope_rows(const Problem &p, size_t elem_bytes, bool transpose, const void *a_in, const void *b_in,
                             void *a_out, void *b_out, int num_sms, cudaStream_t stream)
{
    if (elem_bytes == 2)
        return launch_rope_typed<__nv_bfloat16>(p, transpose, a_in, b_in, a_out, b_out, num_sms, stream);
    return launch_rope_typed<float>(p, transpose, a_in, b_in, a_out, b_out, num_sms, stream);
}

} // namespace ba
