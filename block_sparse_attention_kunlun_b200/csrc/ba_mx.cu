// MX block quantisation (OCP Microscaling, MXFP8 with E4M3 elements) of bf16
// rows, the operand format "Meta Scales GEM Ads Model Across Platforms and
// Thousands of GPUs" (opening section) says GEM's attention layers train in.
//
// The format, from its public definition: 32 consecutive elements along the
// row share one scale X = 2^e stored as an E8M0 byte (e + 127); with amax the
// block's largest magnitude, e = floor(log2 amax) - 8 (8 is E4M3's largest
// exponent), clamped to [-127, 127], and e = -8 for an all-zero block; each
// element is v / X rounded to the nearest E4M3 value, ties to even, with
// magnitudes above E4M3's largest normal (448) clamped to it. Dividing by a
// power of two is exact in float32 here (the quotient stays below 2^9), so
// the only rounding is the final conversion.
#include "ba_kernels.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

namespace ba {

namespace {

// floor(log2 |x|) of a nonzero finite float, from its exponent field
// (subnormals through the position of their leading one).
__device__ __forceinline__ int floor_log2(float x)
{
    const uint32_t b = __float_as_uint(x) & 0x7fffffffu;
    const int ef = int(b >> 23);
    if (ef > 0) return ef - 127;
    return -127 - (__clz(b) - 9); // subnormal: 2^-149 .. 2^-127
}

} // namespace

namespace {

// The 32 values of one block, from 64 bytes of bf16.
__device__ __forceinline__ void load_block(const __nv_bfloat16 *x, float (&v)[32])
{
    const uint4 *src = reinterpret_cast<const uint4 *>(x);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint4 w = src[u];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ws[e]));
            v[8 * u + 2 * e] = f.x;
            v[8 * u + 2 * e + 1] = f.y;
        }
    }
}

// MX code of one block: the scale exponent e (returned) and the 32 E4M3
// element bytes, four to a word.
__device__ __forceinline__ int encode_block(const float (&v)[32], uint32_t (&out)[8])
{
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    int e = amax > 0.f ? floor_log2(amax) - 8 : -8;
    e = e < -127 ? -127 : (e > 127 ? 127 : e);
    // 1 / 2^e as two power-of-two factors (2^127 and 2^-127 are not both floats)
    const float inv_hi = ldexpf(1.f, -e / 2), inv_lo = ldexpf(1.f, -e - (-e / 2));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
            make_float2(v[4 * i] * inv_hi * inv_lo, v[4 * i + 1] * inv_hi * inv_lo), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
            make_float2(v[4 * i + 2] * inv_hi * inv_lo, v[4 * i + 3] * inv_hi * inv_lo), __NV_SATFINITE, __NV_E4M3);
        out[i] = uint32_t(lo) | (uint32_t(hi) << 16);
    }
    return e;
}

} // namespace

// One thread per 32-element block of a [rows, heads, head_dim] bf16 tensor:
// reads 64 bytes, writes 32 element bytes (same layout, E4M3) and one scale
// byte at scales[(row * heads_pad + head) * (head_dim / 32) + block], heads_pad
// = heads rounded up to a multiple of 4 (so that a row of scale words is a
// multiple of 16 bytes and one 16-byte TMA box holds four heads' words).
__global__ void __launch_bounds__(256)
    mx_quantize_e4m3_kernel(const __nv_bfloat16 *__restrict__ x, int64_t nblocks, int32_t heads, int32_t heads_pad,
                            int32_t blocks_per_head, uint8_t *__restrict__ elems, uint8_t *__restrict__ scales)
{
    for (int64_t blk = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; blk < nblocks;
         blk += int64_t(gridDim.x) * blockDim.x) {
        float v[32];
        load_block(x + blk * 32, v);
        uint32_t out[8];
        const int e = encode_block(v, out);
        uint4 *dst = reinterpret_cast<uint4 *>(elems + blk * 32);
        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
        const int64_t rh = blk / blocks_per_head; // (row, head)
        const int64_t row = rh / heads, h = rh % heads;
        scales[(row * heads_pad + h) * blocks_per_head + blk % blocks_per_head] = uint8_t(e + 127);
    }
}

// The round trip: each 32-element block of a bf16 tensor encoded as above and
// decoded again (element value times 2^e) into bf16. An E4M3 value has four
// significant bits, so the decoded value is exact in bf16 unless it falls
// below bf16's normal range (a block whose largest magnitude is under
// 2^-118); there it rounds to the nearest bf16 subnormal.
__global__ void __launch_bounds__(256)
    mx_round_trip_kernel(const __nv_bfloat16 *__restrict__ x, int64_t nblocks, __nv_bfloat16 *__restrict__ y)
{
    for (int64_t blk = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; blk < nblocks;
         blk += int64_t(gridDim.x) * blockDim.x) {
        float v[32];
        load_block(x + blk * 32, v);
        uint32_t code[8];
        const int e = encode_block(v, code);
        const float s_hi = ldexpf(1.f, e / 2), s_lo = ldexpf(1.f, e - e / 2);
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t two = (code[i / 2] >> (16 * (i % 2))) & 0xffffu; // elements 2i, 2i + 1
            const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2(__nv_fp8x2_storage_t(two), __NV_E4M3);
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h2));
            const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * s_hi * s_lo, f.y * s_hi * s_lo);
            packed[i] = *reinterpret_cast<const uint32_t *>(&b);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(y + blk * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            dst[u] = make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
    }
}

cudaError_t launch_mx_quantize(const void *x, int64_t rows, int32_t heads, int32_t head_dim, void *elems,
                               void *scales, int num_sms, cudaStream_t stream)
{
    const int64_t nblocks = rows * heads * (head_dim / 32);
    if (nblocks == 0) return cudaSuccess;
    int64_t g = (nblocks + 255) / 256;
    const int64_t cap = int64_t(num_sms) * 8;
    if (g > cap) g = cap;
    mx_quantize_e4m3_kernel<<<int(g), 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(x), nblocks, heads,
                                                        (heads + 3) / 4 * 4, head_dim / 32,
                                                        static_cast<uint8_t *>(elems), static_cast<uint8_t *>(scales));
    return cudaGetLastError();
}

cudaError_t launch_mx_round_trip(const void *x, int64_t elems, void *y, int num_sms, cudaStream_t stream)
{
    const int64_t nblocks = elems / 32;
    if (nblocks == 0) return cudaSuccess;
    int64_t g = (nblocks + 255) / 256;
    const int64_t cap = int64_t(num_sms) * 8;
    if (g > cap) g = cap;
    mx_round_trip_kernel<<<int(g), 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(x), nblocks,
                                                     static_cast<__nv_bfloat16 *>(y));
    return cudaGetLastError();
}

} // namespace ba
