// Shared definitions for the block-attention kernels: the visibility rule,
// tile ranges, workspace layout and kernel parameter blocks.
//
// Visibility (local 0-based indices within one example, blk(x) = x / block):
//   query i sees key j  <=>  j <= i  and  blk(j) >= blk(i) - (window - 1)
// ("Meta Scales GEM Ads Model Across Platforms and Thousands of GPUs",
// section "Kunlun changes how GEM scales": attention arranged in blocks with
// cost linear in length for a fixed window; "GEM (Meta)", section "Custom
// kernels": independent 64-token blocks = window 1, block 64).
#pragma once

#include <cstddef>
#include <cstdint>

namespace ba {

constexpr int kTile = 128;          // rows per query tile and per key tile
constexpr int kWorklistThreads = 1024;

// Status bits the kernels OR into the workspace status word.
constexpr int kStatusTimeout = 1;
constexpr int kStatusRopeRange = 2; // a row's position was past the rotary tables

// First key visible to query i: the start of block blk(i) - (window - 1),
// clamped at 0. Indices are local to an example and fit in 32 bits; the
// product below never exceeds i, so the 32-bit division is exact and cheap.
__host__ __device__ __forceinline__ int64_t window_start(int64_t i, int64_t block, int64_t window)
{
    const int32_t b = int32_t(i) / int32_t(block);
    return b >= int32_t(window) ? int64_t(b - int32_t(window) + 1) * block : 0;
}

// Last query (of an example of length L) that sees key j.
__host__ __device__ __forceinline__ int64_t last_query_seeing(int64_t j, int64_t L, int64_t block,
                                                              int64_t window)
{
    const int32_t b = int32_t(j) / int32_t(block);
    const int64_t hi = (int64_t(b) + window) * block - 1;
    return hi < L - 1 ? hi : L - 1;
}

__host__ __device__ __forceinline__ bool visible(int64_t i, int64_t j, int64_t block, int64_t window)
{
    return j <= i && j >= window_start(i, block, window);
}

// Workspace layout (all offsets 256-byte aligned):
//   [0, 256)            status word (int32)
//   tile_prefix         int32[batch + 1]: slot of example b's first tile in
//                       tile_info; [batch] = number of live tiles
//   tile_info           int4[max_tiles]: per live tile {first row of its
//                       example, example length, tile index in the example,
//                       example index}, max_tiles = ceil(T / 128) + batch;
//                       examples longest first, an example's tiles in order
//   pair_prefix         int32[batch + 1]: likewise for pairs of consecutive
//                       tiles; [batch] = number of live pairs
//   pair_info           int4[max_pairs]: per pair {row0, length, first tile,
//                       example}, max_pairs = ceil(T / 256) + batch
//   delta   (bwd only)  float[heads * total_tokens]: Delta (fp32 path) or -Delta
//                       (bf16 path, written by the dQ pass for the dK/dV pass)
//   nlse2   (bwd only)  float[heads * total_tokens]: -lse in log2 units (bf16 path)
//   tail_q, tail_do     (bf16 backward only) bf16[batch * 128, heads * head_dim]
//                       each: rows 128b .. 128b + 127 hold example b's last,
//                       partial query tile of q (dout), zeros past the example
//                       (the dK/dV pass reads that tile from here)
struct WorkspaceLayout {
    size_t status, tile_prefix, tile_info, pair_prefix, pair_info, delta, nlse2, tail_q, tail_do, tail_k, total;
};

// Masks under which every 128-row query tile sees only its own key tile: window 1
// with blocks that divide the tile. The bf16 backward then runs as one fused pass.
__host__ __device__ inline bool diagonal_tiles(int64_t block, int64_t window)
{
    return window == 1 && block <= kTile && kTile % block == 0;
}

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline int64_t max_tiles(int64_t batch, int64_t total_tokens)
{
    return (total_tokens + kTile - 1) / kTile + batch;
}

__host__ __device__ inline int64_t max_pairs(int64_t batch, int64_t total_tokens)
{
    return (total_tokens + 2 * kTile - 1) / (2 * kTile) + batch;
}

__host__ __device__ inline WorkspaceLayout workspace_layout(int64_t batch, int64_t total_tokens,
                                                            int64_t heads, int64_t head_dim,
                                                            bool with_delta, bool tail_rows = false,
                                                            bool tail_k = false)
{
    WorkspaceLayout w;
    w.status = 0;
    w.tile_prefix = 256;
    size_t off = align256(w.tile_prefix + sizeof(int32_t) * size_t(batch + 1));
    w.tile_info = off;
    off = align256(off + 16 * size_t(max_tiles(batch, total_tokens)));
    w.pair_prefix = off;
    off = align256(off + sizeof(int32_t) * size_t(batch + 1));
    w.pair_info = off;
    off = align256(off + 16 * size_t(max_pairs(batch, total_tokens)));
    // backward only: per-row Delta, and (bf16 path) -lse in log2 units, both [heads, total_tokens]
    w.delta = off;
    if (with_delta) off = align256(off + sizeof(float) * size_t(heads * total_tokens));
    w.nlse2 = off;
    if (with_delta) off = align256(off + sizeof(float) * size_t(heads * total_tokens));
    const size_t tail_bytes = tail_rows ? align256(size_t(batch) * kTile * size_t(heads * head_dim) * 2) : 0;
    // the partial tiles staged zero-padded: query tiles (q, dout) for the dK/dV pass, and the
    // key tile (k) for the fused backward
    w.tail_q = off;
    w.tail_do = off + tail_bytes;
    w.tail_k = off + 2 * tail_bytes;
    w.total = off + (tail_k ? 3 : 2) * tail_bytes;
    return w;
}

// Common problem description handed to every kernel.
struct Problem {
    const int32_t *seq_offsets; // [batch + 1], device
    const uint8_t *skip;        // [batch] or nullptr
    const int32_t *tile_prefix; // [batch + 1], device (workspace)
    const int4 *tile_info;      // [max_tiles], device (workspace)
    const int32_t *pair_prefix; // [batch + 1], device (workspace)
    const int4 *pair_info;      // [max_pairs], device (workspace)
    int *status;                // workspace status word
    int32_t batch, total_tokens, heads, head_dim, block, window;
    float scale;                // 1 / sqrt(head_dim)
    // rotary tables [rope_rows, head_dim / 2] (cos, sin of position x
    // frequency); rope_cos == nullptr: no rotation
    const float *rope_cos = nullptr;
    const float *rope_sin = nullptr;
    int32_t rope_rows = 0;
    // cross-attention (generalized attention only): the other side's offsets
    // [batch + 1] (key/value rows for the query-tile kernels, query rows for
    // the key-tile kernel); nullptr for self-attention
    const int32_t *other_offsets = nullptr;
};

// Rotary position embedding (RoFormer's rotation, adjacent pairs; "GEM
// (Meta)", section "Custom kernels": the block-attention kernel fuses the
// rotary embedding's backward pass). A row at local position pos turns its
// pair (x0, x1) = (x[2k], x[2k+1]) by the angle whose cosine c and sine s
// the tables hold at [pos, k]:
//   forward:    (x0 c - x1 s,  x0 s + x1 c)
//   transposed: (g0 c + g1 s, -g0 s + g1 c)   (gradient of the unrotated row)
// The forward result is rounded to the input dtype for the tensor cores; it
// is formed with each product and the sum rounded once (no fused
// multiply-add), so which way a value near a rounding tie goes follows from
// the formula evaluated in float32 alone.
__device__ __forceinline__ float2 rope_pair(float x0, float x1, float c, float s)
{
    return make_float2(__fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, s)), __fadd_rn(__fmul_rn(x0, s), __fmul_rn(x1, c)));
}

__device__ __forceinline__ float2 rope_pair_t(float g0, float g1, float c, float s)
{
    return make_float2(fmaf(g0, c, g1 * s), fmaf(g1, c, -g0 * s));
}

// 16 bytes of a read-only table, read through the non-coherent path with the
// load kept where it is written (ahead of the code that waits for other work).
__device__ __forceinline__ float4 ld_nc_early(const float4 *ptr)
{
    float4 v;
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(ptr));
    return v;
}

// Transposed rotation, in place, of 4 NQ adjacent pairs (bit patterns v[2m],
// v[2m+1]) with their cos and sin already loaded (c[u], s[u]: pairs 4u .. 4u + 3).
template <int NQ>
__device__ __forceinline__ void rope_transpose_loaded(const float4 *c, const float4 *s, uint32_t *v)
{
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
        const float cc[4] = {c[u].x, c[u].y, c[u].z, c[u].w}, ss[4] = {s[u].x, s[u].y, s[u].z, s[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int m = 4 * u + e;
            const float2 r = rope_pair_t(__uint_as_float(v[2 * m]), __uint_as_float(v[2 * m + 1]), cc[e], ss[e]);
            v[2 * m] = __float_as_uint(r.x);
            v[2 * m + 1] = __float_as_uint(r.y);
        }
    }
}

// Transposed rotation, in place, of 4 * NQ adjacent pairs held as float bit
// patterns v[2m], v[2m+1] (m < 4 * NQ), pair indices k0 .. k0 + 4 NQ - 1 of
// the row at local position pos (k0 a multiple of 4). A position past the
// tables sets kStatusRopeRange and leaves the values as they are.
template <int NQ>
__device__ __forceinline__ void rope_transpose_bits(const Problem &p, int64_t pos, int k0, uint32_t *v)
{
    if (pos >= p.rope_rows) {
        atomicOr(p.status, kStatusRopeRange);
        return;
    }
    const int64_t base = pos * (p.head_dim / 2) + k0;
    const float4 *cs = reinterpret_cast<const float4 *>(p.rope_cos + base);
    const float4 *sn = reinterpret_cast<const float4 *>(p.rope_sin + base);
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
        const float4 c = __ldg(cs + u), s = __ldg(sn + u);
        const float cc[4] = {c.x, c.y, c.z, c.w}, ss[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int m = 4 * u + e;
            const float2 r = rope_pair_t(__uint_as_float(v[2 * m]), __uint_as_float(v[2 * m + 1]), cc[e], ss[e]);
            v[2 * m] = __float_as_uint(r.x);
            v[2 * m + 1] = __float_as_uint(r.y);
        }
    }
}

// What replaces exp(s - lse) in the attention. kSoftmax: block attention.
// kGelu / kSilu: generalized dot-product attention ("GEM (Meta)", section
// "Custom kernels": GEM's self-, cross- and pooled attention with the softmax
// replaced by an activation such as GELU or SiLU), out_i = sum_j act(s_ij) v_j
// over the visible keys with s_ij = q_i . k_j / sqrt(D), no normalisation,
// so no running maximum and no lse.
enum Act : int { kSoftmax = 0, kGelu = 1, kSilu = 2 };

// 2^x and 1/x on the special-function unit (ex2.approx / rcp.approx, relative
// errors near 2^-22 and 2^-23; 2^-inf = 0 and 1/inf = 0). The attention's
// warps are bound by instruction issue, so the activations below use one
// instruction for each rather than the library's full-precision forms.
__device__ __forceinline__ float act_ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float act_rcp(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// GELU(x) = x Phi(x), Phi the standard normal distribution function, with
// Phi from erf by Abramowitz & Stegun, Handbook of Mathematical Functions,
// formula 7.1.26 (Hastings' approximation): for z >= 0,
//   erf(z) = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) e^(-z^2) + eps(z),
//   t = 1 / (1 + p z), |eps(z)| <= 1.5e-7,
// p = 0.3275911, a1..a5 = 0.254829592, -0.284496736, 1.421413741,
// -1.453152027, 1.061405429. With z = |x| / sqrt(2), e^(-z^2) = e^(-x^2/2) is
// also the exponential of the normal density phi, which GELU' = Phi + x phi
// shares. Returns {Phi(x), e^(-x^2/2)}.
__device__ __forceinline__ float2 gelu_parts(float x)
{
    const float z = fabsf(x) * 0.70710678118654752f;
    const float t = act_rcp(fmaf(0.3275911f, z, 1.f));
    const float poly =
        t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, 1.061405429f, -1.453152027f), 1.421413741f), -0.284496736f),
                 0.254829592f);
    const float e = act_ex2(x * x * -0.72134752044448170f); // e^(-x^2/2) = 2^(-x^2 / (2 ln 2))
    const float tail = 0.5f * poly * e;                     // Phi(-|x|) = (1 - erf(z)) / 2
    return make_float2(x >= 0.f ? 1.f - tail : tail, e);
}

// sigma(x) = 1 / (1 + 2^(-x log2 e)) for SiLU(x) = x sigma(x).
__device__ __forceinline__ float silu_sigma(float x) { return act_rcp(1.f + act_ex2(x * -1.4426950408889634f)); }

// The activation: GELU (the erf form above) or SiLU.
template <int A>
__device__ __forceinline__ float act_value(float x)
{
    static_assert(A == kGelu || A == kSilu, "an activation");
    if constexpr (A == kGelu) return x * gelu_parts(x).x;
    else return x * silu_sigma(x);
}

// The activation and its derivative: GELU' = Phi(x) + x phi(x) with
// phi(x) = e^(-x^2/2) / sqrt(2 pi); SiLU' = sigma(x) (1 + x (1 - sigma(x))).
template <int A>
__device__ __forceinline__ float2 act_value_grad(float x)
{
    static_assert(A == kGelu || A == kSilu, "an activation");
    if constexpr (A == kGelu) {
        const float2 g = gelu_parts(x);
        return make_float2(x * g.x, fmaf(x, 0.39894228040143268f * g.y, g.x));
    } else {
        const float sg = silu_sigma(x);
        return make_float2(x * sg, sg * fmaf(x, 1.f - sg, 1.f));
    }
}

// The activation's derivative alone.
template <int A>
__device__ __forceinline__ float act_grad(float x)
{
    static_assert(A == kGelu || A == kSilu, "an activation");
    if constexpr (A == kGelu) {
        const float2 g = gelu_parts(x);
        return fmaf(x, 0.39894228040143268f * g.y, g.x);
    } else {
        const float sg = silu_sigma(x);
        return sg * fmaf(x, 1.f - sg, 1.f);
    }
}

// One 128-row tile of one (example, head).
struct TileRef {
    int32_t b;         // example index
    int32_t h, t;      // head, tile index within the example
    int32_t s0, L;     // first global row of the example, its length
    int32_t os0, oL;   // the other side's rows (cross-attention: the example's key/value set
                       // for a query tile, its queries for a key tile); self-attention: s0, L
};

// Number of live tiles (read once per kernel role).
__device__ __forceinline__ int32_t live_tile_count(const Problem &p) { return p.tile_prefix[p.batch]; }

// Work item n -> (tile, head); tiles are numbered over live examples in
// order, heads vary fastest. Returns false past the last item.
__device__ __forceinline__ bool decode_item(const Problem &p, int32_t ntiles, int64_t n, TileRef &r)
{
    if (n >= int64_t(ntiles) * p.heads) return false;
    const int32_t tile = int32_t(n / p.heads);
    r.h = int32_t(n % p.heads);
    const int4 info = p.tile_info[tile];
    r.b = info.w;
    r.s0 = info.x;
    r.L = info.y;
    r.t = info.z;
    return true;
}

// Number of live tile pairs (read once per kernel role).
__device__ __forceinline__ int32_t live_pair_count(const Problem &p) { return p.pair_prefix[p.batch]; }

// Work item n -> (pair of query tiles 2k and 2k+1 of one example, head).
// r.t is the first tile; `second` tells whether tile r.t + 1 exists.
__device__ __forceinline__ bool decode_pair(const Problem &p, int32_t npairs, int64_t n, TileRef &r, bool &second)
{
    if (n >= int64_t(npairs) * p.heads) return false;
    const int32_t pair = int32_t(n / p.heads);
    r.h = int32_t(n % p.heads);
    const int4 info = p.pair_info[pair];
    r.b = info.w;
    r.s0 = info.x;
    r.L = info.y;
    r.t = info.z;
    second = int64_t(r.t + 1) * kTile < r.L;
    return true;
}

// Whether a pair item (first tile r.t) has its second tile.
__device__ __forceinline__ bool pair_has_second(const TileRef &r) { return int64_t(r.t + 1) * kTile < r.L; }

} // namespace ba
