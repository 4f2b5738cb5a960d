// The library's C ABI (declared in include/ba.h): host-side argument checks,
// workspace carving, TMA descriptor encoding and the launch sequence.
//
//   ba_fwd: worklist -> skip passthrough (if any flags) -> forward kernel
//           (tcgen05 for bf16, SIMT for fp32)
//   ba_bwd: worklist -> skip passthrough -> bf16: dQ kernel (also writes
//           Delta) -> dK/dV kernel; fp32: Delta pre-pass -> dQ and dK/dV
//           SIMT kernels
//   ba_gdpa_fwd / ba_gdpa_bwd: worklist -> the same tensor-core kernels
//           instantiated with an activation in place of the softmax
//   ba_rope_fwd / ba_rope_bwd: the same, with a rotary pass writing rotated
//           copies of q and k into the workspace before the attention
//           kernels read them; the bf16 backward turns dq and dk back inside
//           the dQ and dK/dV epilogues, the fp32 one in a pass after them
// Nothing here allocates, synchronises or falls back to another device.
#include "ba.h"
#include "ba_common.cuh"
#include "ba_kernels.cuh"

#include <atomic>
#include <cmath>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <type_traits>

namespace {

using namespace ba;

constexpr int kMaxDevices = 64;
std::atomic<int> g_num_sms[kMaxDevices];
std::atomic<int> g_cc_major[kMaxDevices];

bool device_info(int &num_sms, int &cc_major)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    if (dev < kMaxDevices && g_num_sms[dev].load() > 0) {
        num_sms = g_num_sms[dev].load();
        cc_major = g_cc_major[dev].load();
        return true;
    }
    if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    if (dev < kMaxDevices) {
        g_cc_major[dev].store(cc_major);
        g_num_sms[dev].store(num_sms);
    }
    return true;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static std::atomic<void *> fn{nullptr};
    void *f = fn.load();
    if (!f) {
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn.store(f);
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

// 2-D view [total_tokens, heads * head_dim] of a bf16 tensor, boxes of 128
// rows x 64 columns (128 bytes) with the 128-byte swizzle the MMA
// descriptors expect; rows past the end read as zeros.
bool encode_bf16_rows(CUtensorMap *map, const void *base, int64_t T, int64_t H, int64_t D)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cuuint64_t(H * D), cuuint64_t(T)};
    cuuint64_t strides[1] = {cuuint64_t(H * D * 2)};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D byte views for the MXFP8 forward: E4M3 rows [T, H * D] in 128 x 128-byte
// boxes (one 128-byte swizzled row per head at head_dim 128), and scale words
// [T, heads_pad * 4] in 128-row x 16-byte boxes (four heads' words).
bool encode_u8_rows(CUtensorMap *map, const void *base, int64_t T, int64_t row_bytes, uint32_t box_x, bool swizzle)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cuuint64_t(row_bytes), cuuint64_t(T)};
    cuuint64_t strides[1] = {cuuint64_t(row_bytes)};
    cuuint32_t box[2] = {box_x, 128};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The dK/dV pass's partial query tiles: each example's last query tile, when
// it has fewer than 128 rows, copied from q and dout (query rows given by
// offs) into the workspace with zeros past the example, and the tensor maps
// the pass reads them through (rows 128 b .. 128 b + 127 for example b).
bool stage_query_tails(const ba_problem &P, const int32_t *offs, const uint8_t *skip, const void *q,
                       const void *dout, uint8_t *ws, const WorkspaceLayout &lay, CUtensorMap &tqt, CUtensorMap &tdot,
                       cudaStream_t stream, const void *k = nullptr, CUtensorMap *tkt = nullptr)
{
    const int64_t rows = int64_t(P.batch) * kTile;
    if (!encode_bf16_rows(&tqt, ws + lay.tail_q, rows, P.heads, P.head_dim) ||
        !encode_bf16_rows(&tdot, ws + lay.tail_do, rows, P.heads, P.head_dim) ||
        (k && !encode_bf16_rows(tkt, ws + lay.tail_k, rows, P.heads, P.head_dim)))
        return false;
    return launch_stage_query_tails(offs, skip, P.batch, size_t(P.heads) * P.head_dim * 2, q, dout, ws + lay.tail_q,
                                    ws + lay.tail_do, stream, k, k ? ws + lay.tail_k : nullptr) == cudaSuccess;
}

// The bf16 backward runs fused (one pass for dQ, dK and dV) when every query
// tile sees only its own key tile, for block attention without rotation.
bool fused_backward(const ba_problem &P, int32_t block, int32_t window, bool with_rope)
{
    return P.dtype == BA_BF16 && !with_rope && diagonal_tiles(block, window);
}

// The backward's workspace: the per-row statistics, the staged partial tiles
// (bf16), and for the fused backward the staged partial key tiles.
WorkspaceLayout bwd_layout(const ba_problem &P, int32_t block, int32_t window, bool with_rope)
{
    return workspace_layout(P.batch, P.total_tokens, P.heads, P.head_dim, true, P.dtype == BA_BF16,
                            fused_backward(P, block, window, with_rope));
}

bool head_dim_supported(const ba_problem &p)
{
    if (p.dtype == BA_BF16) return p.head_dim == 64 || p.head_dim == 128;
    if (p.dtype == BA_F32) return p.head_dim == 32 || p.head_dim == 64;
    return false;
}

ba_status check_problem(const ba_problem *p, int32_t block, int32_t window)
{
    if (!p) return BA_ERR_INVALID_ARG;
    if (p->batch < 0 || p->total_tokens < 0 || p->heads < 1 || p->head_dim < 1 || block < 1 || window < 1)
        return BA_ERR_INVALID_ARG;
    if (p->dtype != BA_F32 && p->dtype != BA_BF16) return BA_ERR_INVALID_ARG;
    if (p->batch == 0 && p->total_tokens != 0) return BA_ERR_INVALID_ARG;
    // element offsets of one tensor must stay below 2^62 and rows below 2^31
    if (int64_t(p->heads) * p->head_dim > (int64_t(1) << 24)) return BA_ERR_UNSUPPORTED;
    // work items (128-row tiles x heads) and the staged tail rows (128 per example) are numbered in 31 bits
    if (max_tiles(p->batch, p->total_tokens) * p->heads > INT32_MAX || int64_t(p->batch) * kTile > INT32_MAX)
        return BA_ERR_UNSUPPORTED;
    if (!head_dim_supported(*p)) return BA_ERR_UNSUPPORTED;
    return BA_OK;
}

bool tensor_ok(const void *t, int64_t T) { return T == 0 || (t && aligned(t, 16)); }

Problem make_problem(const ba_problem &pp, const int32_t *offs, const uint8_t *skip, int32_t block, int32_t window,
                     void *workspace, const WorkspaceLayout &lay)
{
    Problem p;
    p.seq_offsets = offs;
    p.skip = skip;
    p.tile_prefix = reinterpret_cast<const int32_t *>(static_cast<uint8_t *>(workspace) + lay.tile_prefix);
    p.tile_info = reinterpret_cast<const int4 *>(static_cast<uint8_t *>(workspace) + lay.tile_info);
    p.pair_prefix = reinterpret_cast<const int32_t *>(static_cast<uint8_t *>(workspace) + lay.pair_prefix);
    p.pair_info = reinterpret_cast<const int4 *>(static_cast<uint8_t *>(workspace) + lay.pair_info);
    p.status = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + lay.status);
    p.batch = pp.batch;
    p.total_tokens = pp.total_tokens;
    p.heads = pp.heads;
    p.head_dim = pp.head_dim;
    p.block = block;
    p.window = window;
    p.scale = float(1.0 / std::sqrt(double(pp.head_dim)));
    return p;
}

// Rotated q and k (the rotary entry points) follow the attention workspace.
struct RopeLayout {
    size_t qr, kr, total;
};

RopeLayout rope_layout(const ba_problem &P, size_t base_total)
{
    const size_t esz = P.dtype == BA_BF16 ? 2 : 4;
    const size_t bytes = align256(size_t(P.total_tokens) * size_t(P.heads) * size_t(P.head_dim) * esz);
    return RopeLayout{base_total, base_total + bytes, base_total + 2 * bytes};
}

ba_status check_rope(const ba_rope *r, const ba_problem &P)
{
    if (!r) return BA_ERR_INVALID_ARG;
    if (P.total_tokens == 0) return BA_OK;
    if (!r->cos || !r->sin || !aligned(r->cos, 16) || !aligned(r->sin, 16) || r->rows < 1 || P.head_dim % 2)
        return BA_ERR_INVALID_ARG;
    if (!r->q_rot != !r->k_rot) return BA_ERR_INVALID_ARG;
    if (r->q_rot && (!aligned(r->q_rot, 16) || !aligned(r->k_rot, 16))) return BA_ERR_INVALID_ARG;
    return BA_OK;
}

// Rotated copies in the caller's buffers (both set) or in the workspace.
bool caller_rotated(const ba_rope *r) { return r && r->q_rot && r->k_rot; }

void set_rope(Problem &p, const ba_rope *r)
{
    p.rope_cos = r->cos;
    p.rope_sin = r->sin;
    p.rope_rows = r->rows;
}

thread_local cudaEvent_t t_prof[3][2] = {{nullptr, nullptr}, {nullptr, nullptr}, {nullptr, nullptr}};

cudaError_t prof_mark(int which, int edge, cudaStream_t stream)
{
    cudaEvent_t e = t_prof[which][edge];
    return e ? cudaEventRecord(e, stream) : cudaSuccess;
}

#define BA_TRY(...)                                                                                       \
    do {                                                                                                  \
        if ((__VA_ARGS__) != cudaSuccess) return BA_ERR_CUDA;                                             \
    } while (0)

// ba_fwd (rope == nullptr) and ba_rope_fwd.
ba_status fwd_impl(const ba_problem *pp, const ba_rope *rope, const void *q, const void *k, const void *v,
                   const int32_t *seq_offsets, int32_t block, int32_t window, const uint8_t *skip, void *out,
                   float *lse, void *workspace, size_t workspace_bytes, ba_stream_t stream_, bool with_rope)
{
    ba_status st = check_problem(pp, block, window);
    if (st != BA_OK) return st;
    const ba_problem &P = *pp;
    const int64_t T = P.total_tokens;
    if (!seq_offsets || !aligned(seq_offsets, 4) || !tensor_ok(q, T) || !tensor_ok(k, T) || !tensor_ok(v, T) ||
        !tensor_ok(out, T) || (T > 0 && (!lse || !aligned(lse, 4))))
        return BA_ERR_INVALID_ARG;
    if (with_rope && (st = check_rope(rope, P)) != BA_OK) return st;
    const WorkspaceLayout lay = workspace_layout(P.batch, T, P.heads, P.head_dim, false);
    const RopeLayout rl = rope_layout(P, lay.total);
    const size_t need = with_rope && !caller_rotated(rope) ? rl.total : lay.total;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return BA_ERR_INVALID_ARG;
    int num_sms = 0, cc = 0;
    if (!device_info(num_sms, cc)) return BA_ERR_CUDA;
    if (P.dtype == BA_BF16 && cc != 10) return BA_ERR_UNSUPPORTED;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);

    Problem p = make_problem(P, seq_offsets, skip, block, window, workspace, lay);
    BA_TRY(launch_worklist(p, stream));
    if (T == 0) return BA_OK;
    const size_t esz = P.dtype == BA_BF16 ? 2 : 4;
    BA_TRY(launch_skip_fwd(p, esz, v, out, lse, stream));
    if (with_rope) {
        // the attention kernels read rotated copies of q and k
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        void *qr = caller_rotated(rope) ? rope->q_rot : ws + rl.qr;
        void *kr = caller_rotated(rope) ? rope->k_rot : ws + rl.kr;
        set_rope(p, rope);
        BA_TRY(launch_rope_rows(p, esz, false, q, k, qr, kr, num_sms, stream));
        q = qr;
        k = kr;
    }
    if (P.dtype == BA_F32) {
        BA_TRY(prof_mark(0, 0, stream));
        BA_TRY(launch_fwd_f32(p, static_cast<const float *>(q), static_cast<const float *>(k),
                              static_cast<const float *>(v), static_cast<float *>(out), lse, num_sms, stream));
        BA_TRY(prof_mark(0, 1, stream));
        return BA_OK;
    }
    CUtensorMap tq, tk, tv, to;
    if (!encode_bf16_rows(&tq, q, T, P.heads, P.head_dim) || !encode_bf16_rows(&tk, k, T, P.heads, P.head_dim) ||
        !encode_bf16_rows(&tv, v, T, P.heads, P.head_dim) || !encode_bf16_rows(&to, out, T, P.heads, P.head_dim))
        return BA_ERR_CUDA;
    BA_TRY(prof_mark(0, 0, stream));
    if (P.head_dim == 64) BA_TRY(launch_fwd_bf16_sm100<64, kSoftmax>(tq, tk, tv, to, p, out, lse, num_sms, stream));
    else BA_TRY(launch_fwd_bf16_sm100<128, kSoftmax>(tq, tk, tv, to, p, out, lse, num_sms, stream));
    BA_TRY(prof_mark(0, 1, stream));
    return BA_OK;
}

// ba_bwd (rope == nullptr) and ba_rope_bwd.
ba_status bwd_impl(const ba_problem *pp, const ba_rope *rope, const void *q, const void *k, const void *v,
                   const void *out, const float *lse, const void *dout, const int32_t *seq_offsets, int32_t block,
                   int32_t window, const uint8_t *skip, void *dq, void *dk, void *dv, void *workspace,
                   size_t workspace_bytes, ba_stream_t stream_, bool with_rope)
{
    ba_status st = check_problem(pp, block, window);
    if (st != BA_OK) return st;
    const ba_problem &P = *pp;
    const int64_t T = P.total_tokens;
    if (!seq_offsets || !aligned(seq_offsets, 4) || !tensor_ok(q, T) || !tensor_ok(k, T) || !tensor_ok(v, T) ||
        !tensor_ok(out, T) || !tensor_ok(dout, T) || !tensor_ok(dq, T) || !tensor_ok(dk, T) || !tensor_ok(dv, T) ||
        (T > 0 && (!lse || !aligned(lse, 4))))
        return BA_ERR_INVALID_ARG;
    if (with_rope && (st = check_rope(rope, P)) != BA_OK) return st;
    const bool bf16 = P.dtype == BA_BF16;
    const bool fused = fused_backward(P, block, window, with_rope);
    const WorkspaceLayout lay = bwd_layout(P, block, window, with_rope);
    const RopeLayout rl = rope_layout(P, lay.total);
    const size_t need = with_rope && !caller_rotated(rope) ? rl.total : lay.total;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return BA_ERR_INVALID_ARG;
    int num_sms = 0, cc = 0;
    if (!device_info(num_sms, cc)) return BA_ERR_CUDA;
    if (bf16 && cc != 10) return BA_ERR_UNSUPPORTED;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);

    Problem p = make_problem(P, seq_offsets, skip, block, window, workspace, lay);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *delta = reinterpret_cast<float *>(ws + lay.delta);
    float *nlse2 = reinterpret_cast<float *>(ws + lay.nlse2);
    BA_TRY(launch_worklist(p, stream));
    if (T == 0) return BA_OK;
    const size_t esz = bf16 ? 2 : 4;
    BA_TRY(launch_skip_bwd(p, esz, dout, dq, dk, dv, stream));
    if (with_rope) {
        // the rotated q and k the forward used: the caller's saved copies, or
        // recomputed here; p.rope_* also tells the bf16 dQ and dK/dV epilogues to
        // turn dq and dk back
        set_rope(p, rope);
        if (caller_rotated(rope)) {
            q = rope->q_rot;
            k = rope->k_rot;
        } else {
            BA_TRY(launch_rope_rows(p, esz, false, q, k, ws + rl.qr, ws + rl.kr, num_sms, stream));
            q = ws + rl.qr;
            k = ws + rl.kr;
        }
    }
    if (!bf16) {
        BA_TRY(launch_bwd_pre<float>(p, out, dout, delta, num_sms, stream));
        BA_TRY(prof_mark(1, 0, stream));
        BA_TRY(launch_bwd_f32(p, static_cast<const float *>(q), static_cast<const float *>(k),
                              static_cast<const float *>(v), static_cast<const float *>(dout), lse, delta,
                              static_cast<float *>(dq), static_cast<float *>(dk), static_cast<float *>(dv), num_sms,
                              stream));
        BA_TRY(prof_mark(2, 1, stream));
        if (with_rope) BA_TRY(launch_rope_rows(p, esz, true, dq, dk, dq, dk, num_sms, stream));
        return BA_OK;
    }
    CUtensorMap tq, tk, tv, tdo, to, tdk, tdv, tqt, tdot, tkt, tdq;
    if (!encode_bf16_rows(&tq, q, T, P.heads, P.head_dim) || !encode_bf16_rows(&tk, k, T, P.heads, P.head_dim) ||
        !encode_bf16_rows(&tv, v, T, P.heads, P.head_dim) || !encode_bf16_rows(&tdo, dout, T, P.heads, P.head_dim) ||
        !encode_bf16_rows(&to, out, T, P.heads, P.head_dim) || !encode_bf16_rows(&tdk, dk, T, P.heads, P.head_dim) ||
        !encode_bf16_rows(&tdv, dv, T, P.heads, P.head_dim) ||
        (fused && !encode_bf16_rows(&tdq, dq, T, P.heads, P.head_dim)) ||
        !stage_query_tails(P, seq_offsets, skip, q, dout, ws, lay, tqt, tdot, stream, fused ? k : nullptr, &tkt))
        return BA_ERR_CUDA;
    if (fused) {
        // one pass for dQ, dK and dV; its per-row statistics first (profile slot 1)
        BA_TRY(prof_mark(1, 0, stream));
        BA_TRY(launch_bwd_stats(p, out, dout, lse, delta, nlse2, num_sms, stream));
        BA_TRY(prof_mark(1, 1, stream));
        BA_TRY(prof_mark(2, 0, stream));
        if (P.head_dim == 64)
            BA_TRY(launch_bwd_fused_sm100<64>(tq, tk, tv, tdo, tdk, tdv, tqt, tdot, tkt, tdq, p, nlse2, delta, dq, dk,
                                              dv, num_sms, stream));
        else
            BA_TRY(launch_bwd_fused_sm100<128>(tq, tk, tv, tdo, tdk, tdv, tqt, tdot, tkt, tdq, p, nlse2, delta, dq,
                                               dk, dv, num_sms, stream));
        BA_TRY(prof_mark(2, 1, stream));
        return BA_OK;
    }
    BA_TRY(prof_mark(1, 0, stream));
    if (P.head_dim == 64)
        BA_TRY(launch_bwd_dq_sm100<64, kSoftmax>(tq, tk, tv, tdo, to, p, lse, delta, nlse2, dq, num_sms, stream));
    else
        BA_TRY(launch_bwd_dq_sm100<128, kSoftmax>(tq, tk, tv, tdo, to, p, lse, delta, nlse2, dq, num_sms, stream));
    BA_TRY(prof_mark(1, 1, stream));
    BA_TRY(prof_mark(2, 0, stream));
    if (P.head_dim == 64)
        BA_TRY(launch_bwd_dkdv_sm100<64, kSoftmax>(tq, tk, tv, tdo, tdk, tdv, tqt, tdot, p, nlse2, delta, dk, dv,
                                                   num_sms, stream));
    else
        BA_TRY(launch_bwd_dkdv_sm100<128, kSoftmax>(tq, tk, tv, tdo, tdk, tdv, tqt, tdot, p, nlse2, delta, dk, dv,
                                                    num_sms, stream));
    BA_TRY(prof_mark(2, 1, stream));
    return BA_OK;
}

// ba_gdpa_fwd / ba_gdpa_bwd: the block-attention kernels with the softmax
// replaced by the activation (no lse, no Delta).
template <int A>
cudaError_t gdpa_launch(bool bwd, int D, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                        const CUtensorMap &tdo, const CUtensorMap &to, const CUtensorMap &tdk, const CUtensorMap &tdv,
                        const CUtensorMap &tqt, const CUtensorMap &tdot, const Problem &p, void *out, void *dq, void *dk, void *dv, int num_sms, cudaStream_t stream)
{
    cudaError_t e;
    if (!bwd) {
        if ((e = prof_mark(0, 0, stream)) != cudaSuccess) return e;
        e = D == 64 ? launch_fwd_bf16_sm100<64, A>(tq, tk, tv, to, p, out, nullptr, num_sms, stream)
                    : launch_fwd_bf16_sm100<128, A>(tq, tk, tv, to, p, out, nullptr, num_sms, stream);
        if (e != cudaSuccess) return e;
        return prof_mark(0, 1, stream);
    }
    if ((e = prof_mark(1, 0, stream)) != cudaSuccess) return e;
    e = D == 64 ? launch_bwd_dq_sm100<64, A>(tq, tk, tv, tdo, to, p, nullptr, nullptr, nullptr, dq, num_sms, stream)
                : launch_bwd_dq_sm100<128, A>(tq, tk, tv, tdo, to, p, nullptr, nullptr, nullptr, dq, num_sms, stream);
    if (e != cudaSuccess) return e;
    if ((e = prof_mark(1, 1, stream)) != cudaSuccess || (e = prof_mark(2, 0, stream)) != cudaSuccess) return e;
    e = D == 64 ? launch_bwd_dkdv_sm100<64, A>(tq, tk, tv, tdo, tdk, tdv, tqt, tdot, p, nullptr, nullptr, dk, dv,
                                               num_sms, stream)
                : launch_bwd_dkdv_sm100<128, A>(tq, tk, tv, tdo, tdk, tdv, tqt, tdot, p, nullptr, nullptr, dk, dv,
                                                num_sms, stream);
    if (e != cudaSuccess) return e;
    return prof_mark(2, 1, stream);
}

ba_status gdpa_impl(bool bwd, const ba_problem *pp, ba_activation act, const void *q, const void *k, const void *v,
                    const void *dout, const int32_t *seq_offsets, int32_t block, int32_t window, void *out, void *dq,
                    void *dk, void *dv, void *workspace, size_t workspace_bytes, ba_stream_t stream_)
{
    ba_status st = check_problem(pp, block, window);
    if (st != BA_OK) return st;
    if (act != BA_ACT_GELU && act != BA_ACT_SILU) return BA_ERR_INVALID_ARG;
    const ba_problem &P = *pp;
    const int64_t T = P.total_tokens;
    if (!seq_offsets || !aligned(seq_offsets, 4) || !tensor_ok(q, T) || !tensor_ok(k, T) || !tensor_ok(v, T))
        return BA_ERR_INVALID_ARG;
    if (!bwd && !tensor_ok(out, T)) return BA_ERR_INVALID_ARG;
    if (bwd && (!tensor_ok(dout, T) || !tensor_ok(dq, T) || !tensor_ok(dk, T) || !tensor_ok(dv, T)))
        return BA_ERR_INVALID_ARG;
    if (P.dtype != BA_BF16) return BA_ERR_UNSUPPORTED;
    const WorkspaceLayout lay = workspace_layout(P.batch, T, P.heads, P.head_dim, false, true);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < lay.total) return BA_ERR_INVALID_ARG;
    int num_sms = 0, cc = 0;
    if (!device_info(num_sms, cc)) return BA_ERR_CUDA;
    if (cc != 10) return BA_ERR_UNSUPPORTED;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    Problem p = make_problem(P, seq_offsets, nullptr, block, window, workspace, lay);
    BA_TRY(launch_worklist(p, stream));
    if (T == 0) return BA_OK;
    CUtensorMap tq, tk, tv, tdo, to, tdk, tdv, tqt, tdot;
    if (!encode_bf16_rows(&tq, q, T, P.heads, P.head_dim) || !encode_bf16_rows(&tk, k, T, P.heads, P.head_dim) ||
        !encode_bf16_rows(&tv, v, T, P.heads, P.head_dim))
        return BA_ERR_CUDA;
    if (!bwd && !encode_bf16_rows(&to, out, T, P.heads, P.head_dim)) return BA_ERR_CUDA;
    if (bwd && (!encode_bf16_rows(&tdo, dout, T, P.heads, P.head_dim) ||
                !encode_bf16_rows(&tdk, dk, T, P.heads, P.head_dim) ||
                !encode_bf16_rows(&tdv, dv, T, P.heads, P.head_dim) ||
                !stage_query_tails(P, seq_offsets, nullptr, q, dout, static_cast<uint8_t *>(workspace), lay, tqt,
                                   tdot, stream)))
        return BA_ERR_CUDA;
    if (bwd) to = tdo; // the dQ pass reads no `out` here; any valid map fills the slot
    else tdo = tdk = tdv = tqt = tdot = to;
    const cudaError_t e = act == BA_ACT_GELU
                              ? gdpa_launch<kGelu>(bwd, P.head_dim, tq, tk, tv, tdo, to, tdk, tdv, tqt, tdot, p, out,
                                                   dq, dk, dv, num_sms, stream)
                              : gdpa_launch<kSilu>(bwd, P.head_dim, tq, tk, tv, tdo, to, tdk, tdv, tqt, tdot, p, out,
                                                   dq, dk, dv, num_sms, stream);
    return e == cudaSuccess ? BA_OK : BA_ERR_CUDA;
}

// Cross-attention GDPA: query tiles against their example's key/value set
// (forward, dQ pass), key tiles against their example's query set (dK/dV
// pass); rows whose other side is empty get zeros.
ba_status gdpa_cross_impl(bool bwd, const ba_problem *pp, int32_t kv_total, ba_activation act, const void *q,
                          const void *k, const void *v, const void *dout, const int32_t *q_offsets,
                          const int32_t *kv_offsets, void *out, void *dq, void *dk, void *dv, void *workspace,
                          size_t workspace_bytes, ba_stream_t stream_)
{
    ba_status st = check_problem(pp, 1, 1);
    if (st != BA_OK) return st;
    if (act != BA_ACT_GELU && act != BA_ACT_SILU) return BA_ERR_INVALID_ARG;
    const ba_problem &P = *pp;
    const int64_t Tq = P.total_tokens, Tk = kv_total;
    if (kv_total < 0 || (P.batch == 0 && kv_total != 0)) return BA_ERR_INVALID_ARG;
    if (max_tiles(P.batch, Tk) * P.heads > INT32_MAX) return BA_ERR_UNSUPPORTED;
    if (!q_offsets || !aligned(q_offsets, 4) || !kv_offsets || !aligned(kv_offsets, 4) || !tensor_ok(q, Tq) ||
        !tensor_ok(k, Tk) || !tensor_ok(v, Tk))
        return BA_ERR_INVALID_ARG;
    if (!bwd && !tensor_ok(out, Tq)) return BA_ERR_INVALID_ARG;
    if (bwd && (!tensor_ok(dout, Tq) || !tensor_ok(dq, Tq) || !tensor_ok(dk, Tk) || !tensor_ok(dv, Tk)))
        return BA_ERR_INVALID_ARG;
    if (P.dtype != BA_BF16) return BA_ERR_UNSUPPORTED;
    const WorkspaceLayout lay = workspace_layout(P.batch, Tq > Tk ? Tq : Tk, P.heads, P.head_dim, false, true);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < lay.total) return BA_ERR_INVALID_ARG;
    int num_sms = 0, cc = 0;
    if (!device_info(num_sms, cc)) return BA_ERR_CUDA;
    if (cc != 10) return BA_ERR_UNSUPPORTED;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const size_t row_bytes = size_t(P.heads) * P.head_dim * 2;
    // the query-tile side: tables over the query sets, each paired with its key/value set
    Problem pq = make_problem(P, q_offsets, nullptr, 1, 1, workspace, lay);
    pq.other_offsets = kv_offsets;
    BA_TRY(launch_worklist(pq, stream));
    if (Tq > 0) BA_TRY(launch_zero_unpaired_rows(q_offsets, kv_offsets, P.batch, row_bytes, bwd ? dq : out, nullptr,
                                                 stream));
    if (Tq == 0 || Tk == 0) {
        if (bwd && Tk > 0)
            BA_TRY(launch_zero_unpaired_rows(kv_offsets, q_offsets, P.batch, row_bytes, dk, dv, stream));
        return BA_OK;
    }
    CUtensorMap tq, tk, tv, tdo, to, tdk, tdv, tqt, tdot;
    if (!encode_bf16_rows(&tq, q, Tq, P.heads, P.head_dim) || !encode_bf16_rows(&tk, k, Tk, P.heads, P.head_dim) ||
        !encode_bf16_rows(&tv, v, Tk, P.heads, P.head_dim))
        return BA_ERR_CUDA;
    const auto run = [&](auto act_c, bool dkdv_pass, const Problem &p) -> cudaError_t {
        constexpr int A = decltype(act_c)::value;
        const int D = P.head_dim;
        if (!bwd) {
            cudaError_t e = prof_mark(0, 0, stream);
            if (e == cudaSuccess)
                e = D == 64 ? launch_fwd_bf16_sm100<64, A>(tq, tk, tv, to, p, out, nullptr, num_sms, stream)
                            : launch_fwd_bf16_sm100<128, A>(tq, tk, tv, to, p, out, nullptr, num_sms, stream);
            return e == cudaSuccess ? prof_mark(0, 1, stream) : e;
        }
        const int w = dkdv_pass ? 2 : 1;
        cudaError_t e = prof_mark(w, 0, stream);
        if (e != cudaSuccess) return e;
        if (!dkdv_pass)
            e = D == 64 ? launch_bwd_dq_sm100<64, A>(tq, tk, tv, tdo, tdo, p, nullptr, nullptr, nullptr, dq, num_sms,
                                                     stream)
                        : launch_bwd_dq_sm100<128, A>(tq, tk, tv, tdo, tdo, p, nullptr, nullptr, nullptr, dq, num_sms,
                                                      stream);
        else
            e = D == 64 ? launch_bwd_dkdv_sm100<64, A>(tq, tk, tv, tdo, tdk, tdv, tqt, tdot, p, nullptr, nullptr, dk,
                                                       dv, num_sms, stream)
                        : launch_bwd_dkdv_sm100<128, A>(tq, tk, tv, tdo, tdk, tdv, tqt, tdot, p, nullptr, nullptr, dk,
                                                        dv, num_sms, stream);
        return e == cudaSuccess ? prof_mark(w, 1, stream) : e;
    };
    const auto run_act = [&](bool dkdv_pass, const Problem &p) -> cudaError_t {
        return act == BA_ACT_GELU ? run(std::integral_constant<int, kGelu>{}, dkdv_pass, p)
                                  : run(std::integral_constant<int, kSilu>{}, dkdv_pass, p);
    };
    if (!bwd) {
        if (!encode_bf16_rows(&to, out, Tq, P.heads, P.head_dim)) return BA_ERR_CUDA;
        BA_TRY(run_act(false, pq));
        return BA_OK;
    }
    if (!encode_bf16_rows(&tdo, dout, Tq, P.heads, P.head_dim) || !encode_bf16_rows(&tdk, dk, Tk, P.heads, P.head_dim) ||
        !encode_bf16_rows(&tdv, dv, Tk, P.heads, P.head_dim) ||
        !stage_query_tails(P, q_offsets, nullptr, q, dout, static_cast<uint8_t *>(workspace), lay, tqt, tdot, stream))
        return BA_ERR_CUDA;
    BA_TRY(run_act(false, pq));
    // the key-tile side: tables over the key/value sets, each paired with its query set (the
    // dQ pass's status word is kept)
    ba_problem Pk = P;
    Pk.total_tokens = int32_t(Tk);
    Problem pk = make_problem(Pk, kv_offsets, nullptr, 1, 1, workspace, lay);
    pk.other_offsets = q_offsets;
    BA_TRY(launch_worklist(pk, stream, false));
    BA_TRY(launch_zero_unpaired_rows(kv_offsets, q_offsets, P.batch, row_bytes, dk, dv, stream));
    BA_TRY(run_act(true, pk));
    return BA_OK;
}

// MXFP8 operands in the workspace after the forward's own regions: E4M3 q and
// k [T, H, D], then their scale bytes [T, heads_pad, D / 32].
struct MxLayout {
    size_t q8, k8, qs, ks, total;
};

MxLayout mx_layout(const ba_problem &P, size_t base_total)
{
    const size_t e = align256(size_t(P.total_tokens) * size_t(P.heads) * size_t(P.head_dim));
    const size_t sc = align256(size_t(P.total_tokens) * size_t((P.heads + 3) / 4 * 4) * size_t(P.head_dim / 32));
    return MxLayout{base_total, base_total + e, base_total + 2 * e, base_total + 2 * e + sc, base_total + 2 * e + 2 * sc};
}

ba_status mx_fwd_impl(const ba_problem *pp, const void *q, const void *k, const void *v, const int32_t *seq_offsets,
                      int32_t block, int32_t window, const uint8_t *skip, void *out, float *lse, void *workspace,
                      size_t workspace_bytes, ba_stream_t stream_)
{
    ba_status st = check_problem(pp, block, window);
    if (st != BA_OK) return st;
    const ba_problem &P = *pp;
    const int64_t T = P.total_tokens;
    if (!seq_offsets || !aligned(seq_offsets, 4) || !tensor_ok(q, T) || !tensor_ok(k, T) || !tensor_ok(v, T) ||
        !tensor_ok(out, T) || (T > 0 && (!lse || !aligned(lse, 4))))
        return BA_ERR_INVALID_ARG;
    if (P.dtype != BA_BF16 || P.head_dim != 128) return BA_ERR_UNSUPPORTED;
    const WorkspaceLayout lay = workspace_layout(P.batch, T, P.heads, P.head_dim, false);
    const MxLayout ml = mx_layout(P, lay.total);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < ml.total) return BA_ERR_INVALID_ARG;
    int num_sms = 0, cc = 0;
    if (!device_info(num_sms, cc)) return BA_ERR_CUDA;
    if (cc != 10) return BA_ERR_UNSUPPORTED;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    Problem p = make_problem(P, seq_offsets, skip, block, window, workspace, lay);
    BA_TRY(launch_worklist(p, stream));
    if (T == 0) return BA_OK;
    BA_TRY(launch_skip_fwd(p, 2, v, out, lse, stream));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    BA_TRY(launch_mx_quantize(q, T, P.heads, P.head_dim, ws + ml.q8, ws + ml.qs, num_sms, stream));
    BA_TRY(launch_mx_quantize(k, T, P.heads, P.head_dim, ws + ml.k8, ws + ml.ks, num_sms, stream));
    const int64_t row8 = int64_t(P.heads) * P.head_dim, rows = int64_t((P.heads + 3) / 4 * 4) * 4;
    CUtensorMap tq, tk, tv, to, tqs, tks;
    if (!encode_u8_rows(&tq, ws + ml.q8, T, row8, 128, true) || !encode_u8_rows(&tk, ws + ml.k8, T, row8, 128, true) ||
        !encode_u8_rows(&tqs, ws + ml.qs, T, rows, 16, false) || !encode_u8_rows(&tks, ws + ml.ks, T, rows, 16, false) ||
        !encode_bf16_rows(&tv, v, T, P.heads, P.head_dim) || !encode_bf16_rows(&to, out, T, P.heads, P.head_dim))
        return BA_ERR_CUDA;
    BA_TRY(prof_mark(0, 0, stream));
    BA_TRY(launch_fwd_bf16_sm100<128, kSoftmax>(tq, tk, tv, to, p, out, lse, num_sms, stream, &tqs, &tks));
    BA_TRY(prof_mark(0, 1, stream));
    return BA_OK;
}

// ba_mx_bwd: the bf16 backward on the MX round trips of q and k (the
// operands the MXFP8 forward's score product used), kept in the workspace
// after the backward's own regions (so that the status word stays first).
size_t mx_bwd_operand_bytes(const ba_problem &P)
{
    return align256(size_t(P.total_tokens) * size_t(P.heads) * size_t(P.head_dim) * 2);
}

ba_status mx_bwd_impl(const ba_problem *pp, const void *q, const void *k, const void *v, const void *out,
                      const float *lse, const void *dout, const int32_t *seq_offsets, int32_t block, int32_t window,
                      const uint8_t *skip, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                      ba_stream_t stream_)
{
    ba_status st = check_problem(pp, block, window);
    if (st != BA_OK) return st;
    const ba_problem &P = *pp;
    const int64_t T = P.total_tokens;
    if (!seq_offsets || !aligned(seq_offsets, 4) || !tensor_ok(q, T) || !tensor_ok(k, T) || !tensor_ok(v, T) ||
        !tensor_ok(out, T) || !tensor_ok(dout, T) || !tensor_ok(dq, T) || !tensor_ok(dk, T) || !tensor_ok(dv, T) ||
        (T > 0 && (!lse || !aligned(lse, 4))))
        return BA_ERR_INVALID_ARG;
    if (P.dtype != BA_BF16 || P.head_dim != 128) return BA_ERR_UNSUPPORTED;
    const size_t rt = mx_bwd_operand_bytes(P);
    const size_t base = bwd_layout(P, block, window, false).total;
    const size_t need = base + 2 * rt;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return BA_ERR_INVALID_ARG;
    int num_sms = 0, cc = 0;
    if (!device_info(num_sms, cc)) return BA_ERR_CUDA;
    if (cc != 10) return BA_ERR_UNSUPPORTED;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    uint8_t *qr = static_cast<uint8_t *>(workspace) + base, *kr = qr + rt;
    const int64_t elems = T * P.heads * P.head_dim;
    BA_TRY(launch_mx_round_trip(q, elems, qr, num_sms, stream));
    BA_TRY(launch_mx_round_trip(k, elems, kr, num_sms, stream));
    return bwd_impl(pp, nullptr, qr, kr, v, out, lse, dout, seq_offsets, block, window, skip, dq, dk, dv, workspace,
                    workspace_bytes, stream_, false);
}

} // namespace

extern "C" {

size_t ba_fwd_workspace_size(const ba_problem *p, int32_t block, int32_t window)
{
    if (check_problem(p, block, window) == BA_ERR_INVALID_ARG) return 0;
    return workspace_layout(p->batch, p->total_tokens, p->heads, p->head_dim, false).total;
}

size_t ba_bwd_workspace_size(const ba_problem *p, int32_t block, int32_t window)
{
    if (check_problem(p, block, window) == BA_ERR_INVALID_ARG) return 0;
    return bwd_layout(*p, block, window, false).total;
}

ba_status ba_fwd(const ba_problem *p, const void *q, const void *k, const void *v, const int32_t *seq_offsets,
                 int32_t block, int32_t window, const uint8_t *skip, void *out, float *lse, void *workspace,
                 size_t workspace_bytes, ba_stream_t stream)
{
    return fwd_impl(p, nullptr, q, k, v, seq_offsets, block, window, skip, out, lse, workspace, workspace_bytes,
                    stream, false);
}

ba_status ba_bwd(const ba_problem *p, const void *q, const void *k, const void *v, const void *out,
                 const float *lse, const void *dout, const int32_t *seq_offsets, int32_t block, int32_t window,
                 const uint8_t *skip, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                 ba_stream_t stream)
{
    return bwd_impl(p, nullptr, q, k, v, out, lse, dout, seq_offsets, block, window, skip, dq, dk, dv, workspace,
                    workspace_bytes, stream, false);
}

// Rotary position embedding on q and k, then block attention.
size_t ba_rope_fwd_workspace_size(const ba_problem *p, int32_t block, int32_t window)
{
    const size_t base = ba_fwd_workspace_size(p, block, window);
    return base ? rope_layout(*p, base).total : 0;
}

size_t ba_rope_bwd_workspace_size(const ba_problem *p, int32_t block, int32_t window)
{
    const size_t base = ba_bwd_workspace_size(p, block, window);
    return base ? rope_layout(*p, base).total : 0;
}

ba_status ba_rope_fwd(const ba_problem *p, const ba_rope *rope, const void *q, const void *k, const void *v,
                      const int32_t *seq_offsets, int32_t block, int32_t window, const uint8_t *skip, void *out,
                      float *lse, void *workspace, size_t workspace_bytes, ba_stream_t stream)
{
    return fwd_impl(p, rope, q, k, v, seq_offsets, block, window, skip, out, lse, workspace, workspace_bytes,
                    stream, true);
}

ba_status ba_rope_bwd(const ba_problem *p, const ba_rope *rope, const void *q, const void *k, const void *v,
                      const void *out, const float *lse, const void *dout, const int32_t *seq_offsets,
                      int32_t block, int32_t window, const uint8_t *skip, void *dq, void *dk, void *dv,
                      void *workspace, size_t workspace_bytes, ba_stream_t stream)
{
    return bwd_impl(p, rope, q, k, v, out, lse, dout, seq_offsets, block, window, skip, dq, dk, dv, workspace,
                    workspace_bytes, stream, true);
}

// Sliding-window attention: the block rule with block = 1 (one token per block),
// so window counts tokens.
size_t ba_swa_fwd_workspace_size(const ba_problem *p, int32_t window_tokens)
{
    return ba_fwd_workspace_size(p, 1, window_tokens);
}

size_t ba_swa_bwd_workspace_size(const ba_problem *p, int32_t window_tokens)
{
    return ba_bwd_workspace_size(p, 1, window_tokens);
}

ba_status ba_swa_fwd(const ba_problem *p, const void *q, const void *k, const void *v, const int32_t *seq_offsets,
                     int32_t window_tokens, const uint8_t *skip, void *out, float *lse, void *workspace,
                     size_t workspace_bytes, ba_stream_t stream)
{
    return ba_fwd(p, q, k, v, seq_offsets, 1, window_tokens, skip, out, lse, workspace, workspace_bytes, stream);
}

ba_status ba_swa_bwd(const ba_problem *p, const void *q, const void *k, const void *v, const void *out,
                     const float *lse, const void *dout, const int32_t *seq_offsets, int32_t window_tokens,
                     const uint8_t *skip, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                     ba_stream_t stream)
{
    return ba_bwd(p, q, k, v, out, lse, dout, seq_offsets, 1, window_tokens, skip, dq, dk, dv, workspace,
                  workspace_bytes, stream);
}

size_t ba_gdpa_workspace_size(const ba_problem *p, int32_t block, int32_t window)
{
    if (check_problem(p, block, window) == BA_ERR_INVALID_ARG) return 0;
    return workspace_layout(p->batch, p->total_tokens, p->heads, p->head_dim, false, true).total;
}

ba_status ba_gdpa_fwd(const ba_problem *p, ba_activation act, const void *q, const void *k, const void *v,
                      const int32_t *seq_offsets, int32_t block, int32_t window, void *out, void *workspace,
                      size_t workspace_bytes, ba_stream_t stream)
{
    return gdpa_impl(false, p, act, q, k, v, nullptr, seq_offsets, block, window, out, nullptr, nullptr, nullptr,
                     workspace, workspace_bytes, stream);
}

ba_status ba_gdpa_bwd(const ba_problem *p, ba_activation act, const void *q, const void *k, const void *v,
                      const void *dout, const int32_t *seq_offsets, int32_t block, int32_t window, void *dq, void *dk,
                      void *dv, void *workspace, size_t workspace_bytes, ba_stream_t stream)
{
    return gdpa_impl(true, p, act, q, k, v, dout, seq_offsets, block, window, nullptr, dq, dk, dv, workspace,
                     workspace_bytes, stream);
}

size_t ba_gdpa_cross_workspace_size(const ba_problem *p, int32_t kv_total_tokens)
{
    if (check_problem(p, 1, 1) == BA_ERR_INVALID_ARG || kv_total_tokens < 0) return 0;
    const int64_t t = p->total_tokens > kv_total_tokens ? p->total_tokens : kv_total_tokens;
    return workspace_layout(p->batch, t, p->heads, p->head_dim, false, true).total;
}

ba_status ba_gdpa_cross_fwd(const ba_problem *p, int32_t kv_total_tokens, ba_activation act, const void *q,
                            const void *k, const void *v, const int32_t *q_offsets, const int32_t *kv_offsets,
                            void *out, void *workspace, size_t workspace_bytes, ba_stream_t stream)
{
    return gdpa_cross_impl(false, p, kv_total_tokens, act, q, k, v, nullptr, q_offsets, kv_offsets, out, nullptr,
                           nullptr, nullptr, workspace, workspace_bytes, stream);
}

ba_status ba_gdpa_cross_bwd(const ba_problem *p, int32_t kv_total_tokens, ba_activation act, const void *q,
                            const void *k, const void *v, const void *dout, const int32_t *q_offsets,
                            const int32_t *kv_offsets, void *dq, void *dk, void *dv, void *workspace,
                            size_t workspace_bytes, ba_stream_t stream)
{
    return gdpa_cross_impl(true, p, kv_total_tokens, act, q, k, v, dout, q_offsets, kv_offsets, nullptr, dq, dk, dv,
                           workspace, workspace_bytes, stream);
}

ba_status ba_mx_quantize(const void *x, int64_t rows, int32_t heads, int32_t head_dim, void *elements,
                         void *scales, ba_stream_t stream)
{
    if (rows < 0 || heads < 1 || head_dim < 32 || head_dim % 32 || rows > (int64_t(1) << 40)) return BA_ERR_INVALID_ARG;
    if (rows > 0 && (!x || !elements || !scales || !aligned(x, 16) || !aligned(elements, 16)))
        return BA_ERR_INVALID_ARG;
    int num_sms = 0, cc = 0;
    if (rows > 0 && !device_info(num_sms, cc)) return BA_ERR_CUDA;
    BA_TRY(launch_mx_quantize(x, rows, heads, head_dim, elements, scales, num_sms,
                              reinterpret_cast<cudaStream_t>(stream)));
    return BA_OK;
}

size_t ba_mx_fwd_workspace_size(const ba_problem *p, int32_t block, int32_t window)
{
    const size_t base = ba_fwd_workspace_size(p, block, window);
    return base ? mx_layout(*p, base).total : 0;
}

ba_status ba_mx_fwd(const ba_problem *p, const void *q, const void *k, const void *v, const int32_t *seq_offsets,
                    int32_t block, int32_t window, const uint8_t *skip, void *out, float *lse, void *workspace,
                    size_t workspace_bytes, ba_stream_t stream)
{
    return mx_fwd_impl(p, q, k, v, seq_offsets, block, window, skip, out, lse, workspace, workspace_bytes, stream);
}

size_t ba_mx_bwd_workspace_size(const ba_problem *p, int32_t block, int32_t window)
{
    if (check_problem(p, block, window) == BA_ERR_INVALID_ARG) return 0;
    return 2 * mx_bwd_operand_bytes(*p) + bwd_layout(*p, block, window, false).total;
}

ba_status ba_mx_bwd(const ba_problem *p, const void *q, const void *k, const void *v, const void *out,
                    const float *lse, const void *dout, const int32_t *seq_offsets, int32_t block, int32_t window,
                    const uint8_t *skip, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                    ba_stream_t stream)
{
    return mx_bwd_impl(p, q, k, v, out, lse, dout, seq_offsets, block, window, skip, dq, dk, dv, workspace,
                       workspace_bytes, stream);
}

ba_status ba_device_status(const void *workspace, ba_stream_t stream_)
{
    if (!workspace) return BA_ERR_INVALID_ARG;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return BA_ERR_CUDA;
    if (word & kStatusTimeout) return BA_ERR_TIMEOUT;
    return (word & kStatusRopeRange) ? BA_ERR_INVALID_ARG : BA_OK;
}

ba_status ba_selftest_wait_timeout(void *workspace, size_t workspace_bytes, int32_t limit_us, ba_stream_t stream_)
{
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < 256 || limit_us < 1 || limit_us > 1000000)
        return BA_ERR_INVALID_ARG;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int *status = static_cast<int *>(workspace);
    if (cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return BA_ERR_CUDA;
    BA_TRY(launch_wait_selftest(status, uint64_t(limit_us) * 1000, stream));
    return BA_OK;
}

ba_status ba_selftest_activation(ba_activation act, const float *x, float *y, float *dy, int64_t n,
                                 ba_stream_t stream_)
{
    if (act != BA_ACT_GELU && act != BA_ACT_SILU) return BA_ERR_INVALID_ARG;
    if (n < 0 || (n > 0 && (!x || !y || !dy || !aligned(x, 4) || !aligned(y, 4) || !aligned(dy, 4))))
        return BA_ERR_INVALID_ARG;
    BA_TRY(launch_activation_selftest(act == BA_ACT_GELU ? kGelu : kSilu, x, y, dy, n,
                                      reinterpret_cast<cudaStream_t>(stream_)));
    return BA_OK;
}

ba_status ba_selftest_exp2(const float *x, float *y, int64_t n, ba_stream_t stream_)
{
    if (n < 0 || (n > 0 && (!x || !y || !aligned(x, 4) || !aligned(y, 4)))) return BA_ERR_INVALID_ARG;
    BA_TRY(launch_exp2_selftest(x, y, n, reinterpret_cast<cudaStream_t>(stream_)));
    return BA_OK;
}

ba_status ba_set_profile_events(int32_t which, void *start, void *stop)
{
    if (which < 0 || which > 2) return BA_ERR_INVALID_ARG;
    t_prof[which][0] = static_cast<cudaEvent_t>(start);
    t_prof[which][1] = static_cast<cudaEvent_t>(stop);
    return BA_OK;
}

const char *ba_status_string(ba_status s)
{
    switch (s) {
    case BA_OK: return "ok";
    case BA_ERR_INVALID_ARG: return "invalid argument";
    case BA_ERR_UNSUPPORTED: return "unsupported combination";
    case BA_ERR_CUDA: return "CUDA error";
    case BA_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

int32_t ba_version(void) { return 100; }

} // extern "C"
