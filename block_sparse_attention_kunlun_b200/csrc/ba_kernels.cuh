// Host-side launchers of the library's kernels (internal; the public C ABI is
// include/ba.h).
#pragma once

#include "ba_common.cuh"

#include <cuda.h>
#include <cuda_runtime.h>

namespace ba {

// Builds the work tables; reset_status = false keeps the status word (a second
// table for the same call).
cudaError_t launch_worklist(const Problem &p, cudaStream_t stream, bool reset_status = true);
// Cross-attention: zero the rows (of a, and of b unless nullptr) of examples whose other side is empty.
cudaError_t launch_zero_unpaired_rows(const int32_t *offs, const int32_t *other, int32_t batch, size_t row_bytes,
                                      void *a, void *b, cudaStream_t stream);
// The dK/dV pass's partial query tiles of a (q) and b (dout), zero-padded to 128 rows, into ta and tb;
// with c (k) and tc given, the partial key tiles too (the fused backward).
cudaError_t launch_stage_query_tails(const int32_t *offs, const uint8_t *skip, int32_t batch, size_t row_bytes,
                                     const void *a, const void *b, void *ta, void *tb, cudaStream_t stream,
                                     const void *c = nullptr, void *tc = nullptr);
// -Delta and -lse log2(e) of every row, [heads, total_tokens] (bf16 out and dout).
cudaError_t launch_bwd_stats(const Problem &p, const void *out, const void *dout, const float *lse,
                             float *neg_delta, float *nlse2, int num_sms, cudaStream_t stream);
cudaError_t launch_wait_selftest(int *status, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_exp2_selftest(const float *x, float *y, int64_t n, cudaStream_t stream);
cudaError_t launch_activation_selftest(int act, const float *x, float *y, float *dy, int64_t n, cudaStream_t stream);

template <typename T>
cudaError_t launch_bwd_pre(const Problem &p, const void *out, const void *dout, float *delta, int num_sms,
                           cudaStream_t stream);

cudaError_t launch_skip_fwd(const Problem &p, size_t elem_bytes, const void *v, void *out, float *lse,
                            cudaStream_t stream);
cudaError_t launch_skip_bwd(const Problem &p, size_t elem_bytes, const void *dout, void *dq, void *dk, void *dv,
                            cudaStream_t stream);

// Rotary embedding over every row of the batch: (a_out, b_out) = R(pos) (a_in, b_in),
// or with transpose = true R(pos)^T (in place when a_out == a_in, b_out == b_in).
cudaError_t launch_rope_rows(const Problem &p, size_t elem_bytes, bool transpose, const void *a_in, const void *b_in,
                             void *a_out, void *b_out, int num_sms, cudaStream_t stream);

// MX quantisation (E4M3 elements, E8M0 scales per 32 along head_dim) of a
// [rows, heads, head_dim] bf16 tensor; scales [rows, heads rounded up to 4, head_dim / 32].
cudaError_t launch_mx_quantize(const void *x, int64_t rows, int32_t heads, int32_t head_dim, void *elems,
                               void *scales, int num_sms, cudaStream_t stream);
// The same quantisation followed by dequantisation, bf16 to bf16 (elems a multiple of 32).
cudaError_t launch_mx_round_trip(const void *x, int64_t elems, void *y, int num_sms, cudaStream_t stream);

cudaError_t launch_fwd_f32(const Problem &p, const float *q, const float *k, const float *v, float *out, float *lse,
                           int num_sms, cudaStream_t stream);
cudaError_t launch_bwd_f32(const Problem &p, const float *q, const float *k, const float *v, const float *dout,
                           const float *lse, const float *delta, float *dq, float *dk, float *dv, int num_sms,
                           cudaStream_t stream);

// tqs / tks: the MXFP8 mode's maps of the Q and K scale words (q, k then E4M3);
// nullptr for the bf16 operands.
template <int D, int A>
cudaError_t launch_fwd_bf16_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const CUtensorMap &to, const Problem &p, void *out, float *lse, int num_sms,
                                  cudaStream_t stream, const CUtensorMap *tqs = nullptr,
                                  const CUtensorMap *tks = nullptr);

template <int D, int A>
cudaError_t launch_bwd_dq_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                const CUtensorMap &tdo, const CUtensorMap &to, const Problem &p, const float *lse,
                                float *neg_delta, float *nlse2, void *dq, int num_sms, cudaStream_t stream);
// The fused backward (masks with diagonal_tiles(block, window); block attention,
// no rotary): dQ, dK and dV in one pass. tkt maps the staged partial key tiles,
// tdq the dq output.
template <int D>
cudaError_t launch_bwd_fused_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                   const CUtensorMap &tdo, const CUtensorMap &tdk, const CUtensorMap &tdv,
                                   const CUtensorMap &tqt, const CUtensorMap &tdot, const CUtensorMap &tkt,
                                   const CUtensorMap &tdq, const Problem &p, const float *nlse2,
                                   const float *neg_delta, void *dq, void *dk, void *dv, int num_sms,
                                   cudaStream_t stream);
template <int D, int A>
cudaError_t launch_bwd_dkdv_sm100(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const CUtensorMap &tdo, const CUtensorMap &tdk, const CUtensorMap &tdv,
                                  const CUtensorMap &tqt, const CUtensorMap &tdot, const Problem &p,
                                  const float *nlse2, const float *neg_delta, void *dk, void *dv, int num_sms,
                                  cudaStream_t stream);

} // namespace ba
