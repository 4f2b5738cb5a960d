/*
 * ba.h -- block attention on NVIDIA B200 (sm_100a): the library's C ABI.
 *
 * Block attention is the sparse self-attention of Kunlun, the architecture
 * behind Meta's GEM ads model: attention over a long user-engagement history
 * restricted to blocks, so that cost grows linearly with sequence length for a
 * fixed window ("Meta Scales GEM Ads Model Across Platforms and Thousands of
 * GPUs", section "Kunlun changes how GEM scales"; "GEM (Meta)", section
 * "Custom kernels", BlockAttention; "Scaling Meta's Generative Ads Model (GEM)
 * for Ads Recommendations", section "Kunlun Architecture Details"). The pages
 * give no formula; this library fixes one rule and keeps it everywhere:
 *
 *   within one example, with 0-based local indices and blk(x) = x / block,
 *   query i sees key j  <=>  j <= i  and  blk(j) >= blk(i) - (window - 1).
 *
 * window = 1 is the pages' "independent 64-token blocks" case (block = 64),
 * causal inside each block. Blocks start at each example's first token.
 *
 * Batches are jagged ("GEM (Meta)", section "Training infrastructure":
 * histories of hundreds to tens of thousands of events, not padded): example
 * b owns rows seq_offsets[b] .. seq_offsets[b+1]-1 of every token-major
 * tensor.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - q, k, v, out, dout, dq, dk, dv: DEVICE pointers to contiguous row-major
 *    [total_tokens, heads, head_dim] tensors of the problem's dtype, 16-byte
 *    aligned. out/dq/dk/dv must not alias any input.
 *  - lse: DEVICE pointer, float32 [heads, total_tokens]: the natural log of
 *    sum_j exp(q_i . k_j / sqrt(head_dim)) over the visible keys.
 *  - seq_offsets: DEVICE pointer, int32 [batch + 1], seq_offsets[0] = 0,
 *    non-decreasing, seq_offsets[batch] = total_tokens (empty examples are
 *    allowed). This precondition is not checked on the device.
 *  - skip: DEVICE pointer to uint8 [batch] or NULL. A nonzero flag bypasses
 *    attention for that example (component skip, "Meta Scales GEM Ads Model
 *    ...", section "Kunlun changes how GEM scales"): out = v, lse = 0,
 *    dq = dk = 0, dv = dout, and none of its tiles is scheduled.
 *  - Scores are scaled by 1/sqrt(head_dim). Accumulation is float32; bf16
 *    results are rounded to nearest even.
 *  - workspace: DEVICE scratch owned by the caller, at least the size the
 *    matching *_workspace_size query returns, 256-byte aligned. Its contents
 *    need not be initialised. One workspace must not be used by two calls
 *    that may run at the same time.
 *  - stream: every launch is asynchronous on this stream; no call
 *    synchronises the device or allocates memory (ba_device_status is the
 *    one call that waits, and only on `stream`).
 *  - Errors: argument checks run on the host before anything is launched and
 *    return BA_ERR_INVALID_ARG (bad pointer, size or alignment) or
 *    BA_ERR_UNSUPPORTED (a valid combination this build has no kernel for).
 *    A launch failure returns BA_ERR_CUDA. Kernel-side waits are bounded;
 *    one that runs out records BA_ERR_TIMEOUT in the workspace, readable with
 *    ba_device_status. The library never traps.
 *  - Thread safety: no global mutable state besides a per-device cache of
 *    the SM count and the thread-local profiling hook below; calls on
 *    different streams with different workspaces are independent.
 */
#ifndef BA_H
#define BA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *ba_stream_t; /* same as cudaStream_t; NULL = legacy default stream */

typedef enum {
    BA_OK = 0,
    BA_ERR_INVALID_ARG = 1,
    BA_ERR_UNSUPPORTED = 2,
    BA_ERR_CUDA = 3,
    BA_ERR_TIMEOUT = 4
} ba_status;

typedef enum {
    BA_F32 = 0,  /* float32 tensors; SIMT kernels, no TF32 */
    BA_BF16 = 1  /* bfloat16 tensors; tcgen05 tensor-core kernels */
} ba_dtype;

/* Host-side description of one jagged batch. */
typedef struct {
    int32_t batch;        /* number of examples, >= 0 */
    int32_t total_tokens; /* seq_offsets[batch], >= 0 */
    int32_t heads;        /* >= 1; q, k, v share heads */
    int32_t head_dim;     /* BA_BF16: 64 or 128; BA_F32: 32 or 64 */
    ba_dtype dtype;
} ba_problem;

/*
 * Bytes of workspace ba_fwd / ba_bwd need for this problem (0 on an invalid
 * problem): a status word and a work table of about 16 bytes per 128-row
 * tile, plus, for the backward, two float32 per-row buffers [heads,
 * total_tokens]: the row dot product Delta = dO . out and (bf16) the
 * forward's lse in the form the dK/dV pass reads, and (bf16) 128 rows of q
 * and 128 of dout per example, 2 * batch * 128 * heads * head_dim bf16
 * values in all: each example's last query tile, when partial, staged with
 * zeros past the example's end for the key-side gradient pass. With window 1
 * and a block that divides 128 (every 128-row query tile then sees only its
 * own key tile) the bf16 backward runs as one fused pass for dq, dk and dv,
 * and the workspace also holds 128 staged rows of k per example (batch * 128
 * * heads * head_dim more bf16 values), since that pass's dq sums over the
 * partial key tile's rows. A batch of more than 2^31 / 128 examples is
 * BA_ERR_UNSUPPORTED.
 */
size_t ba_fwd_workspace_size(const ba_problem *p, int32_t block, int32_t window);
size_t ba_bwd_workspace_size(const ba_problem *p, int32_t block, int32_t window);

/*
 * Forward pass: out[i] = sum_j softmax_j(q_i . k_j / sqrt(head_dim)) v_j over
 * the keys visible to query i under the rule above, and lse as defined above.
 * block >= 1, window >= 1.
 */
ba_status ba_fwd(const ba_problem *p, const void *q, const void *k, const void *v,
                 const int32_t *seq_offsets, int32_t block, int32_t window,
                 const uint8_t *skip, void *out, float *lse,
                 void *workspace, size_t workspace_bytes, ba_stream_t stream);

/*
 * Backward pass: given the forward's out and lse and the upstream gradient
 * dout, writes the exact gradients dq, dk, dv of sum(out * dout) with respect
 * to q, k, v. Probabilities are recomputed from lse (nothing else is saved
 * by the forward). Same shapes and conventions as ba_fwd.
 */
ba_status ba_bwd(const ba_problem *p, const void *q, const void *k, const void *v,
                 const void *out, const float *lse, const void *dout,
                 const int32_t *seq_offsets, int32_t block, int32_t window,
                 const uint8_t *skip, void *dq, void *dk, void *dv,
                 void *workspace, size_t workspace_bytes, ba_stream_t stream);

/*
 * Generalized dot-product attention (GDPA): "GEM (Meta)", section "Custom
 * kernels", describes GEM's self-, cross- and pooled attention with the
 * softmax replaced by an activation such as GELU or SiLU; "Scaling Meta's
 * Generative Ads Model (GEM) for Ads Recommendations", section "Kunlun
 * Architecture Details", adds that per-example feed-forward networks were
 * recast as it. The pages give no formula; the reading implemented here is
 * that the activation takes the softmax's place and nothing else changes:
 *     out_i = sum over visible j of act(q_i . k_j / sqrt(head_dim)) v_j
 * with the block rule above for visibility, no normalisation (hence no lse),
 * act = GELU (x Phi(x), exact erf form) or SiLU (x sigma(x)). The backward
 * writes the exact gradients dq, dk, dv of sum(out * dout).
 *  - BF16 only (BA_ERR_UNSUPPORTED for BA_F32); head_dim 64 or 128; no skip
 *    flags. Same tensor layouts, ownership and errors as ba_fwd / ba_bwd.
 *  - Workspace: ba_gdpa_workspace_size bytes, for either direction: the
 *    staged query tiles described at ba_bwd_workspace_size, never its
 *    staged k rows (the generalized attention has no fused backward).
 *  - act outside the enumeration: BA_ERR_INVALID_ARG.
 */
typedef enum { BA_ACT_GELU = 1, BA_ACT_SILU = 2 } ba_activation;

size_t ba_gdpa_workspace_size(const ba_problem *p, int32_t block, int32_t window);
ba_status ba_gdpa_fwd(const ba_problem *p, ba_activation act, const void *q, const void *k, const void *v,
                      const int32_t *seq_offsets, int32_t block, int32_t window, void *out, void *workspace,
                      size_t workspace_bytes, ba_stream_t stream);
ba_status ba_gdpa_bwd(const ba_problem *p, ba_activation act, const void *q, const void *k, const void *v,
                      const void *dout, const int32_t *seq_offsets, int32_t block, int32_t window, void *dq,
                      void *dk, void *dv, void *workspace, size_t workspace_bytes, ba_stream_t stream);

/*
 * GDPA cross-attention, GEM's cross- and pooled attention ("GEM (Meta)",
 * section "Custom kernels": the generalized attention serves them too and is
 * fastest with short keys/values). Example b's queries, rows
 * q_offsets[b] .. q_offsets[b+1]-1 of q (and of out, dout, dq), see every key
 * of example b's own key/value set, rows kv_offsets[b] .. kv_offsets[b+1]-1
 * of k and v (and of dk, dv); there is no mask:
 *     out_i = sum over the example's keys j of act(q_i . k_j / sqrt(head_dim)) v_j.
 * An example with no keys gets out = 0 (the empty sum) and dq = 0; one with no
 * queries gets dk = dv = 0. Pooled attention is this with a set of seed
 * queries repeated for every example (the caller sums the seeds' dq over
 * examples).
 *  - p describes the queries: batch, total_tokens = q_offsets[batch], heads,
 *    head_dim, dtype (BF16 only); kv_total_tokens = kv_offsets[batch]. Both
 *    offset arrays are DEVICE int32 [batch + 1], non-decreasing from 0.
 *  - q, out, dout, dq: DEVICE [total_tokens, heads, head_dim]; k, v, dk, dv:
 *    DEVICE [kv_total_tokens, heads, head_dim]; 16-byte aligned.
 *  - Workspace: ba_gdpa_cross_workspace_size bytes, for either direction
 *    (it includes 128 staged rows of q and of dout per example).
 *  - Errors as for ba_gdpa_fwd / ba_gdpa_bwd.
 */
size_t ba_gdpa_cross_workspace_size(const ba_problem *p, int32_t kv_total_tokens);
ba_status ba_gdpa_cross_fwd(const ba_problem *p, int32_t kv_total_tokens, ba_activation act, const void *q,
                            const void *k, const void *v, const int32_t *q_offsets, const int32_t *kv_offsets,
                            void *out, void *workspace, size_t workspace_bytes, ba_stream_t stream);
ba_status ba_gdpa_cross_bwd(const ba_problem *p, int32_t kv_total_tokens, ba_activation act, const void *q,
                            const void *k, const void *v, const void *dout, const int32_t *q_offsets,
                            const int32_t *kv_offsets, void *dq, void *dk, void *dv, void *workspace,
                            size_t workspace_bytes, ba_stream_t stream);

/*
 * MXFP8 operands for the score product ("Meta Scales GEM Ads Model Across
 * Platforms and Thousands of GPUs", opening section: GEM trains attention in
 * MXFP8; the pages define neither the format nor the operands). The format is
 * the public OCP Microscaling one: 32 consecutive elements along head_dim
 * share a power-of-two scale 2^e stored as an E8M0 byte (e + 127), with
 * e = floor(log2 max|v|) - 8 clamped to [-127, 127] (e = -8 for an all-zero
 * block); each element is v / 2^e rounded to the nearest E4M3 value, ties to
 * even, magnitudes above 448 clamped to 448.
 *
 * ba_mx_quantize: x DEVICE bf16 [rows, heads, head_dim] (head_dim a multiple
 * of 32) -> elements DEVICE E4M3 bytes [rows, heads, head_dim] and scales
 * DEVICE E8M0 bytes [rows, heads_pad, head_dim / 32], heads_pad = heads
 * rounded up to a multiple of 4 (padding entries are not written).
 *
 * ba_mx_fwd: block attention (same rule, arguments, outputs and errors as
 * ba_fwd) whose score product Q K^T takes MXFP8 Q and K: it quantises q and k
 * into its workspace and runs the block-scaled tensor-core product (E4M3
 * operands, E8M0 scale factors); softmax and P V are unchanged (bf16 P and
 * V). The result is block attention of the dequantised Q and K. BF16 with
 * head_dim 128 only (BA_ERR_UNSUPPORTED otherwise). Workspace:
 * ba_mx_fwd_workspace_size bytes.
 */
ba_status ba_mx_quantize(const void *x, int64_t rows, int32_t heads, int32_t head_dim, void *elements,
                         void *scales, ba_stream_t stream);
size_t ba_mx_fwd_workspace_size(const ba_problem *p, int32_t block, int32_t window);
ba_status ba_mx_fwd(const ba_problem *p, const void *q, const void *k, const void *v, const int32_t *seq_offsets,
                    int32_t block, int32_t window, const uint8_t *skip, void *out, float *lse, void *workspace,
                    size_t workspace_bytes, ba_stream_t stream);

/*
 * ba_mx_bwd: the backward of ba_mx_fwd (the pages say GEM's training uses
 * MXFP8 in forward and backward). Reading: the score product is recomputed
 * from the same MXFP8 Q and K as the forward, and the gradient passes
 * through the quantisation unchanged (its derivative taken as the identity),
 * so dq and dk are the gradients with respect to the dequantised q and k and
 * dv is the usual P^T dout. It writes the MX round trips of q and k (quantise,
 * then dequantise; exact in bf16 unless a block's largest magnitude is below
 * 2^-118) into its workspace and runs ba_bwd's kernels on them, so the
 * backward's products are bf16 MMAs of the dequantised values: the same
 * products, summed in another order, as the forward's block-scaled MMA.
 * Arguments, layouts, outputs and errors as ba_bwd; out and lse come from
 * ba_mx_fwd. BF16 with head_dim 128 only (BA_ERR_UNSUPPORTED otherwise).
 * Workspace: ba_mx_bwd_workspace_size bytes (ba_bwd_workspace_size plus two
 * bf16 [total_tokens, heads, head_dim] copies); ba_device_status reads it.
 */
size_t ba_mx_bwd_workspace_size(const ba_problem *p, int32_t block, int32_t window);
ba_status ba_mx_bwd(const ba_problem *p, const void *q, const void *k, const void *v, const void *out,
                    const float *lse, const void *dout, const int32_t *seq_offsets, int32_t block, int32_t window,
                    const uint8_t *skip, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                    ba_stream_t stream);

/*
 * Token-granular sliding-window attention, the predecessor that block
 * attention replaced ("GEM (Meta)", section "Custom kernels": long
 * user-history self-attention first moved to a sliding window, then to
 * independent blocks; the pages compare the two by self-attention layer
 * MFU). Query i of an example sees key j <=> i - window_tokens < j <= i
 * (local indices, causal, window_tokens >= 1). This is the block rule above
 * with block = 1 and window = window_tokens, and these entry points run
 * exactly that: same kernels, arguments, layouts, workspace, ownership and
 * errors as ba_fwd / ba_bwd / ba_*_workspace_size.
 */
size_t ba_swa_fwd_workspace_size(const ba_problem *p, int32_t window_tokens);
size_t ba_swa_bwd_workspace_size(const ba_problem *p, int32_t window_tokens);
ba_status ba_swa_fwd(const ba_problem *p, const void *q, const void *k, const void *v,
                     const int32_t *seq_offsets, int32_t window_tokens, const uint8_t *skip,
                     void *out, float *lse, void *workspace, size_t workspace_bytes,
                     ba_stream_t stream);
ba_status ba_swa_bwd(const ba_problem *p, const void *q, const void *k, const void *v,
                     const void *out, const float *lse, const void *dout,
                     const int32_t *seq_offsets, int32_t window_tokens, const uint8_t *skip,
                     void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                     ba_stream_t stream);

/*
 * Rotary position embedding fused with block attention ("GEM (Meta)",
 * section "Custom kernels": the production block-attention kernel carries a
 * fused rotary position embedding backward pass; the pages say nothing more
 * about it). The reading this library implements is RoFormer's rotation
 * applied to q and k (not v) before the scores. The adjacent pair
 * (x[2m], x[2m+1]) of a row at position pos, its 0-based index within its
 * own example (the origin the blocks use), becomes
 *     (x[2m] c - x[2m+1] s,  x[2m] s + x[2m+1] c),
 *     c = cos[pos * head_dim/2 + m],  s = sin[pos * head_dim/2 + m].
 * The caller owns the tables and so picks the frequencies (RoFormer's are
 * angle = pos * 10000^(-2m / head_dim)).
 *
 *  - ba_rope_fwd: block attention of the rotated q and k. A rotation pass
 *    writes rotated copies of q and k, in the problem's dtype, into the
 *    workspace; the attention kernels read those. q and k are not modified.
 *    Every row is rotated, skipped examples' too.
 *  - ba_rope_bwd: the gradients with respect to the UNROTATED q and k, which
 *    are the transposed rotations of the gradients of the rotated ones
 *    (g0 c + g1 s, -g0 s + g1 c). dv is as for ba_bwd. It recomputes the
 *    rotated copies, then runs the bf16 dQ and dK/dV kernels, which turn dq
 *    and dk back in their epilogues before the single store. The fp32 path
 *    does that in a pass after its kernels. out and lse are ba_rope_fwd's.
 *  - Rotated copies: by default ba_rope_fwd writes them into its workspace,
 *    and ba_rope_bwd recomputes them. A caller that keeps activations from
 *    the forward for the backward (as training does) can set q_rot and k_rot
 *    in the struct. ba_rope_fwd then writes R q and R k there, and
 *    ba_rope_bwd given the same buffers (holding those values, for the same
 *    q, k and tables) reads them and runs no rotation pass. Either both are
 *    NULL or both are set: DEVICE [total_tokens, heads, head_dim] tensors of
 *    the problem's dtype, 16-byte aligned, not aliasing any other argument.
 *  - Workspace: without q_rot / k_rot, the *_workspace_size of the plain
 *    entry point plus two 256-byte-aligned copies of a [total_tokens, heads,
 *    head_dim] tensor (ba_rope_*_workspace_size); with them, the plain entry
 *    point's size suffices.
 *  - Errors: as for ba_fwd / ba_bwd. In addition, BA_ERR_INVALID_ARG when
 *    rope is NULL, or, with total_tokens > 0, when cos or sin is NULL or not
 *    16-byte aligned, when rows < 1, or when exactly one of q_rot, k_rot is
 *    set or either is not 16-byte aligned. Nothing is launched in those
 *    cases.
 *    An example longer than the tables cannot be seen on the host. Its rows
 *    at positions >= rows are left unrotated (their results are wrong, but
 *    no memory outside the tables is read), and the workspace status word
 *    records it: ba_device_status then returns BA_ERR_INVALID_ARG.
 */
typedef struct {
    const float *cos; /* DEVICE, float32 [rows, head_dim / 2], row-major, 16-byte aligned */
    const float *sin; /* DEVICE, same layout */
    int32_t rows;     /* table rows; must cover the longest example, skipped ones included */
    void *q_rot;      /* optional DEVICE [total_tokens, heads, head_dim]: R q (see above) */
    void *k_rot;      /* optional, likewise R k; both NULL or both set */
} ba_rope;

size_t ba_rope_fwd_workspace_size(const ba_problem *p, int32_t block, int32_t window);
size_t ba_rope_bwd_workspace_size(const ba_problem *p, int32_t block, int32_t window);
ba_status ba_rope_fwd(const ba_problem *p, const ba_rope *rope, const void *q, const void *k,
                      const void *v, const int32_t *seq_offsets, int32_t block, int32_t window,
                      const uint8_t *skip, void *out, float *lse, void *workspace,
                      size_t workspace_bytes, ba_stream_t stream);
ba_status ba_rope_bwd(const ba_problem *p, const ba_rope *rope, const void *q, const void *k,
                      const void *v, const void *out, const float *lse, const void *dout,
                      const int32_t *seq_offsets, int32_t block, int32_t window,
                      const uint8_t *skip, void *dq, void *dk, void *dv, void *workspace,
                      size_t workspace_bytes, ba_stream_t stream);

/*
 * Forward pass that allocates nothing and takes no workspace (the pages have
 * no counterpart; this is a convenience of this library). For callers that
 * cannot call cudaMalloc: a host framework that owns every byte of device
 * memory through its own pool and hands kernels only their inputs and
 * outputs, or a plugin running inside such a framework with no handle on its
 * allocator. Same arguments and results as ba_fwd minus the workspace.
 *  - Scratch: a fixed 1 MiB array inside the library, held by every GPU that
 *    loads it until the process exits. A problem whose ba_fwd_workspace_size
 *    exceeds 1 MiB is rejected with BA_ERR_INVALID_ARG before anything runs.
 *    The size is about 16 bytes per 128-row tile plus 16 per pair of tiles
 *    plus 8 per example (and 1 KiB of fixed overhead), so one example of up
 *    to about 5.5 million tokens fits; compare ba_fwd_workspace_size with
 *    1 MiB to know for sure.
 *  - The first call on each device, with that device current, looks up the
 *    array's device address and caches it for the process. A context that is
 *    destroyed and created again (cudaDeviceReset) may load the library's
 *    device code elsewhere; do not use this entry point across such a reset.
 *  - All calls share the array: calls that may overlap on the GPU race and
 *    must be ordered by the caller (one stream, or events). Nothing a call
 *    reads from the array is left over from an earlier call.
 *  - ba_device_status cannot be used with this entry point (no workspace), so
 *    a kernel wait that timed out here is not reported; use ba_fwd where that
 *    matters.
 */
ba_status ba_fwd_noalloc(const ba_problem *p, const void *q, const void *k, const void *v,
                         const int32_t *seq_offsets, int32_t block, int32_t window,
                         const uint8_t *skip, void *out, float *lse, ba_stream_t stream);

/*
 * Waits for `stream`, then reads the status word that previous calls (ba_fwd,
 * ba_bwd and the other entry points) left in `workspace`. Returns:
 *  - BA_OK;
 *  - BA_ERR_TIMEOUT if a kernel gave up waiting (its outputs are then
 *    undefined);
 *  - BA_ERR_INVALID_ARG if a rotary call met an example longer than its
 *    tables;
 *  - BA_ERR_CUDA if the read itself failed.
 */
ba_status ba_device_status(const void *workspace, ba_stream_t stream);

/*
 * Self-test of the bounded waits (the pages have no counterpart; this checks
 * the library's own failure detection without faulting anything). Every
 * wait in the attention kernels gives up after 2 s, makes the kernel return,
 * and sets the workspace status word that ba_device_status reports as
 * BA_ERR_TIMEOUT. This launches one warp that waits, through that same code,
 * on a barrier nothing ever completes, with a limit of limit_us microseconds
 * (1 .. 1,000,000). Afterwards ba_device_status(workspace) returns
 * BA_ERR_TIMEOUT and the device stays usable. workspace: at least 256 bytes,
 * 256-byte aligned; its status word is overwritten. Returns
 * BA_ERR_INVALID_ARG for bad arguments (nothing launched).
 */
ba_status ba_selftest_wait_timeout(void *workspace, size_t workspace_bytes, int32_t limit_us,
                                   ba_stream_t stream);

/*
 * Self-test of the attention kernels' FMA-pipe 2^x (the pages have no
 * counterpart). To take load off the special-function unit, the softmax in
 * the bf16 forward evaluates one exponential pair in eight on the fused
 * multiply-add pipe: x is split into the nearest integer n and f = x - n in
 * [-1/2, 1/2], 2^f comes from a cubic fitted to it (relative error below
 * 1e-4), and n is added to the exponent field; x below -125 is first raised
 * to -125 (such values are far below anything a bf16 probability can hold
 * next to the row maximum). This writes y[i] = that 2^x(i) for the n DEVICE
 * floats x (y: DEVICE, n floats, not aliasing x), asynchronously on stream.
 * Returns BA_ERR_INVALID_ARG for n < 0 or null/misaligned pointers.
 */
ba_status ba_selftest_exp2(const float *x, float *y, int64_t n, ba_stream_t stream);

/*
 * Self-test of the generalized attention's activations (ba_gdpa_*): writes
 * y[i] = act(x[i]) and dy[i] = act'(x[i]) for the n DEVICE floats x (y, dy:
 * DEVICE, n floats each, aliasing nothing), asynchronously on stream, through
 * the device functions the kernels use. GELU's Phi comes from erf by
 * Abramowitz & Stegun's formula 7.1.26 (absolute error at most 1.5e-7);
 * e^(-x^2/2), 2^x and reciprocals come from the special-function unit.
 * SiLU's sigma(x) = 1 / (1 + 2^(-x log2 e)) likewise. dy[i] is NaN if the
 * kernels' three forms of the activation (value, derivative, both at once)
 * disagree for x[i]. BA_ERR_INVALID_ARG for an unknown act, n < 0 or
 * null/misaligned pointers.
 */
ba_status ba_selftest_activation(ba_activation act, const float *x, float *y, float *dy, int64_t n,
                                 ba_stream_t stream);

/*
 * Profiling hook. Until changed, calls made from THIS host thread record
 * `start` on their stream right before one kernel and `stop` right after it,
 * so that cudaEventElapsedTime(start, stop) is that kernel's own duration:
 * which = 0 the forward attention kernel of ba_fwd (or ba_gdpa_fwd), 1 the
 * dQ kernel of ba_bwd (ba_gdpa_bwd), 2 its dK/dV kernel. The events are cudaEvent_t handles owned by
 * the caller; pass NULL, NULL to stop recording. Returns BA_ERR_INVALID_ARG
 * for another `which`. Only the hook pointers are stored (thread-local);
 * nothing is synchronised.
 */
ba_status ba_set_profile_events(int32_t which, void *start, void *stop);

/* Static, human-readable name of a status code. */
const char *ba_status_string(ba_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t ba_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BA_H */
