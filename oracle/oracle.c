/*
 * Block attention — CPU oracle (TEST INFRASTRUCTURE ONLY).
 *
 * This file is the reference that the CUDA path is checked against. Only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg load it;
 * the library itself never calls it, links it or falls back to it.
 *
 * What it computes. "Meta Scales GEM Ads Model Across Platforms and Thousands
 * of GPUs" (section "Kunlun changes how GEM scales") describes block attention
 * as self-attention made sparse by arranging it in blocks, so that cost grows
 * linearly in sequence length for a fixed window; "GEM (Meta)" (section
 * "Custom kernels", BlockAttention) describes the long user-history
 * self-attention split into independent 64-token blocks; "Scaling Meta's
 * Generative Ads Model (GEM) for Ads Recommendations" (section "Kunlun
 * Architecture Details") repeats the quadratic-to-linear claim. The pages
 * give no formula. The rule used everywhere in this project:
 *
 *   local query index i, local key index j (0-based within one example),
 *   blk(x) = floor(x / block),
 *   Allowed(i, j)  <=>  j <= i  and  blk(j) >= blk(i) - (window - 1).
 *
 * window = 1 gives the pages' "independent blocks" literally (causal inside
 * each block). Blocks start at each example's first token ("GEM (Meta)",
 * section "Training infrastructure": histories are jagged and are not padded).
 *
 * For each example e and head h, in fp64, with the L x L mask evaluated
 * explicitly for every (i, j) pair:
 *   s_ij  = (q_i . k_j) / sqrt(D)            if Allowed(i, j), else -inf
 *   m_i   = max_j s_ij
 *   l_i   = sum_j exp(s_ij - m_i)
 *   p_ij  = exp(s_ij - m_i) / l_i
 *   o_i   = sum_j p_ij v_j
 *   lse_i = m_i + ln(l_i)                    (natural log, scaled scores)
 * Backward (exact gradient of o with respect to q, k, v for upstream dO):
 *   Delta_i = dO_i . o_i
 *   dp_ij   = dO_i . v_j
 *   ds_ij   = p_ij (dp_ij - Delta_i)
 *   dq_i    = (1/sqrt(D)) sum_j ds_ij k_j
 *   dk_j    = (1/sqrt(D)) sum_i ds_ij q_i
 *   dv_j    = sum_i p_ij dO_i
 * Component skip ("Meta Scales GEM Ads Model ...", section "Kunlun changes
 * how GEM scales": sequence modules are selectively bypassed): a flagged
 * example passes its values through, o = v, so dq = dk = 0 and dv = dO; its
 * lse is written as 0 by convention.
 *
 * Layouts: q, k, v, dout, out, dq, dk, dv are [total_tokens, heads, head_dim]
 * row-major fp64; lse is [heads, total_tokens]; seq_offsets has batch + 1
 * entries, seq_offsets[0] = 0, non-decreasing. Work is split over
 * (example, head) pairs only; each pair is computed serially, so the results
 * do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static int allowed(int64_t i, int64_t j, int64_t block, int64_t window)
{
    if (j > i) return 0;
    return (j / block) >= (i / block) - (window - 1);
}

/* Scores of one query row against every key of the example; masked pairs get
 * -inf without evaluating the dot product (exp(-inf) is exactly 0, so this is
 * the same arithmetic as evaluating and then masking). Returns the row max. */
static double score_row(int64_t i, int64_t L, int64_t H, int64_t D, int64_t h,
                        int64_t block, int64_t window, const double *q,
                        const double *k, double *s)
{
    const double scale = 1.0 / sqrt((double)D);
    const double *qi = q + (i * H + h) * D;
    double m = -INFINITY;
    for (int64_t j = 0; j < L; ++j) {
        if (!allowed(i, j, block, window)) {
            s[j] = -INFINITY;
            continue;
        }
        const double *kj = k + (j * H + h) * D;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qi[d] * kj[d];
        s[j] = dot * scale;
        if (s[j] > m) m = s[j];
    }
    return m;
}

/* Turns the score row into probabilities in place; returns l_i. */
static double softmax_row(int64_t L, double m, double *s)
{
    double l = 0.0;
    for (int64_t j = 0; j < L; ++j) l += exp(s[j] - m);
    for (int64_t j = 0; j < L; ++j) s[j] = exp(s[j] - m) / l;
    return l;
}

static void fwd_pair(int64_t L, int64_t H, int64_t D, int64_t h, int64_t block,
                     int64_t window, const double *q, const double *k,
                     const double *v, double *out, double *lse_h, double *s)
{
    for (int64_t i = 0; i < L; ++i) {
        double m = score_row(i, L, H, D, h, block, window, q, k, s);
        double l = softmax_row(L, m, s);
        double *oi = out + (i * H + h) * D;
        for (int64_t d = 0; d < D; ++d) oi[d] = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            if (s[j] == 0.0) continue;
            const double *vj = v + (j * H + h) * D;
            for (int64_t d = 0; d < D; ++d) oi[d] += s[j] * vj[d];
        }
        lse_h[i] = m + log(l);
    }
}

static void bwd_pair(int64_t L, int64_t H, int64_t D, int64_t h, int64_t block,
                     int64_t window, const double *q, const double *k,
                     const double *v, const double *dout, double *dq,
                     double *dk, double *dv, double *s, double *o)
{
    const double scale = 1.0 / sqrt((double)D);
    for (int64_t j = 0; j < L; ++j) {
        for (int64_t d = 0; d < D; ++d) {
            dk[(j * H + h) * D + d] = 0.0;
            dv[(j * H + h) * D + d] = 0.0;
        }
    }
    for (int64_t i = 0; i < L; ++i) {
        double m = score_row(i, L, H, D, h, block, window, q, k, s);
        softmax_row(L, m, s);
        for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            if (s[j] == 0.0) continue;
            const double *vj = v + (j * H + h) * D;
            for (int64_t d = 0; d < D; ++d) o[d] += s[j] * vj[d];
        }
        const double *doi = dout + (i * H + h) * D;
        const double *qi = q + (i * H + h) * D;
        double delta = 0.0;
        for (int64_t d = 0; d < D; ++d) delta += doi[d] * o[d];
        double *dqi = dq + (i * H + h) * D;
        for (int64_t d = 0; d < D; ++d) dqi[d] = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            if (!allowed(i, j, block, window)) continue;
            const double *vj = v + (j * H + h) * D;
            const double *kj = k + (j * H + h) * D;
            double dp = 0.0;
            for (int64_t d = 0; d < D; ++d) dp += doi[d] * vj[d];
            const double p = s[j];
            const double ds = p * (dp - delta);
            double *dkj = dk + (j * H + h) * D;
            double *dvj = dv + (j * H + h) * D;
            for (int64_t d = 0; d < D; ++d) {
                dqi[d] += scale * ds * kj[d];
                dkj[d] += scale * ds * qi[d];
                dvj[d] += p * doi[d];
            }
        }
    }
}

static int64_t max_len(int32_t batch, const int32_t *offs)
{
    int64_t m = 0;
    for (int32_t e = 0; e < batch; ++e) {
        int64_t L = (int64_t)offs[e + 1] - offs[e];
        if (L > m) m = L;
    }
    return m;
}

int oracle_fwd(int32_t batch, const int32_t *seq_offsets, int32_t heads,
               int32_t head_dim, int32_t block, int32_t window,
               const uint8_t *skip, const double *q, const double *k,
               const double *v, double *out, double *lse, int32_t nthreads)
{
    if (batch < 0 || heads < 1 || head_dim < 1 || block < 1 || window < 1)
        return 1;
    const int64_t T = seq_offsets[batch];
    const int64_t H = heads, D = head_dim;
    const int64_t Lmax = max_len(batch, seq_offsets);
    const int64_t npairs = (int64_t)batch * H;
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
        if (!s) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t p = 0; p < npairs; ++p) {
            if (!s) continue;
            const int64_t e = p / H, h = p % H;
            const int64_t s0 = seq_offsets[e], L = seq_offsets[e + 1] - s0;
            const double *qe = q + s0 * H * D, *ke = k + s0 * H * D, *ve = v + s0 * H * D;
            double *oe = out + s0 * H * D;
            double *lse_h = lse + h * T + s0;
            if (skip && skip[e]) {
                for (int64_t i = 0; i < L; ++i) {
                    memcpy(oe + (i * H + h) * D, ve + (i * H + h) * D, sizeof(double) * D);
                    lse_h[i] = 0.0;
                }
                continue;
            }
            fwd_pair(L, H, D, h, block, window, qe, ke, ve, oe, lse_h, s);
        }
        free(s);
    }
    return err;
}

int oracle_bwd(int32_t batch, const int32_t *seq_offsets, int32_t heads,
               int32_t head_dim, int32_t block, int32_t window,
               const uint8_t *skip, const double *q, const double *k,
               const double *v, const double *dout, double *dq, double *dk,
               double *dv, int32_t nthreads)
{
    if (batch < 0 || heads < 1 || head_dim < 1 || block < 1 || window < 1)
        return 1;
    const int64_t H = heads, D = head_dim;
    const int64_t Lmax = max_len(batch, seq_offsets);
    const int64_t npairs = (int64_t)batch * H;
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)((Lmax > 0 ? Lmax : 1) + D));
        if (!s) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t p = 0; p < npairs; ++p) {
            if (!s) continue;
            const int64_t e = p / H, h = p % H;
            const int64_t s0 = seq_offsets[e], L = seq_offsets[e + 1] - s0;
            const int64_t base = s0 * H * D;
            if (skip && skip[e]) {
                for (int64_t i = 0; i < L; ++i) {
                    const int64_t r = base + (i * H + h) * D;
                    for (int64_t d = 0; d < D; ++d) {
                        dq[r + d] = 0.0;
                        dk[r + d] = 0.0;
                        dv[r + d] = dout[r + d];
                    }
                }
                continue;
            }
            bwd_pair(L, H, D, h, block, window, q + base, k + base, v + base,
                     dout + base, dq + base, dk + base, dv + base, s, s + Lmax);
        }
        free(s);
    }
    return err;
}

/*
 * Sampled rows of one (example, head), for problems too large to compute in
 * full on the host. q, k, v, dout point at the example's first row
 * ([L, heads, head_dim]). For each requested local row r the same definition
 * as above is evaluated: out[r], lse[r], dq[r] from query row r, and dk[r],
 * dv[r] from every query row i with Allowed(i, r) (each such row's softmax is
 * recomputed in full). Any of the output pointers may be NULL.
 */
int oracle_rows(int32_t L, int32_t heads, int32_t head_dim, int32_t block,
                int32_t window, int32_t h, const double *q, const double *k,
                const double *v, const double *dout, int32_t nrows,
                const int32_t *rows, double *out_rows, double *lse_rows,
                double *dq_rows, double *dk_rows, double *dv_rows,
                int32_t nthreads)
{
    if (L < 1 || heads < 1 || head_dim < 1 || block < 1 || window < 1 ||
        h < 0 || h >= heads)
        return 1;
    const int64_t H = heads, D = head_dim;
    const double scale = 1.0 / sqrt((double)D);
    const int need_bwd = dq_rows || dk_rows || dv_rows;
    if (need_bwd && !dout) return 1;
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(L + 2 * D));
        if (!s) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int32_t n = 0; n < nrows; ++n) {
            if (!s) continue;
            const int64_t r = rows[n];
            if (r < 0 || r >= L) {
#pragma omp atomic write
                err = 1;
                continue;
            }
            double *o = s + L, *acc = s + L + D;
            /* query side: out, lse, dq of row r */
            if (out_rows || lse_rows || dq_rows) {
                double m = score_row(r, L, H, D, h, block, window, q, k, s);
                double l = softmax_row(L, m, s);
                for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
                for (int64_t j = 0; j < L; ++j) {
                    if (s[j] == 0.0) continue;
                    for (int64_t d = 0; d < D; ++d) o[d] += s[j] * v[(j * H + h) * D + d];
                }
                if (out_rows) memcpy(out_rows + n * D, o, sizeof(double) * D);
                if (lse_rows) lse_rows[n] = m + log(l);
                if (dq_rows) {
                    const double *dor = dout + (r * H + h) * D;
                    double delta = 0.0;
                    for (int64_t d = 0; d < D; ++d) delta += dor[d] * o[d];
                    for (int64_t d = 0; d < D; ++d) acc[d] = 0.0;
                    for (int64_t j = 0; j < L; ++j) {
                        if (!allowed(r, j, block, window)) continue;
                        double dp = 0.0;
                        for (int64_t d = 0; d < D; ++d) dp += dor[d] * v[(j * H + h) * D + d];
                        const double ds = s[j] * (dp - delta);
                        for (int64_t d = 0; d < D; ++d) acc[d] += scale * ds * k[(j * H + h) * D + d];
                    }
                    memcpy(dq_rows + n * D, acc, sizeof(double) * D);
                }
            }
            /* key side: dk, dv of row r, summing over every query that sees it */
            if (dk_rows || dv_rows) {
                double *dkr = dk_rows ? dk_rows + n * D : NULL;
                double *dvr = dv_rows ? dv_rows + n * D : NULL;
                for (int64_t d = 0; d < D; ++d) {
                    if (dkr) dkr[d] = 0.0;
                    if (dvr) dvr[d] = 0.0;
                }
                for (int64_t i = 0; i < L; ++i) {
                    if (!allowed(i, r, block, window)) continue;
                    double m = score_row(i, L, H, D, h, block, window, q, k, s);
                    softmax_row(L, m, s);
                    const double *doi = dout + (i * H + h) * D;
                    const double p = s[r];
                    if (dvr)
                        for (int64_t d = 0; d < D; ++d) dvr[d] += p * doi[d];
                    if (dkr) {
                        for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
                        for (int64_t j = 0; j < L; ++j) {
                            if (s[j] == 0.0) continue;
                            for (int64_t d = 0; d < D; ++d) o[d] += s[j] * v[(j * H + h) * D + d];
                        }
                        double delta = 0.0, dp = 0.0;
                        for (int64_t d = 0; d < D; ++d) {
                            delta += doi[d] * o[d];
                            dp += doi[d] * v[(r * H + h) * D + d];
                        }
                        const double ds = p * (dp - delta);
                        const double *qi = q + (i * H + h) * D;
                        for (int64_t d = 0; d < D; ++d) dkr[d] += scale * ds * qi[d];
                    }
                }
            }
        }
        free(s);
    }
    return err;
}
