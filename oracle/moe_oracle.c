/*
 * CPU oracle for the local MoE expert forward on the non-expand routed layout.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; it is used by the tests, by the smoke check and by the
 * benchmark's CPU-baseline leg.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * Everything here is the plain definition of what the method computes,
 * written as loops over tokens and their valid slots:
 *
 *  - pair list, histogram, offsets and the stable sort by expert follow the
 *    metadata list of sonic-moe issue #68 ("End-to-end DeepEP v2 non-expand +
 *    SonicMoE integration": expert_frequency, expert_frequency_offset,
 *    x_gather_idx, s_scatter_idx, s_reverse_scatter_idx,
 *    num_activated_expert_per_token_offset, compact router_scores) and its
 *    question 3 (pairs are taken in ascending token order);
 *  - the expert MLP is the gated up projection, "silu times up", and the down
 *    projection (qwen3_5.py commit notes, the CCCL segmented-sort recipe,
 *    step 4; sonic-moe write-up, "The MoE class takes a routing count and a
 *    kernel backend": SWIGLU, optional biases);
 *  - the gate/up column pairing is interleaved (g0,u0,g1,u1,...) or
 *    concatenated (all gates, then all ups) (sonic-moe write-up, "Interleaved
 *    by default, concatenated if your model is HuggingFace");
 *  - the combine sums score x expert row over a token's pairs back to [N,H]
 *    (issue #68 dataflow, local_out [N_recv,H]; qwen3_5.py notes, step 5).
 *
 * Precision: inputs are bf16 (exactly representable in double); all
 * arithmetic is in double with no intermediate rounding.
 *
 * Parity pins: every function is pinned by the not-gpu tests (invariants,
 * brute force, closed forms, a torch-CPU cross-implementation of the recipe).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_value(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------
 * Routing metadata.
 *
 * Pair q counts the valid slots in row-major (token, slot) order.  A slot is
 * valid when its id lies in [0,E); -1 marks an invalid slot (issue #68,
 * non-expand receive layout).  Any other id is counted in *bad_ids and
 * skipped like -1.
 *
 * Outputs (all caller-allocated; pair arrays need room for N*K entries):
 *   freq[E]          number of pairs per expert
 *   off[E+1]         exclusive prefix sum of freq, off[E] = P
 *   x_gather_idx[p]  token of the pair at expert-sorted position p
 *   s_scatter_idx[p] pair index q at sorted position p
 *   s_rev[q]         sorted position p of pair q
 *   token_offset[N+1] pairs of token t are q in [token_offset[t], token_offset[t+1])
 *   scores[q]        topk_w of pair q
 * Returns P.
 * ---------------------------------------------------------------------- */
int64_t oracle_metadata(int64_t N, int32_t K, int32_t E,
                        const int32_t *topk_idx, const float *topk_w,
                        int32_t *freq, int32_t *off,
                        int32_t *x_gather_idx, int32_t *s_scatter_idx,
                        int32_t *s_rev, int32_t *token_offset, float *scores,
                        int64_t *bad_ids)
{
    int64_t nbad = 0;
    int64_t q = 0;
    int32_t *pair_token = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N * K + 1));
    int32_t *pair_expert = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N * K + 1));
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));

    /* 1. pair list in ascending token order, slot order within a token */
    for (int64_t t = 0; t < N; ++t) {
        token_offset[t] = (int32_t)q;
        for (int32_t k = 0; k < K; ++k) {
            int32_t e = topk_idx[t * K + k];
            if (e >= 0 && e < E) {
                pair_token[q] = (int32_t)t;
                pair_expert[q] = e;
                scores[q] = topk_w[t * K + k];
                ++q;
            } else if (e != -1) {
                ++nbad;
            }
        }
    }
    token_offset[N] = (int32_t)q;

    /* 2. histogram and its exclusive prefix sum */
    for (int32_t e = 0; e < E; ++e) freq[e] = 0;
    for (int64_t i = 0; i < q; ++i) freq[pair_expert[i]] += 1;
    off[0] = 0;
    for (int32_t e = 0; e < E; ++e) off[e + 1] = off[e] + freq[e];

    /* 3. stable counting sort of the pairs by expert */
    for (int32_t e = 0; e < E; ++e) cursor[e] = off[e];
    for (int64_t i = 0; i < q; ++i) {
        int32_t p = cursor[pair_expert[i]]++;
        x_gather_idx[p] = pair_token[i];
        s_scatter_idx[p] = (int32_t)i;
        s_rev[i] = p;
    }

    free(pair_token);
    free(pair_expert);
    free(cursor);
    if (bad_ids) *bad_ids = nbad;
    return q;
}

/* ------------------------------------------------------------------------
 * Routing metadata of a compact pair list (sonic-moe issue #68, the general
 * routing API the non-expand path is proposed beside: token_indices,
 * expert_indices and router_scores, one entry per (token, expert) pair, in
 * ascending token order).
 *
 * Entry i of the list is kept when expert_idx[i] is in [0,E) and
 * token_idx[i] is in [0,N); pair q counts the kept entries in list order.
 * Expert id -1 drops an entry silently; any other out-of-range expert id is
 * counted in *bad_ids; a kept-looking entry (valid expert) whose token is out
 * of range is counted in *bad_tokens.  *unsorted is set when some entry's
 * token is smaller than the one before it (the metadata then assumes an
 * order it does not have and token_offset means nothing).
 *
 * Outputs are those of oracle_metadata, with
 *   token_offset[t] = number of kept entries whose token is below t
 * (t = 0..N), which for an ascending list makes pairs of token t the q in
 * [token_offset[t], token_offset[t+1]).  Pair arrays need room for P_list.
 * Returns P.
 * ---------------------------------------------------------------------- */
int64_t oracle_metadata_pairs(int64_t N, int64_t P_list, int32_t E,
                              const int64_t *token_idx, const int64_t *expert_idx,
                              const float *weights,
                              int32_t *freq, int32_t *off,
                              int32_t *x_gather_idx, int32_t *s_scatter_idx,
                              int32_t *s_rev, int32_t *token_offset, float *scores,
                              int64_t *bad_ids, int64_t *bad_tokens, int32_t *unsorted)
{
    int64_t nbad = 0, nbadtok = 0, q = 0;
    int32_t *pair_token = (int32_t *)malloc(sizeof(int32_t) * (size_t)(P_list + 1));
    int32_t *pair_expert = (int32_t *)malloc(sizeof(int32_t) * (size_t)(P_list + 1));
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));

    /* 1. kept entries in list order */
    *unsorted = 0;
    for (int64_t i = 0; i < P_list; ++i) {
        int64_t t = token_idx[i], e = expert_idx[i];
        if (i > 0 && token_idx[i - 1] > t) *unsorted = 1;
        if (e >= 0 && e < E) {
            if (t >= 0 && t < N) {
                pair_token[q] = (int32_t)t;
                pair_expert[q] = (int32_t)e;
                scores[q] = weights[i];
                ++q;
            } else {
                ++nbadtok;
            }
        } else if (e != -1) {
            ++nbad;
        }
    }

    /* 2. token offsets: kept pairs whose token is below t */
    for (int64_t t = 0; t <= N; ++t) {
        int64_t below = 0;
        for (int64_t j = 0; j < q; ++j)
            if (pair_token[j] < t) ++below;
        token_offset[t] = (int32_t)below;
    }

    /* 3. histogram, offsets and the stable counting sort by expert */
    for (int32_t e = 0; e < E; ++e) freq[e] = 0;
    for (int64_t j = 0; j < q; ++j) freq[pair_expert[j]] += 1;
    off[0] = 0;
    for (int32_t e = 0; e < E; ++e) off[e + 1] = off[e] + freq[e];
    for (int32_t e = 0; e < E; ++e) cursor[e] = off[e];
    for (int64_t j = 0; j < q; ++j) {
        int32_t p = cursor[pair_expert[j]]++;
        x_gather_idx[p] = pair_token[j];
        s_scatter_idx[p] = (int32_t)j;
        s_rev[j] = p;
    }

    free(pair_token);
    free(pair_expert);
    free(cursor);
    *bad_ids = nbad;
    *bad_tokens = nbadtok;
    return q;
}

/* ------------------------------------------------------------------------
 * Router top-k (sonic-moe write-up, "Three routing strategies, selected on
 * the command line").  Per token, from its E logits:
 *
 *   chosen experts  the K largest logits, largest first; equal logits are
 *                   taken in ascending expert id
 *   mode 0          TC top-K: softmax over the K chosen logits
 *   mode 1          Qwen3-style: softmax over all E logits, read at the chosen
 *   mode 2          mode 1 divided by its sum over the K chosen
 *
 * logits are doubles (the caller widens fp32 or bf16 exactly and reads NaN
 * as -inf); topk_w is double.
 * ---------------------------------------------------------------------- */
void oracle_router_topk(int64_t N, int32_t E, int32_t K, int32_t mode,
                        const double *logits, int32_t *topk_idx, double *topk_w)
{
    char *taken = (char *)malloc((size_t)E);
    for (int64_t t = 0; t < N; ++t) {
        const double *row = logits + t * E;
        int32_t *ix = topk_idx + t * K;
        double *w = topk_w + t * K;
        memset(taken, 0, (size_t)E);
        /* the K largest, one at a time */
        for (int32_t k = 0; k < K; ++k) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || row[e] > row[best])) best = e;
            taken[best] = 1;
            ix[k] = best;
        }
        const double top = row[ix[0]];
        if (mode == 0) {
            double s = 0.0;
            for (int32_t k = 0; k < K; ++k) s += exp(row[ix[k]] - top);
            for (int32_t k = 0; k < K; ++k) w[k] = exp(row[ix[k]] - top) / s;
        } else {
            double z = 0.0;
            for (int32_t e = 0; e < E; ++e) z += exp(row[e] - top);
            for (int32_t k = 0; k < K; ++k) w[k] = exp(row[ix[k]] - top) / z;
            if (mode == 2) {
                double s = 0.0;
                for (int32_t k = 0; k < K; ++k) s += w[k];
                for (int32_t k = 0; k < K; ++k) w[k] /= s;
            }
        }
    }
    free(taken);
}

/* ------------------------------------------------------------------------
 * One expert applied to one token row, in double.
 *   z   = x_t . W1[e] + b1[e]                       (2I values)
 *   h_j = silu(gate_j) * up_j,  silu(g) = g / (1 + exp(-g))
 *         interleaved:  gate_j = z[2j],  up_j = z[2j+1]
 *         concatenated: gate_j = z[j],   up_j = z[I+j]
 *   y   = h . W2[e] + b2[e]                         (H values)
 * w1e is [H][2I], w2e is [I][H], row-major.  b1e / b2e may be NULL.
 * z must hold 2I doubles.
 * ---------------------------------------------------------------------- */
void oracle_expert_row(int32_t H, int32_t I, int32_t layout,
                       const uint16_t *x_row, const uint16_t *w1e, const uint16_t *b1e,
                       const uint16_t *w2e, const uint16_t *b2e,
                       double *z, double *h, double *y)
{
    const int32_t two_i = 2 * I;
    for (int32_t j = 0; j < two_i; ++j) z[j] = b1e ? bf16_value(b1e[j]) : 0.0;
    for (int32_t k = 0; k < H; ++k) {
        const double xv = bf16_value(x_row[k]);
        const uint16_t *wr = w1e + (size_t)k * two_i;
        for (int32_t j = 0; j < two_i; ++j) z[j] += xv * bf16_value(wr[j]);
    }
    for (int32_t j = 0; j < I; ++j) {
        double g, u;
        if (layout == 0) { g = z[2 * j]; u = z[2 * j + 1]; }
        else             { g = z[j];     u = z[I + j]; }
        h[j] = g / (1.0 + exp(-g)) * u;
    }
    for (int32_t n = 0; n < H; ++n) y[n] = b2e ? bf16_value(b2e[n]) : 0.0;
    for (int32_t j = 0; j < I; ++j) {
        const double hv = h[j];
        const uint16_t *wr = w2e + (size_t)j * H;
        for (int32_t n = 0; n < H; ++n) y[n] += hv * bf16_value(wr[n]);
    }
}

/* ------------------------------------------------------------------------
 * Forward output rows for a chosen set of tokens:
 *   out[i,:] = sum over valid slots k of token tokens[i], in slot order,
 *              topk_w[t,k] * expert_row(x_t, expert topk_idx[t,k])
 * A token with no valid slot gets a zero row.  Invalid slots' weights are
 * never read.  out is [n_tokens][H] double.
 * ---------------------------------------------------------------------- */
void oracle_forward_rows(int64_t N, int32_t H, int32_t I, int32_t E, int32_t K,
                         int32_t layout,
                         const uint16_t *x, const int32_t *topk_idx, const float *topk_w,
                         const uint16_t *w1, const uint16_t *b1,
                         const uint16_t *w2, const uint16_t *b2,
                         int64_t n_tokens, const int64_t *tokens, double *out,
                         int32_t n_threads)
{
    (void)N;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
#endif
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)(2 * I));
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
        double *y = (double *)malloc(sizeof(double) * (size_t)H);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t i = 0; i < n_tokens; ++i) {
            const int64_t t = tokens[i];
            double *o = out + (size_t)i * H;
            for (int32_t n = 0; n < H; ++n) o[n] = 0.0;
            for (int32_t k = 0; k < K; ++k) {
                const int32_t e = topk_idx[t * K + k];
                if (e < 0 || e >= E) continue;
                const double w = (double)topk_w[t * K + k];
                oracle_expert_row(H, I, layout, x + (size_t)t * H,
                                  w1 + (size_t)e * H * 2 * I, b1 ? b1 + (size_t)e * 2 * I : NULL,
                                  w2 + (size_t)e * I * H, b2 ? b2 + (size_t)e * H : NULL,
                                  z, h, y);
                for (int32_t n = 0; n < H; ++n) o[n] += w * y[n];
            }
        }
        free(z);
        free(h);
        free(y);
    }
}

/* ------------------------------------------------------------------------
 * The combine alone, given expert rows in expert-sorted order ysorted[p][H]
 * (any values, in double) and the metadata:
 *   out[t,:] = sum over q in [token_offset[t], token_offset[t+1]), in q order,
 *              of scores[q] * ysorted[s_rev[q], :]
 * Used to check the combine kernel in isolation.
 * ---------------------------------------------------------------------- */
void oracle_combine(int64_t N, int32_t H, const int32_t *token_offset,
                    const int32_t *s_rev, const float *scores,
                    const double *ysorted, double *out)
{
    for (int64_t t = 0; t < N; ++t) {
        double *o = out + (size_t)t * H;
        for (int32_t n = 0; n < H; ++n) o[n] = 0.0;
        for (int32_t q = token_offset[t]; q < token_offset[t + 1]; ++q) {
            const double w = (double)scores[q];
            const double *yr = ysorted + (size_t)s_rev[q] * H;
            for (int32_t n = 0; n < H; ++n) o[n] += w * yr[n];
        }
    }
}

/* ------------------------------------------------------------------------
 * Per-pair intermediate rows for a list of (token, expert) pairs:
 *   h_out[i,:] = silu(gate) * up of expert experts[i] on token tokens[i]  [I]
 *   y_out[i,:] = h . W2[e] + b2[e]                                        [H]
 * Used to localise a disagreement to the up or the down projection.
 * ---------------------------------------------------------------------- */
void oracle_pair_rows(int32_t H, int32_t I, int32_t layout,
                      const uint16_t *x, const uint16_t *w1, const uint16_t *b1,
                      const uint16_t *w2, const uint16_t *b2,
                      int64_t n_pairs, const int64_t *tokens, const int32_t *experts,
                      double *h_out, double *y_out, int32_t n_threads)
{
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
#endif
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)(2 * I));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t i = 0; i < n_pairs; ++i) {
            const int32_t e = experts[i];
            oracle_expert_row(H, I, layout, x + (size_t)tokens[i] * H,
                              w1 + (size_t)e * H * 2 * I, b1 ? b1 + (size_t)e * 2 * I : NULL,
                              w2 + (size_t)e * I * H, b2 ? b2 + (size_t)e * H : NULL,
                              z, h_out + (size_t)i * I, y_out + (size_t)i * H);
        }
        free(z);
    }
}

/* ------------------------------------------------------------------------
 * Backward of the local expert compute, in double (the pages leave the
 * backward open; this is the chain rule applied to the forward above).
 *
 * For one pair (token row x, expert e, score s) and the output gradient dout
 * of its token:
 *   forward  z = x.W1[e] + b1[e];  h_j = silu(g_j) u_j;  y = h.W2[e] + b2[e]
 *   dy   = s dout                      (the pair's share of out = sum s y)
 *   ds   = <dout, y>                   (gradient of the score)
 *   dh   = dy . W2[e]^T                (I values)
 *   dg_j = dh_j u_j silu'(g_j),  silu'(g) = sig(g) (1 + g (1 - sig(g)))
 *   du_j = dh_j silu(g_j)
 *   dz   = (dg, du) at the gate/up columns of the layout
 * The caller sums dW2[e] += h^T dy, db2[e] += dy, dW1[e] += x^T dz,
 * db1[e] += dz and dx[t] += dz . W1[e]^T over the pairs.
 *
 * w1e [H][2I], w2e [I][H] row-major doubles; b1e / b2e may be NULL.
 * ---------------------------------------------------------------------- */
void oracle_pair_backward(int32_t H, int32_t I, int32_t layout,
                          const double *x, const double *w1e, const double *b1e,
                          const double *w2e, const double *b2e,
                          const double *dout, double s,
                          double *z, double *h, double *y, double *dy, double *dz, double *ds)
{
    for (int32_t j = 0; j < 2 * I; ++j) z[j] = b1e ? b1e[j] : 0.0;
    for (int32_t k = 0; k < H; ++k) {
        const double xv = x[k];
        const double *wr = w1e + (size_t)k * 2 * I;
        for (int32_t j = 0; j < 2 * I; ++j) z[j] += xv * wr[j];
    }
    for (int32_t j = 0; j < I; ++j) {
        const int32_t gi = layout == 0 ? 2 * j : j, ui = layout == 0 ? 2 * j + 1 : I + j;
        const double g = z[gi], u = z[ui];
        h[j] = g / (1.0 + exp(-g)) * u;
    }
    for (int32_t n = 0; n < H; ++n) y[n] = b2e ? b2e[n] : 0.0;
    for (int32_t j = 0; j < I; ++j) {
        const double *wr = w2e + (size_t)j * H;
        for (int32_t n = 0; n < H; ++n) y[n] += h[j] * wr[n];
    }
    double acc = 0.0;
    for (int32_t n = 0; n < H; ++n) {
        dy[n] = s * dout[n];
        acc += dout[n] * y[n];
    }
    *ds = acc;
    for (int32_t j = 0; j < I; ++j) {
        const double *wr = w2e + (size_t)j * H;
        double dh = 0.0;
        for (int32_t n = 0; n < H; ++n) dh += dy[n] * wr[n];
        const int32_t gi = layout == 0 ? 2 * j : j, ui = layout == 0 ? 2 * j + 1 : I + j;
        const double g = z[gi], u = z[ui];
        const double sig = 1.0 / (1.0 + exp(-g));
        dz[gi] = dh * u * sig * (1.0 + g * (1.0 - sig));
        dz[ui] = dh * g * sig;
    }
}

/* oracle_pair_backward over n pairs (OpenMP).  x [N][H], w1 [E][H][2I],
 * w2 [E][I][H], b1 [E][2I] / b2 [E][H] or NULL, dout [N][H]; pair i is
 * (tokens[i], experts[i], scores[i]).  Outputs per pair: h [n][I], y [n][H],
 * dy [n][H], dz [n][2I], ds [n]. */
void oracle_pairs_backward(int32_t H, int32_t I, int32_t layout,
                           const double *x, const double *w1, const double *b1,
                           const double *w2, const double *b2, const double *dout,
                           int64_t n, const int64_t *tokens, const int32_t *experts,
                           const double *scores, double *h, double *y, double *dy,
                           double *dz, double *ds, int32_t n_threads)
{
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#endif
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)(2 * I));
#pragma omp for schedule(dynamic, 4)
        for (int64_t i = 0; i < n; ++i) {
            const int64_t t = tokens[i];
            const int32_t e = experts[i];
            oracle_pair_backward(H, I, layout, x + t * H, w1 + (size_t)e * H * 2 * I,
                                 b1 ? b1 + (size_t)e * 2 * I : NULL, w2 + (size_t)e * I * H,
                                 b2 ? b2 + (size_t)e * H : NULL, dout + t * H, scores[i],
                                 z, h + i * I, y + i * H, dy + i * H, dz + i * 2 * I, ds + i);
        }
        free(z);
    }
}
