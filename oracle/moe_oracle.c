/*
 * CPU oracle for the int4 expert-grouped mixture-of-experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code with the CUDA library.
 *
 * What the layer computes comes from the inblix article "Perplexity's Lily
 * engine beats MLX by 35% on M5 Max, no PyTorch needed", third paragraph
 * (cited below as "inblix, paragraph 3"): expert routing,
 * a prefix scan of per-expert counts, a scatter into expert order with a
 * block map, and a grouped GEMM over 4-bit weights that are dequantised
 * inside the GEMM.  The pages fix no formula; the readings taken where they
 * are silent are listed with each function (routing by softmax top-k,
 * SwiGLU experts, affine int4 groups along the reduction dimension, a
 * routing-weighted combine).
 *
 * Precision: the router logits decide an integer (the top-k choice), so
 * they are computed in fp32 in one fixed summation order that the CUDA
 * router also follows (oracle_router_logits).  Everything else is float64,
 * which makes it the exact value of the definition to well below the
 * tolerance the layer output is checked against.
 *
 * Parallelism: OpenMP only splits independent outputs (tokens, rows);
 * no sum is split or reordered by it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

int oracle_abi_version(void) { return 1; }

/*
 * Router logits (expert routing: inblix, paragraph 3; the blog post
 * "Perplexity's Lily beats MLX by 1.35x by doing one thing: single-model
 * Rust/Metal engines", section "Why one model on one chip is faster", says
 * the routing is hard-coded for the one MoE model).
 *
 * l[t,e] = S[t,e] + b_r[e], where S is x[t,:] . W_r[:,e] summed in this
 * order, in fp32:
 *   - 32 partial chains: chain p holds the terms i = p, p+32, p+64, ... and
 *     accumulates them in ascending i with fused multiply-add,
 *     v_p <- fmaf(x[t,i], W_r[i,e], v_p), starting from v_p = 0;
 *   - the chains are combined by a butterfly: for m = 16, 8, 4, 2, 1 every
 *     v_p becomes v_p + v_(p xor m) (all p at once); S is v_0 afterwards;
 *   - the bias is one fp32 add (b_r == NULL means no bias).
 * Reading: the pages give no summation order, but the top-k indices must
 * match the CUDA path exactly, so both follow this one.
 *
 * x: bf16 bits [T, d] row-major; W_r: fp32 [d, E] row-major; logits: [T, E].
 */
void oracle_router_logits(const uint16_t *x, int64_t T, int64_t d,
                          const float *W_r, int64_t E, const float *b_r,
                          float *logits)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = 0; t < T; ++t) {
        float *v = (float *)calloc((size_t)(E * 32), sizeof(float));
        float w[32];
        const uint16_t *xr = x + t * d;
        for (int64_t i = 0; i < d; ++i) {
            const int p = (int)(i % 32);
            const float xi = bf16_to_float(xr[i]);
            const float *wr = W_r + i * E;
            for (int64_t e = 0; e < E; ++e)
                v[e * 32 + p] = fmaf(xi, wr[e], v[e * 32 + p]);
        }
        for (int64_t e = 0; e < E; ++e) {
            float *ve = v + e * 32;
            for (int m = 16; m >= 1; m >>= 1) {
                for (int p = 0; p < 32; ++p)
                    w[p] = ve[p] + ve[p ^ m];
                memcpy(ve, w, sizeof w);
            }
            float l = ve[0];
            if (b_r)
                l = l + b_r[e];
            logits[t * E + e] = l;
        }
        free(v);
    }
}

/*
 * Top-k selection.  Experts are ranked by logit, larger first; equal
 * logits rank the lower expert id first (so -0 and +0 tie).  The k best,
 * in rank order, form topk_idx[t, 0..k-1].
 * Inputs must be finite.
 */
void oracle_topk(const float *logits, int64_t T, int64_t E, int64_t k,
                 int32_t *topk_idx)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        unsigned char *taken = (unsigned char *)calloc((size_t)E, 1);
        for (int64_t j = 0; j < k; ++j) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                if (taken[e])
                    continue;
                if (best < 0 || l[e] > l[best])
                    best = e;
            }
            taken[best] = 1;
            topk_idx[t * k + j] = (int32_t)best;
        }
        free(taken);
    }
}

/*
 * Routing weights: a softmax over the k selected logits,
 * w[t,j] = exp(l_j - l_0) / sum_j' exp(l_j' - l_0), in float64 from the fp32
 * logits.  Reading: softmax top-k with the weights renormalised over the
 * selected experts so they sum to one per token.
 */
void oracle_topk_weights(const float *logits, const int32_t *topk_idx,
                         int64_t T, int64_t E, int64_t k, double *topk_w)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        const int32_t *idx = topk_idx + t * k;
        const double l0 = (double)l[idx[0]];
        double denom = 0.0;
        for (int64_t j = 0; j < k; ++j)
            denom += exp((double)l[idx[j]] - l0);
        for (int64_t j = 0; j < k; ++j)
            topk_w[t * k + j] = exp((double)l[idx[j]] - l0) / denom;
    }
}

/*
 * Prefix scan (inblix, paragraph 3): counts[e] is the number of
 * assignments a = t*k + j with topk_idx[a] == e; offsets is their exclusive
 * prefix sum, offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e].
 * Reading: offsets carry no padding; padding only exists in the block map.
 */
void oracle_counts_offsets(const int32_t *topk_idx, int64_t T, int64_t k,
                           int64_t E, int32_t *counts, int32_t *offsets)
{
    for (int64_t e = 0; e < E; ++e)
        counts[e] = 0;
    for (int64_t a = 0; a < T * k; ++a)
        counts[topk_idx[a]] += 1;
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
}

/*
 * Scatter into expert-contiguous order (inblix, paragraph 3): visit the
 * assignments a = 0 .. T*k-1 in ascending order; each is placed at the next
 * free slot of its expert, p = offsets[e] + cursor[e]++.  sorted_assign[p]
 * = a and pos[a] = p.  Reading: inside one expert the order is ascending a,
 * which is ascending token (a token never picks an expert twice).
 */
void oracle_scatter(const int32_t *topk_idx, const int32_t *offsets,
                    int64_t T, int64_t k, int64_t E, int32_t *sorted_assign,
                    int32_t *pos)
{
    int32_t *cursor = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    for (int64_t a = 0; a < T * k; ++a) {
        const int32_t e = topk_idx[a];
        const int32_t p = offsets[e] + cursor[e];
        cursor[e] += 1;
        sorted_assign[p] = (int32_t)a;
        pos[a] = p;
    }
    free(cursor);
}

/*
 * Block map (inblix, paragraph 3): expert e's rows are cut into
 * ceil(counts[e] / BT) tiles of BT rows, in ascending e and ascending row;
 * entry b = (e, offsets[e] + i*BT, min(BT, counts[e] - i*BT)), stored as three
 * int32.  block_offsets is the exclusive prefix sum of the tile counts, so
 * block_offsets[E] is the number of tiles, which is returned.  Experts with
 * no rows get no tile.  BT is the tile height chosen by the GEMM.
 */
int64_t oracle_block_map(const int32_t *counts, const int32_t *offsets,
                         int64_t E, int64_t BT, int32_t *block_offsets,
                         int32_t *block_map)
{
    int64_t nb = 0;
    for (int64_t e = 0; e < E; ++e) {
        block_offsets[e] = (int32_t)nb;
        const int64_t tiles = (counts[e] + BT - 1) / BT;
        for (int64_t i = 0; i < tiles; ++i) {
            const int64_t rows = counts[e] - i * BT < BT ? counts[e] - i * BT : BT;
            block_map[3 * nb + 0] = (int32_t)e;
            block_map[3 * nb + 1] = (int32_t)(offsets[e] + i * BT);
            block_map[3 * nb + 2] = (int32_t)rows;
            ++nb;
        }
    }
    block_offsets[E] = (int32_t)nb;
    return nb;
}

/*
 * 4-bit dequantisation (inblix, paragraph 3: 4-bit weights expanded to
 * bfloat16 inside the GEMM).  Weight (n, kk) of one expert:
 *   q = (byte[n, kk/2] >> (4 * (kk % 2))) & 0xF   (low nibble = even kk),
 *   w = q * scale[n, kk/G] + bias[n, kk/G],
 * in float64, where it is exact.  Reading: affine groups of G weights along
 * K, the reduction dimension of the projection.
 *
 * q: [N, K/2] bytes; scale, bias: bf16 bits [N, K/G]; out: float64 [N, K].
 */
void oracle_dequant(const uint8_t *q, const uint16_t *scale,
                    const uint16_t *bias, int64_t N, int64_t K, int64_t G,
                    double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t kk = 0; kk < K; ++kk) {
            const unsigned nib = (q[n * (K / 2) + kk / 2] >> (4 * (kk % 2))) & 0xFu;
            const double s = (double)bf16_to_float(scale[n * (K / G) + kk / G]);
            const double b = (double)bf16_to_float(bias[n * (K / G) + kk / G]);
            out[n * K + kk] = (double)nib * s + b;
        }
    }
}

/* silu(g) = g / (1 + exp(-g)) */
static double silu(double g) { return g / (1.0 + exp(-g)); }

/*
 * One expert applied to one token (SwiGLU expert, float64):
 *   g[n] = sum_kk Wg[n,kk] x[kk],  u[n] = sum_kk Wu[n,kk] x[kk]  (kk ascending)
 *   h[n] = silu(g[n]) * u[n]
 *   o[m] = sum_n Wd[m,n] h[n]                                    (n ascending)
 * Reading: SwiGLU = silu(gate) * up, no shared expert.
 * Wg, Wu: float64 [f, d]; Wd: float64 [d, f]; x: float64 [d].
 */
static void expert_apply(const double *Wg, const double *Wu, const double *Wd,
                         int64_t d, int64_t f, const double *x, double *h,
                         double *o)
{
    for (int64_t n = 0; n < f; ++n) {
        double g = 0.0, u = 0.0;
        for (int64_t kk = 0; kk < d; ++kk) {
            g += Wg[n * d + kk] * x[kk];
            u += Wu[n * d + kk] * x[kk];
        }
        h[n] = silu(g) * u;
    }
    for (int64_t m = 0; m < d; ++m) {
        double acc = 0.0;
        for (int64_t n = 0; n < f; ++n)
            acc += Wd[m * f + n] * h[n];
        o[m] = acc;
    }
}

typedef struct {
    const uint8_t *gate_q, *up_q, *down_q;
    const uint16_t *gate_s, *gate_b, *up_s, *up_b, *down_s, *down_b;
} oracle_weights_t;

/*
 * The expert MLP over the expert-ordered rows (the grouped GEMM of the
 * inblix, paragraph 3, without any tiling):
 * for every sorted row p, with a = sorted_assign[p], t = a / k and
 * e = topk_idx[a]: (h[p,:], o[p,:]) = expert e applied to x[t,:].
 * Each expert's weights are dequantised once (oracle_dequant) and used for
 * all of its rows.
 * h: float64 [T*k, f] (may be NULL); o: float64 [T*k, d].
 */
void oracle_expert_rows(const uint16_t *x, int64_t T, int64_t d, int64_t E,
                        int64_t k, int64_t f, int64_t G,
                        const oracle_weights_t *w, const int32_t *topk_idx,
                        const int32_t *offsets, const int32_t *sorted_assign,
                        double *h_out, double *o_out)
{
    double *Wg = (double *)malloc((size_t)(f * d) * sizeof(double));
    double *Wu = (double *)malloc((size_t)(f * d) * sizeof(double));
    double *Wd = (double *)malloc((size_t)(d * f) * sizeof(double));
    for (int64_t e = 0; e < E; ++e) {
        const int64_t r0 = offsets[e], r1 = offsets[e + 1];
        if (r1 == r0)
            continue;
        oracle_dequant(w->gate_q + e * f * (d / 2), w->gate_s + e * f * (d / G),
                       w->gate_b + e * f * (d / G), f, d, G, Wg);
        oracle_dequant(w->up_q + e * f * (d / 2), w->up_s + e * f * (d / G),
                       w->up_b + e * f * (d / G), f, d, G, Wu);
        oracle_dequant(w->down_q + e * d * (f / 2), w->down_s + e * d * (f / G),
                       w->down_b + e * d * (f / G), d, f, G, Wd);
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t p = r0; p < r1; ++p) {
            const int64_t a = sorted_assign[p];
            const int64_t t = a / k;
            double *xv = (double *)malloc((size_t)d * sizeof(double));
            double *hv = (double *)malloc((size_t)f * sizeof(double));
            for (int64_t i = 0; i < d; ++i)
                xv[i] = (double)bf16_to_float(x[t * d + i]);
            expert_apply(Wg, Wu, Wd, d, f, xv, hv, o_out + p * d);
            if (h_out)
                memcpy(h_out + p * f, hv, (size_t)f * sizeof(double));
            free(xv);
            free(hv);
        }
        (void)topk_idx;
    }
    free(Wg);
    free(Wu);
    free(Wd);
}

/*
 * Routing-weighted gather-combine: y[t,m] = sum_{j=0..k-1} topk_w[t,j] *
 * o[pos[t*k+j], m], float64, j ascending.
 */
void oracle_combine(const double *o, const double *topk_w, const int32_t *pos,
                    int64_t T, int64_t k, int64_t d, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t m = 0; m < d; ++m) {
            double acc = 0.0;
            for (int64_t j = 0; j < k; ++j)
                acc += topk_w[t * k + j] * o[(int64_t)pos[t * k + j] * d + m];
            y[t * d + m] = acc;
        }
    }
}

/*
 * The whole layer for the given tokens through the pages' steps in order:
 * routing -> counts and prefix scan -> scatter -> expert rows -> combine.
 * All intermediates are caller buffers so the tests can compare them:
 * logits f32 [T,E], topk_idx [T,k], topk_w f64 [T,k], counts [E],
 * offsets [E+1], sorted_assign [T*k], pos [T*k], o f64 [T*k, d],
 * h f64 [T*k, f] (may be NULL), y f64 [T, d].
 */
void oracle_forward(const uint16_t *x, int64_t T, int64_t d, int64_t E,
                    int64_t k, int64_t f, int64_t G, const float *W_r,
                    const float *b_r, const oracle_weights_t *w, float *logits,
                    int32_t *topk_idx, double *topk_w, int32_t *counts,
                    int32_t *offsets, int32_t *sorted_assign, int32_t *pos,
                    double *h, double *o, double *y)
{
    oracle_router_logits(x, T, d, W_r, E, b_r, logits);
    oracle_topk(logits, T, E, k, topk_idx);
    oracle_topk_weights(logits, topk_idx, T, E, k, topk_w);
    oracle_counts_offsets(topk_idx, T, k, E, counts, offsets);
    oracle_scatter(topk_idx, offsets, T, k, E, sorted_assign, pos);
    oracle_expert_rows(x, T, d, E, k, f, G, w, topk_idx, offsets, sorted_assign, h, o);
    oracle_combine(o, topk_w, pos, T, k, d, y);
}

/*
 * The layer output for a few chosen tokens of a large batch, one token at a
 * time: route token t alone, then y[t] = sum_j w_j * expert_{e_j}(x[t]).
 * The expert weights are dequantised row by row on the fly, so no expert is
 * expanded in full.  Used to check sampled outputs at sizes where the full
 * forward is too slow.  tokens: [n]; y: float64 [n, d];
 * idx_out: [n, k] (may be NULL); w_out: float64 [n, k] (may be NULL).
 */
void oracle_token_outputs(const uint16_t *x, int64_t d, int64_t E, int64_t k,
                          int64_t f, int64_t G, const float *W_r,
                          const float *b_r, const oracle_weights_t *w,
                          const int64_t *tokens, int64_t n, double *y,
                          int32_t *idx_out, double *w_out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t s = 0; s < n; ++s) {
        const int64_t t = tokens[s];
        float *l = (float *)malloc((size_t)E * sizeof(float));
        int32_t *idx = (int32_t *)malloc((size_t)k * sizeof(int32_t));
        double *rw = (double *)malloc((size_t)k * sizeof(double));
        double *xv = (double *)malloc((size_t)d * sizeof(double));
        double *hv = (double *)malloc((size_t)f * sizeof(double));
        double *rowg = (double *)malloc((size_t)d * sizeof(double));
        double *rowu = (double *)malloc((size_t)d * sizeof(double));
        double *rowd = (double *)malloc((size_t)f * sizeof(double));
        oracle_router_logits(x + t * d, 1, d, W_r, E, b_r, l);
        oracle_topk(l, 1, E, k, idx);
        oracle_topk_weights(l, idx, 1, E, k, rw);
        for (int64_t i = 0; i < d; ++i)
            xv[i] = (double)bf16_to_float(x[t * d + i]);
        for (int64_t m = 0; m < d; ++m)
            y[s * d + m] = 0.0;
        for (int64_t j = 0; j < k; ++j) {
            const int64_t e = idx[j];
            for (int64_t nn = 0; nn < f; ++nn) {
                const int64_t row = e * f + nn;
                oracle_dequant(w->gate_q + row * (d / 2), w->gate_s + row * (d / G),
                               w->gate_b + row * (d / G), 1, d, G, rowg);
                oracle_dequant(w->up_q + row * (d / 2), w->up_s + row * (d / G),
                               w->up_b + row * (d / G), 1, d, G, rowu);
                double g = 0.0, u = 0.0;
                for (int64_t kk = 0; kk < d; ++kk) {
                    g += rowg[kk] * xv[kk];
                    u += rowu[kk] * xv[kk];
                }
                hv[nn] = silu(g) * u;
            }
            for (int64_t m = 0; m < d; ++m) {
                const int64_t row = e * d + m;
                oracle_dequant(w->down_q + row * (f / 2), w->down_s + row * (f / G),
                               w->down_b + row * (f / G), 1, f, G, rowd);
                double acc = 0.0;
                for (int64_t nn = 0; nn < f; ++nn)
                    acc += rowd[nn] * hv[nn];
                /* j ascending, as in oracle_combine */
                y[s * d + m] += rw[j] * acc;
            }
        }
        if (idx_out)
            memcpy(idx_out + s * k, idx, (size_t)k * sizeof(int32_t));
        if (w_out)
            memcpy(w_out + s * k, rw, (size_t)k * sizeof(double));
        free(l); free(idx); free(rw); free(xv); free(hv);
        free(rowg); free(rowu); free(rowd);
    }
}
