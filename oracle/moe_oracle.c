/*
 * moe_oracle.c -- plain, slow CPU oracle for the sparse MoE FFN layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the reference the CUDA path is
 * checked against.  Only the tests, the smoke check and the benchmark's CPU
 * baseline leg load it; the product path never does.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Arithmetic: every sum, product, exp and division is done in IEEE double
 * (fp64).  Inputs are stored as bf16 or fp32 and are widened exactly to
 * double before use.  Loops run in the plain order of the definitions below;
 * there is no blocking, fusion or reordering beyond what the definitions
 * state.  OpenMP is used only to spread independent tokens (and the
 * independent channels of the FP8 weight encoder) over cores.
 *
 * What is computed, per token t (x_t is the row x[t, 0:H]):
 *
 *  1. Router logits: l[e] = sum_h x_t[h] * Wgate[e, h]  (+ bias[e] if given).
 *     The router is a bias-free linear layer hidden -> experts
 *     (page "腾讯混元Hy4 Preview深度技术解析", MoERouter sketch: a
 *     Linear(hidden, num_experts, bias=False) gate; page "腾讯混元Hy3正式版
 *     深度解析", SparseMoERouter sketch).
 *     The optional bias only realises a synthetic skewed-routing workload.
 *  2. p = softmax(l) over the experts, max-subtracted
 *     (page "腾讯混元Hy3正式版深度解析", SparseMoERouter.forward: softmax,
 *     then top-k).
 *  3. S = the k experts with the largest p, in descending order of p; exact
 *     ties are broken towards the lower expert index (torch.topk leaves the
 *     order of equal values unspecified; this is the reading adopted).
 *  4. w_j = scale * p_{S_j} / sum_{j'} p_{S_j'}: top-k renormalisation
 *     (page "腾讯混元Hy3正式版深度解析", SparseMoERouter.forward, weight
 *     normalisation; page "Hy4 preview config.json 终极深度解读", section
 *     "MoE 路由专家256 选 8", norm_topk_prob = true) followed by the global
 *     routed scaling factor (same config.json page and section:
 *     routed_scaling_factor 2.827 scales the routed experts' weighted
 *     output).  The 1e-8 epsilon of the Hy3 sketch is not added: the
 *     selected sum is >= k/E > 0.
 *  5. Expert FFN (SwiGLU, bias-free; page "腾讯混元Hy3正式版深度解析",
 *     MoEFeedForward sketch):
 *       g[i] = sum_h x_t[h] * W[e,0,i,h]      (gate_proj, nn.Linear [I,H])
 *       u[i] = sum_h x_t[h] * W[e,1,i,h]      (up_proj,   nn.Linear [I,H])
 *       g, u <- clamp(., -L, +L)  when L > 0  (page "Hy4 preview config.json
 *               终极深度解读", section "MoE 路由专家256 选 8",
 *               swiglu_limit 10.0: the SwiGLU activation is truncated to
 *               +-10; read as clamping both projections before the product)
 *       a[i] = g[i] / (1 + exp(-g[i])) * u[i]  (silu(g) * u)
 *       y[h] = sum_i a[i] * W[e,2,i,h]        (down projection, stored [I,H])
 *     Clamping is compare-and-select, so a NaN passes through unchanged.
 *  6. out_t = sum_j w_j * y_{S_j}  +  shared(x_t)
 *     where shared() is step 5 with the shared expert's weights and weight 1,
 *     no routed scale (page "腾讯混元Hy4 Preview深度技术解析", MoELayer.forward:
 *     routed output plus shared output; page "Hy4 preview config.json
 *     终极深度解读", n_shared_experts 1).
 *
 * Parity pins (what ties this file to something other than itself) are in
 * tests/test_oracle.py; every function here is pinned.
 */
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_F32 0
#define OR_BF16 1

/* Exact widening of one stored element to double. */
static double load_elem(const void* base, int dtype, int64_t i) {
    if (dtype == OR_F32) {
        return (double)((const float*)base)[i];
    }
    uint32_t bits = ((uint32_t)((const uint16_t*)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double clamp_keep_nan(double v, double limit) {
    if (v > limit) return limit;
    if (v < -limit) return -limit;
    return v; /* NaN compares false both ways and is returned unchanged */
}

/* Steps 1-4 for one token. logits/probs: [E] out; idx/w: [k] out. */
static void route_one(int64_t t, int H, int E, int k, int dtype,
                      const void* x, const void* gate_w, const float* bias,
                      double scale, double* logits, double* probs,
                      int32_t* idx, double* w) {
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int h = 0; h < H; ++h) {
            acc += load_elem(x, dtype, t * (int64_t)H + h) *
                   load_elem(gate_w, dtype, (int64_t)e * H + h);
        }
        if (bias) acc += (double)bias[e];
        logits[e] = acc;
    }
    double mx = logits[0];
    for (int e = 1; e < E; ++e)
        if (logits[e] > mx) mx = logits[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) {
        probs[e] = exp(logits[e] - mx);
        z += probs[e];
    }
    for (int e = 0; e < E; ++e) probs[e] /= z;

    /* top-k by repeated selection of the largest remaining probability;
     * scanning e upwards with a strict '>' keeps the lower index on ties. */
    unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
    double sel_sum = 0.0;
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || probs[e] > probs[best]) best = e;
        }
        taken[best] = 1;
        idx[j] = best;
        sel_sum += probs[best];
    }
    free(taken);
    for (int j = 0; j < k; ++j) w[j] = scale * probs[idx[j]] / sel_sum;
}

/* Step 5 for one token and one expert whose three [I,H] matrices start at
 * element offsets wg, wu, wd of `wbase`.  a: [I] scratch; y: [H] out. */
static void expert_ffn(int64_t t, int H, int I, int dtype, const void* x,
                       const void* wbase, int64_t wg, int64_t wu, int64_t wd,
                       double clip, double* a, double* y) {
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            double xv = load_elem(x, dtype, t * (int64_t)H + h);
            g += xv * load_elem(wbase, dtype, wg + (int64_t)i * H + h);
            u += xv * load_elem(wbase, dtype, wu + (int64_t)i * H + h);
        }
        if (clip > 0.0) {
            g = clamp_keep_nan(g, clip);
            u = clamp_keep_nan(u, clip);
        }
        a[i] = g / (1.0 + exp(-g)) * u;
    }
    for (int h = 0; h < H; ++h) y[h] = 0.0;
    for (int i = 0; i < I; ++i) {
        for (int h = 0; h < H; ++h) {
            y[h] += a[i] * load_elem(wbase, dtype, wd + (int64_t)i * H + h);
        }
    }
}

/* Element offsets of routed expert e's gate/up/down matrices in [E,3,I,H]. */
static int64_t mat_off(int e, int which, int I, int H) {
    return (((int64_t)e * 3 + which) * I) * (int64_t)H;
}

/*
 * oracle_route: steps 1-4 for the tokens listed in `tokens` (n_tok entries).
 * Outputs are per listed token: logits, probs [n_tok,E]; idx [n_tok,k];
 * w [n_tok,k].  logits/probs may be NULL.
 */
void oracle_route(int64_t T, int H, int E, int k, int dtype, const void* x,
                  const void* gate_w, const float* bias, double scale,
                  const int64_t* tokens, int64_t n_tok, double* logits,
                  double* probs, int32_t* idx, double* w) {
    (void)T;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t n = 0; n < n_tok; ++n) {
        double* l = (double*)malloc(sizeof(double) * (size_t)E);
        double* p = (double*)malloc(sizeof(double) * (size_t)E);
        route_one(tokens[n], H, E, k, dtype, x, gate_w, bias, scale, l, p,
                  idx + n * k, w + n * k);
        if (logits) memcpy(logits + n * E, l, sizeof(double) * (size_t)E);
        if (probs) memcpy(probs + n * E, p, sizeof(double) * (size_t)E);
        free(l);
        free(p);
    }
}

/*
 * oracle_forward: steps 1-6 for the listed tokens.
 *   expert_w : [E,3,I,H];  shared_w : [3,I,H] or NULL (no shared expert).
 *   forced_idx : NULL, or [n_tok,k] expert sets to use instead of the top-k
 *                of step 3 (the weights are still formed by step 4 from this
 *                oracle's own probabilities).  Tests use it only with sets
 *                this oracle itself derives (alternatives at near-ties).
 *   out : [n_tok,H]; idx_out : [n_tok,k] or NULL; w_out : [n_tok,k] or NULL.
 */
void oracle_forward(int64_t T, int H, int E, int k, int I, int dtype,
                    const void* x, const void* gate_w, const float* bias,
                    const void* expert_w, const void* shared_w, double scale,
                    double clip, const int64_t* tokens, int64_t n_tok,
                    const int32_t* forced_idx, double* out, int32_t* idx_out,
                    double* w_out) {
    (void)T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < n_tok; ++n) {
        int64_t t = tokens[n];
        double* l = (double*)malloc(sizeof(double) * (size_t)E);
        double* p = (double*)malloc(sizeof(double) * (size_t)E);
        double* a = (double*)malloc(sizeof(double) * (size_t)I);
        double* y = (double*)malloc(sizeof(double) * (size_t)H);
        int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
        double* w = (double*)malloc(sizeof(double) * (size_t)k);
        route_one(t, H, E, k, dtype, x, gate_w, bias, scale, l, p, idx, w);
        if (forced_idx) {
            double s = 0.0;
            for (int j = 0; j < k; ++j) {
                idx[j] = forced_idx[n * k + j];
                s += p[idx[j]];
            }
            for (int j = 0; j < k; ++j) w[j] = scale * p[idx[j]] / s;
        }
        double* o = out + n * (int64_t)H;
        for (int h = 0; h < H; ++h) o[h] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = idx[j];
            expert_ffn(t, H, I, dtype, x, expert_w, mat_off(e, 0, I, H),
                       mat_off(e, 1, I, H), mat_off(e, 2, I, H), clip, a, y);
            for (int h = 0; h < H; ++h) o[h] += w[j] * y[h];
        }
        if (shared_w) {
            expert_ffn(t, H, I, dtype, x, shared_w, mat_off(0, 0, I, H),
                       mat_off(0, 1, I, H), mat_off(0, 2, I, H), clip, a, y);
            for (int h = 0; h < H; ++h) o[h] += y[h];
        }
        if (idx_out) memcpy(idx_out + n * k, idx, sizeof(int32_t) * (size_t)k);
        if (w_out) memcpy(w_out + n * k, w, sizeof(double) * (size_t)k);
        free(l);
        free(p);
        free(a);
        free(y);
        free(idx);
        free(w);
    }
}

/*
 * oracle_dense_bruteforce: evaluates ALL E routed experts for each listed
 * token and combines them with a caller-given dense weight vector
 * dense_w [n_tok,E] (zero outside the selected set), plus the shared expert.
 * out: [n_tok,H].  Used to cross-check the sparse dispatch of
 * oracle_forward.
 */
void oracle_dense_bruteforce(int64_t T, int H, int E, int I, int dtype,
                             const void* x, const void* expert_w,
                             const void* shared_w, double clip,
                             const int64_t* tokens, int64_t n_tok,
                             const double* dense_w, double* out) {
    (void)T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < n_tok; ++n) {
        int64_t t = tokens[n];
        double* a = (double*)malloc(sizeof(double) * (size_t)I);
        double* y = (double*)malloc(sizeof(double) * (size_t)H);
        double* o = out + n * (int64_t)H;
        for (int h = 0; h < H; ++h) o[h] = 0.0;
        for (int e = 0; e < E; ++e) {
            expert_ffn(t, H, I, dtype, x, expert_w, mat_off(e, 0, I, H),
                       mat_off(e, 1, I, H), mat_off(e, 2, I, H), clip, a, y);
            for (int h = 0; h < H; ++h) o[h] += dense_w[n * E + e] * y[h];
        }
        if (shared_w) {
            expert_ffn(t, H, I, dtype, x, shared_w, mat_off(0, 0, I, H),
                       mat_off(0, 1, I, H), mat_off(0, 2, I, H), clip, a, y);
            for (int h = 0; h < H; ++h) o[h] += y[h];
        }
        free(a);
        free(y);
    }
}

/*
 * oracle_expert_rows: step 5 alone, row by row.  For each of n_rows rows,
 * runs expert row_expert[r] (or the shared expert when row_expert[r] == E,
 * using shared_w) on token row_token[r] of x.  out: [n_rows,H].
 * This is the per-row content of the permuted expert output.
 */
void oracle_expert_rows(int H, int E, int I, int dtype, const void* x,
                        const void* expert_w, const void* shared_w,
                        double clip, const int32_t* row_token,
                        const int32_t* row_expert, int64_t n_rows,
                        double* out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        double* a = (double*)malloc(sizeof(double) * (size_t)I);
        int e = row_expert[r];
        if (e == E) {
            expert_ffn(row_token[r], H, I, dtype, x, shared_w,
                       mat_off(0, 0, I, H), mat_off(0, 1, I, H),
                       mat_off(0, 2, I, H), clip, a, out + r * (int64_t)H);
        } else {
            expert_ffn(row_token[r], H, I, dtype, x, expert_w,
                       mat_off(e, 0, I, H), mat_off(e, 1, I, H),
                       mat_off(e, 2, I, H), clip, a, out + r * (int64_t)H);
        }
        free(a);
    }
}

/*
 * oracle_permute: the dispatch bookkeeping, written as a counting sort.
 * Every (token t, slot j) assignment goes to expert idx[t,j].  Rows of the
 * permuted order are grouped by expert (expert 0 first) and, inside an
 * expert, ordered by token then slot.  (The per-expert mask dispatch of page
 * tqpw.cn/news/149001, section 2.1 "MoE 的基本工作原理", visits an expert's
 * tokens in token order; the triple loop of page "腾讯混元Hy4 Preview深度技术
 * 解析", MoELayer.forward, visits (token, slot) in that order.)
 *   counts  : [E]     number of assignments per expert
 *   offsets : [E+1]   exclusive prefix sum of counts; offsets[E] = T*k
 *   pos     : [T,k]   permuted row of assignment (t,j)
 *   src     : [T*k]   token of each permuted row
 */
void oracle_permute(int64_t T, int E, int k, const int32_t* idx,
                    int32_t* counts, int32_t* offsets, int32_t* pos,
                    int32_t* src) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) counts[idx[t * k + j]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (int64_t t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int e = idx[t * k + j];
            int32_t r = fill[e]++;
            pos[t * k + j] = r;
            src[r] = (int32_t)t;
        }
    }
    free(fill);
}

/*
 * oracle_combine: out[t] = sum_j w[t,j] * y_perm[pos[t,j]] + shared_y[t]
 * (shared_y may be NULL).  y_perm/shared_y are given as double arrays.
 * out: [T,H].
 */
void oracle_combine(int64_t T, int H, int k, const double* y_perm,
                    const int32_t* pos, const double* w,
                    const double* shared_y, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double* o = out + t * (int64_t)H;
        for (int h = 0; h < H; ++h) o[h] = 0.0;
        for (int j = 0; j < k; ++j) {
            const double* y = y_perm + (int64_t)pos[t * k + j] * H;
            for (int h = 0; h < H; ++h) o[h] += w[t * k + j] * y[h];
        }
        if (shared_y) {
            for (int h = 0; h < H; ++h) o[h] += shared_y[t * (int64_t)H + h];
        }
    }
}

/*
 * oracle_router_stats: the router's load-balancing statistics (page
 * "腾讯混元Hy3正式版深度解析", SparseMoERouter._compute_load_balancing_loss and
 * the expert-count update in forward), over all T tokens:
 *   P[e]   = (1/T) * sum_t p[t,e]                 mean routing probability
 *   cnt[e] = #{(t,j) : idx[t,j] == e}             selections of expert e
 *   f[e]   = cnt[e] / (T*k)                        selection frequency
 *   aux    = E * sum_e P[e] * f[e]                 auxiliary loss
 *   ema_counts[e] <- momentum * ema_counts[e] + (1 - momentum) * cnt[e]
 *   ema_total     <- momentum * ema_total + (1 - momentum) * T
 * (the sketch uses momentum 0.9).  p and idx are steps 2 and 3 above.
 * ema_counts / ema_total may be NULL (not updated).
 */
void oracle_router_stats(int64_t T, int H, int E, int k, int dtype, const void* x,
                         const void* gate_w, const float* bias, double momentum, double* P,
                         double* f, int64_t* cnt, double* aux, double* ema_counts,
                         double* ema_total) {
    for (int e = 0; e < E; ++e) {
        P[e] = 0.0;
        cnt[e] = 0;
    }
    double* l = (double*)malloc(sizeof(double) * (size_t)E);
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* w = (double*)malloc(sizeof(double) * (size_t)k);
    for (int64_t t = 0; t < T; ++t) {
        route_one(t, H, E, k, dtype, x, gate_w, bias, 1.0, l, p, idx, w);
        for (int e = 0; e < E; ++e) P[e] += p[e];
        for (int j = 0; j < k; ++j) cnt[idx[j]] += 1;
    }
    double a = 0.0;
    for (int e = 0; e < E; ++e) {
        P[e] /= (double)T;
        f[e] = (double)cnt[e] / ((double)T * (double)k);
        a += P[e] * f[e];
    }
    *aux = (double)E * a;
    if (ema_counts)
        for (int e = 0; e < E; ++e)
            ema_counts[e] = momentum * ema_counts[e] + (1.0 - momentum) * (double)cnt[e];
    if (ema_total) *ema_total = momentum * (*ema_total) + (1.0 - momentum) * (double)T;
    free(l);
    free(p);
    free(idx);
    free(w);
}

/* ------------------------------------------------------------------------
 * FP8 expert weights (the FP8 deployment noted on page "1M上下文实战：Hy4
 * preview如何从容处理百万token级长文档", section "最快部署 1M 上下文"; the pages
 * give no number format, so the reading is stated here).
 *
 * E4M3 (OCP FP8): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; no
 * infinities; code S.1111.111 is NaN; largest finite 448; subnormals
 * m * 2^-9.  Encoding rounds to nearest, ties to even, saturating to +-448.
 *
 * Scales are powers of two, so dividing by a scale is exact in any binary
 * floating-point format and the encoding decision is the same wherever it
 * is taken:
 *   pow2_scale(amax) = 2^ceil(log2(amax / 448))  (1 when amax == 0)
 * Weights: gate/up rows i and down columns h each get
 *   s = pow2_scale(max |w| over that row / column), q = e4m3(w / s).
 * Token rows x_t: s_x = pow2_scale(max_h |x_t[h]|), q = e4m3(x_t / s_x).
 * The SwiGLU output h is bounded by the clamp L (|h| <= silu(L) L), so it
 * uses one fixed scale s_h = pow2_scale(silu(L) * L): h_q = e4m3(h / s_h).
 * The expert FFN then computes, in fp64 on the decoded codes,
 *   g[i] = s_x s_g[i] sum_h xq[h] gq[i,h],   u[i] likewise,
 *   h[i] = silu(clamp g) clamp u,   y[c] = s_h s_d[c] sum_i hq[i] dq[i,c].
 * ------------------------------------------------------------------------ */

double e4m3_decode(uint8_t code) {
    const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

uint8_t e4m3_encode(double v) {
    if (isnan(v)) return 0x7F;
    const int sign = v < 0 || (v == 0.0 && signbit(v));
    double a = fabs(v);
    if (a >= 448.0) return (uint8_t)((sign << 7) | 0x7E);
    /* all finite codes in increasing order of magnitude: pick the nearest,
     * ties to the even code (codes 0..126 encode increasing magnitudes) */
    int lo = 0, hi = 126;
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (e4m3_decode((uint8_t)mid) <= a) lo = mid;
        else hi = mid;
    }
    double dlo = a - e4m3_decode((uint8_t)lo), dhi = e4m3_decode((uint8_t)hi) - a;
    int c;
    if (dlo < dhi) c = lo;
    else if (dhi < dlo) c = hi;
    else c = (lo % 2 == 0) ? lo : hi;
    return (uint8_t)((sign << 7) | c);
}

double pow2_scale(double amax) {
    if (!(amax > 0.0)) return 1.0;
    return ldexp(1.0, (int)ceil(log2(amax / 448.0)));
}

/*
 * oracle_quantize_weights_fp8: w [n_mats/3 experts,3,I,H] (bf16/fp32) ->
 * q (same shape, E4M3 codes), s_gu [n_experts,2,I] (gate, up row scales),
 * s_d [n_experts,H] (down column scales).
 */
void oracle_quantize_weights_fp8(int n_experts, int I, int H, int dtype, const void* w,
                                 uint8_t* q, double* s_gu, double* s_d) {
    /* gate and up rows: row r = (e*2 + m)*I + i */
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < (int64_t)n_experts * 2 * I; ++r) {
        const int64_t e = r / (2 * (int64_t)I), m = (r / I) % 2, i = r % I;
        const int64_t base = ((e * 3 + m) * I + i) * H;
        double amax = 0.0;
        for (int h = 0; h < H; ++h) {
            double v = fabs(load_elem(w, dtype, base + h));
            if (v > amax) amax = v;
        }
        const double sc = pow2_scale(amax);
        s_gu[r] = sc;
        for (int h = 0; h < H; ++h) q[base + h] = e4m3_encode(load_elem(w, dtype, base + h) / sc);
    }
    /* down columns: column c = e*H + h */
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < (int64_t)n_experts * H; ++c) {
        const int64_t e = c / H, h = c % H;
        const int64_t dbase = (e * 3 + 2) * I * (int64_t)H;
        double amax = 0.0;
        for (int i = 0; i < I; ++i) {
            double v = fabs(load_elem(w, dtype, dbase + (int64_t)i * H + h));
            if (v > amax) amax = v;
        }
        const double sc = pow2_scale(amax);
        s_d[c] = sc;
        for (int i = 0; i < I; ++i)
            q[dbase + (int64_t)i * H + h] =
                e4m3_encode(load_elem(w, dtype, dbase + (int64_t)i * H + h) / sc);
    }
}

/* One expert's FFN on quantized codes (see above).  xq: [H] codes of the
 * token, sx its scale; q/s_gu/s_d as produced above for expert e. */
static void expert_ffn_fp8(int H, int I, const uint8_t* xq, double sx, const uint8_t* q,
                           const double* s_gu, const double* s_d, int e, double clip,
                           double s_h, double* y) {
    double* hq = (double*)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < I; ++i) {
        const uint8_t* gr = q + (((int64_t)e * 3 + 0) * I + i) * H;
        const uint8_t* ur = q + (((int64_t)e * 3 + 1) * I + i) * H;
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            double xv = e4m3_decode(xq[h]);
            g += xv * e4m3_decode(gr[h]);
            u += xv * e4m3_decode(ur[h]);
        }
        g *= sx * s_gu[((int64_t)e * 2 + 0) * I + i];
        u *= sx * s_gu[((int64_t)e * 2 + 1) * I + i];
        g = clamp_keep_nan(g, clip);
        u = clamp_keep_nan(u, clip);
        double hv = g / (1.0 + exp(-g)) * u;
        hq[i] = e4m3_decode(e4m3_encode(hv / s_h));
    }
    const uint8_t* dm = q + ((int64_t)e * 3 + 2) * I * (int64_t)H;
    for (int c = 0; c < H; ++c) y[c] = 0.0;
    for (int i = 0; i < I; ++i)
        for (int c = 0; c < H; ++c) y[c] += hq[i] * e4m3_decode(dm[(int64_t)i * H + c]);
    for (int c = 0; c < H; ++c) y[c] *= s_h * s_d[(int64_t)e * H + c];
    free(hq);
}

/*
 * oracle_forward_fp8: the layer with FP8 expert weights (shared expert too),
 * routing as in oracle_forward (bf16/fp32 gate, unquantized).  clip > 0 is
 * required (it bounds h).  q/s_gu/s_d: routed experts; sq/ss_gu/ss_d: the
 * shared expert (NULL when absent).  out: [n_tok,H]; idx_out/w_out as above.
 */
void oracle_forward_fp8(int64_t T, int H, int E, int k, int I, int dtype, const void* x,
                        const void* gate_w, const float* bias, const uint8_t* q,
                        const double* s_gu, const double* s_d, const uint8_t* sq,
                        const double* ss_gu, const double* ss_d, double scale, double clip,
                        const int64_t* tokens, int64_t n_tok, const int32_t* forced_idx,
                        double* out, int32_t* idx_out, double* w_out) {
    (void)T;
    const double s_h = pow2_scale(clip / (1.0 + exp(-clip)) * clip);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < n_tok; ++n) {
        int64_t t = tokens[n];
        double* l = (double*)malloc(sizeof(double) * (size_t)E);
        double* p = (double*)malloc(sizeof(double) * (size_t)E);
        double* y = (double*)malloc(sizeof(double) * (size_t)H);
        uint8_t* xq = (uint8_t*)malloc((size_t)H);
        int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
        double* w = (double*)malloc(sizeof(double) * (size_t)k);
        route_one(t, H, E, k, dtype, x, gate_w, bias, scale, l, p, idx, w);
        if (forced_idx) {
            double sum = 0.0;
            for (int j = 0; j < k; ++j) {
                idx[j] = forced_idx[n * k + j];
                sum += p[idx[j]];
            }
            for (int j = 0; j < k; ++j) w[j] = scale * p[idx[j]] / sum;
        }
        double amax = 0.0;
        for (int h = 0; h < H; ++h) {
            double v = fabs(load_elem(x, dtype, t * (int64_t)H + h));
            if (v > amax) amax = v;
        }
        const double sx = pow2_scale(amax);
        for (int h = 0; h < H; ++h) xq[h] = e4m3_encode(load_elem(x, dtype, t * (int64_t)H + h) / sx);
        double* o = out + n * (int64_t)H;
        for (int h = 0; h < H; ++h) o[h] = 0.0;
        for (int j = 0; j < k; ++j) {
            expert_ffn_fp8(H, I, xq, sx, q, s_gu, s_d, idx[j], clip, s_h, y);
            for (int h = 0; h < H; ++h) o[h] += w[j] * y[h];
        }
        if (sq) {
            expert_ffn_fp8(H, I, xq, sx, sq, ss_gu, ss_d, 0, clip, s_h, y);
            for (int h = 0; h < H; ++h) o[h] += y[h];
        }
        if (idx_out) memcpy(idx_out + n * k, idx, sizeof(int32_t) * (size_t)k);
        if (w_out) memcpy(w_out + n * k, w, sizeof(double) * (size_t)k);
        free(l);
        free(p);
        free(y);
        free(xq);
        free(idx);
        free(w);
    }
}

/* Number of OpenMP threads the oracle will use (for reporting). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
