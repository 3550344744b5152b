/*
 * moe_oracle.c -- fp64 CPU oracle for the forward pass of a Mixtral-style
 * sparse Mixture-of-Experts feed-forward layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load this file
 * or the library built from it: only the tests, the smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA library; it reads the same bf16 input bits and nothing
 * else.
 *
 * What it computes, per token t (a plain restatement of the method, evaluated
 * token by token in double precision with no intermediate rounding):
 *
 *   l[e]   = sum_i x[t,i] * Wg[e,i]  (+ bias[e] when a bias is given)
 *       -- the router is a bias-free linear layer d -> E
 *          ("Mistral 8x7B SMoE ..." (jsqmd.com) sec. 3.2 Gating Network;
 *           "MoE: ..." (theaiera.top, LLMs-from-scratch ch.10) sec. 10.3)
 *   sel    = the k experts with the largest l, ordered by (l descending,
 *            expert index ascending): equal logits go to the lower index
 *       -- torch.topk in sec. 10.3 / sec. 3.2; the pages fix no tie rule,
 *          the lower-index rule is the reading this library adopts
 *   w[j]   = exp(l[sel[j]] - m) / sum_j' exp(l[sel[j']] - m),  m = l[sel[0]]
 *       -- softmax over the k selected logits only, so the weights sum to 1
 *          (sec. 10.3; sec. 3.2 step 3)
 *   h_e[f] = silu(sum_i W1[e,f,i] x[t,i]) * (sum_i W3[e,f,i] x[t,i])
 *   y_e[o] = sum_f W2[e,o,f] h_e[f]
 *       -- the SwiGLU expert w2(silu(w1 x) * w3 x)
 *          ("Mistral 8x7B SMoE ..." sec. 3.1 FeedForward;
 *           "Mixtral and MoE architecture" (astro-blog) FeedForward listing)
 *   out[t] = sum_j w[j] * y_{sel[j]}   summed in slot order j = 0..k-1
 *            (+ the shared expert's SwiGLU output, unweighted, when given)
 *       -- weighted scatter-add back to token order and the always-on shared
 *          expert (sec. 10.4 and sec. 10.5 of the theaiera.top chapter)
 *   silu(z) = z / (1 + exp(-z))
 *
 * Sums run in index order with one accumulator; OpenMP only splits the
 * independent tokens across threads and changes no arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Widen raw bf16 bits to double; exact (bf16 is the top half of a float). */
static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Router for one token: logits, the selected set, the softmax weights over
 * that set and the gap between the k-th and (k+1)-th largest logits
 * (+inf when k == E).  The selection is k rounds of "largest remaining
 * logit"; a strict '>' keeps the lower index on equal values. */
static void route_one(int d, int E, int k, const double *xt, const uint16_t *Wg,
                      const double *bias, double *l, int32_t *sel, double *w,
                      double *gap, unsigned char *taken)
{
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        const uint16_t *row = Wg + (size_t)e * d;
        for (int i = 0; i < d; ++i) acc += xt[i] * bf16_bits_to_double(row[i]);
        if (bias) acc += bias[e];
        l[e] = acc;
        taken[e] = 0;
    }
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
        sel[j] = best;
        taken[best] = 1;
    }
    if (gap) {
        if (k < E) {
            int next = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (next < 0 || l[e] > l[next])) next = e;
            *gap = l[sel[k - 1]] - l[next];
        } else {
            *gap = INFINITY;
        }
    }
    double m = l[sel[0]];
    double s = 0.0;
    for (int j = 0; j < k; ++j) {
        w[j] = exp(l[sel[j]] - m);
        s += w[j];
    }
    for (int j = 0; j < k; ++j) w[j] /= s;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* One gated expert on one token: y = W2 (act(W1 x) * (W3 x)) with
 * act = silu (act_mode 0, SwiGLU) or act = the logistic sigmoid (act_mode 1:
 * the "万亿 MoE" forward listing's h = a * sigmoid(g), whose gate g is the
 * W1 half and whose linear half a is the W3 half of its concatenated
 * up-projection).  W1, W3 are [dff, d] and W2 is [d, dff], row-major
 * (nn.Linear's [out, in]). */
static void expert_one(int d, int dff, const uint16_t *W1, const uint16_t *W3,
                       const uint16_t *W2, const double *xt, double *h, double *y, int act_mode)
{
    for (int f = 0; f < dff; ++f) {
        const uint16_t *r1 = W1 + (size_t)f * d;
        const uint16_t *r3 = W3 + (size_t)f * d;
        double a = 0.0, b = 0.0;
        for (int i = 0; i < d; ++i) a += bf16_bits_to_double(r1[i]) * xt[i];
        for (int i = 0; i < d; ++i) b += bf16_bits_to_double(r3[i]) * xt[i];
        if (act_mode == 1) h[f] = sigmoid(a) * b;
        else h[f] = silu(a) * b;
    }
    for (int o = 0; o < d; ++o) {
        const uint16_t *r2 = W2 + (size_t)o * dff;
        double acc = 0.0;
        for (int f = 0; f < dff; ++f) acc += bf16_bits_to_double(r2[f]) * h[f];
        y[o] = acc;
    }
}

/* The method's expert: SwiGLU. */
static void swiglu_one(int d, int dff, const uint16_t *W1, const uint16_t *W3,
                       const uint16_t *W2, const double *xt, double *h, double *y)
{
    expert_one(d, dff, W1, W3, W2, xt, h, y, 0);
}

/* Gate weights of the selected experts sel[0..k) for the routing variants
 * (w_mode 0, the softmax over the selected logits, is computed by route_one
 * or the forced-set code):
 *   w_mode 1: softmax over all E logits; the selected experts keep their
 *             probabilities, not renormalised ("Mixtral 8x7B模型架构解析"
 *             (bjdmk.com.cn), Router.forward: softmax, then top-k of the
 *             probabilities)
 *   w_mode 2: the logistic sigmoid of each selected logit ("万亿 MoE"
 *             (m.xxqk.cn) forward listing: w = 1 / (1 + exp(-logit)))
 *   w_mode 3: entropy-controlled k ("Mixtral 8x7B模型架构解析", routing-
 *             strategy section, entropy_aware_routing): p = softmax(l / tau)
 *             over all E logits with tau = 0.1, its entropy
 *             H = -sum_e p_e ln p_e (a term with p_e = 0 counts 0); the token
 *             keeps k experts when H > 0.8 and k - 1 otherwise (the listing's
 *             3 and 2 for k = 3), weighted by their p, not renormalised.
 * *k_used gets the number of slots the token uses (k except in w_mode 3);
 * slots from *k_used on are unused. */
#define ENTROPY_TAU 0.1
#define ENTROPY_THRESHOLD 0.8

static void variant_weights(int E, int k, const double *l, const int32_t *sel, int w_mode,
                            double *w, int *k_used)
{
    *k_used = k;
    if (w_mode == 3) {
        double m = l[0], s = 0.0, H = 0.0;
        for (int e = 1; e < E; ++e)
            if (l[e] > m) m = l[e];
        for (int e = 0; e < E; ++e) s += exp((l[e] - m) / ENTROPY_TAU);
        for (int e = 0; e < E; ++e) {
            double pe = exp((l[e] - m) / ENTROPY_TAU) / s;
            if (pe > 0.0) H -= pe * log(pe);
        }
        *k_used = H > ENTROPY_THRESHOLD ? k : k - 1;
        for (int j = 0; j < k; ++j) w[j] = exp((l[sel[j]] - m) / ENTROPY_TAU) / s;
        return;
    }
    if (w_mode == 1) {
        double m = l[0], s = 0.0;
        for (int e = 1; e < E; ++e)
            if (l[e] > m) m = l[e];
        for (int e = 0; e < E; ++e) s += exp(l[e] - m);
        for (int j = 0; j < k; ++j) w[j] = exp(l[sel[j]] - m) / s;
    } else if (w_mode == 2) {
        for (int j = 0; j < k; ++j) w[j] = sigmoid(l[sel[j]]);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Routing for all T tokens.
 *   x [T,d], Wg [E,d] : bf16 bits;  bias [E] or NULL (added to the logits
 *   before both the selection and the softmax)
 *   idx [T,k] int32, w [T,k], gap [T] (may be NULL), logits [T,E] (may be
 *   NULL), counts [E] (may be NULL): number of (token, slot) pairs per expert.
 * Returns 0, or -1 on bad arguments. */
int oracle_route_v(int T, int d, int E, int k, const uint16_t *x, const uint16_t *Wg,
                   const double *bias, int w_mode, int32_t *idx, double *w, double *gap,
                   double *logits, int64_t *counts);

int oracle_route(int T, int d, int E, int k, const uint16_t *x, const uint16_t *Wg,
                 const double *bias, int32_t *idx, double *w, double *gap,
                 double *logits, int64_t *counts)
{
    return oracle_route_v(T, d, E, k, x, Wg, bias, 0, idx, w, gap, logits, counts);
}

/* oracle_route with the gate weights of routing variant w_mode (0, 1, 2 as
 * in variant_weights; the selected set and the gap do not depend on it:
 * the softmax over all logits and the sigmoid keep the logits' order). */
int oracle_route_v(int T, int d, int E, int k, const uint16_t *x, const uint16_t *Wg,
                   const double *bias, int w_mode, int32_t *idx, double *w, double *gap,
                   double *logits, int64_t *counts)
{
    if (w_mode < 0 || w_mode > 3 || (w_mode == 3 && k < 2)) return -1;
    if (T < 0 || d < 1 || E < 1 || k < 1 || k > E || !x || !Wg || !idx || !w) return -1;
    int err = 0;
#pragma omp parallel
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        if (!xt || !l || !taken) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(static)
            for (int t = 0; t < T; ++t) {
                for (int i = 0; i < d; ++i) xt[i] = bf16_bits_to_double(x[(size_t)t * d + i]);
                route_one(d, E, k, xt, Wg, bias, l, idx + (size_t)t * k, w + (size_t)t * k,
                          gap ? gap + t : NULL, taken);
                if (w_mode) {
                    int ku;
                    variant_weights(E, k, l, idx + (size_t)t * k, w_mode, w + (size_t)t * k, &ku);
                    for (int j = ku; j < k; ++j) {  /* unused slots */
                        idx[(size_t)t * k + j] = -1;
                        w[(size_t)t * k + j] = 0.0;
                    }
                }
                if (logits) memcpy(logits + (size_t)t * E, l, sizeof(double) * (size_t)E);
            }
        }
        free(xt);
        free(l);
        free(taken);
    }
    if (err) return -1;
    if (counts) {
        for (int e = 0; e < E; ++e) counts[e] = 0;
        for (size_t s = 0; s < (size_t)T * k; ++s)
            if (idx[s] >= 0) counts[idx[s]] += 1;
    }
    return 0;
}

/* Layer output for n selected tokens.
 *   tokens [n] : token indices into x (NULL means tokens 0..n-1)
 *   x [T,d], Wg [E,d], W1/W3 [E,dff,d], W2 [E,d,dff] : bf16 bits
 *   bias [E] or NULL
 *   dffs > 0 with Ws1/Ws3 [dffs,d], Ws2 [d,dffs]: shared expert, added with
 *   weight 1; dffs == 0 means no shared expert
 *   forced [n,k] or NULL: when given, token r uses experts forced[r,*] in that
 *   order instead of its own top-k; the weights are still the softmax over
 *   those experts' logits.  This re-evaluates a token with another set
 *   (used where the k-th and (k+1)-th logits nearly tie).
 *   out [n,d] double.
 * Returns 0, or -1 on bad arguments. */
int oracle_forward_v(int n, const int32_t *tokens, int T, int d, int E, int dff, int k,
                     const uint16_t *x, const uint16_t *Wg, const double *bias,
                     const uint16_t *W1, const uint16_t *W3, const uint16_t *W2,
                     int dffs, const uint16_t *Ws1, const uint16_t *Ws3, const uint16_t *Ws2,
                     const int32_t *forced, int w_mode, int act_mode, long long cap,
                     const int32_t *route_all, double *out);

int oracle_forward(int n, const int32_t *tokens, int T, int d, int E, int dff, int k,
                   const uint16_t *x, const uint16_t *Wg, const double *bias,
                   const uint16_t *W1, const uint16_t *W3, const uint16_t *W2,
                   int dffs, const uint16_t *Ws1, const uint16_t *Ws3, const uint16_t *Ws2,
                   const int32_t *forced, double *out)
{
    return oracle_forward_v(n, tokens, T, d, E, dff, k, x, Wg, bias, W1, W3, W2, dffs, Ws1, Ws3,
                            Ws2, forced, 0, 0, -1, NULL, out);
}

/* oracle_forward for the variants the pages describe besides the method:
 *   w_mode, act_mode: gate weights and expert activation (variant_weights,
 *     expert_one); with forced experts the weights are those of the forced
 *     set under the same rule
 *   cap >= 0: expert capacity ("Mistral 8x7B SMoE" (jsqmd.com) sec. 2.4,
 *     capacity factor): of the (token, slot) pairs routed to an expert only
 *     the first cap in token order are computed, the others add nothing to
 *     their token's output (the other slots keep their weights).  The ranks
 *     need the routing of all T tokens: route_all [T,k] (e.g. a routing with
 *     forced near ties), or NULL for the oracle's own top-k.  cap < 0:
 *     dropless. */
int oracle_forward_v(int n, const int32_t *tokens, int T, int d, int E, int dff, int k,
                     const uint16_t *x, const uint16_t *Wg, const double *bias,
                     const uint16_t *W1, const uint16_t *W3, const uint16_t *W2,
                     int dffs, const uint16_t *Ws1, const uint16_t *Ws3, const uint16_t *Ws2,
                     const int32_t *forced, int w_mode, int act_mode, long long cap,
                     const int32_t *route_all, double *out)
{
    if (n < 0 || T < 1 || d < 1 || E < 1 || dff < 1 || k < 1 || k > E) return -1;
    if (!x || !Wg || !W1 || !W3 || !W2 || !out) return -1;
    if (dffs < 0 || (dffs > 0 && (!Ws1 || !Ws3 || !Ws2))) return -1;
    if (w_mode < 0 || w_mode > 3 || act_mode < 0 || act_mode > 1) return -1;
    if (w_mode == 3 && (k < 2 || cap >= 0)) return -1;
    for (int r = 0; r < n; ++r) {
        int t = tokens ? tokens[r] : r;
        if (t < 0 || t >= T) return -1;
        /* In w_mode 3 a forced set may end in one unused slot (-1). */
        if (forced)
            for (int j = 0; j < k; ++j) {
                int e = forced[(size_t)r * k + j];
                int unused_ok = w_mode == 3 && j == k - 1 && e == -1;
                if ((e < 0 || e >= E) && !unused_ok) return -1;
            }
    }
    /* Capacity: which (token, slot) pairs are kept. */
    unsigned char *keep = NULL;
    if (cap >= 0) {
        int32_t *sel_all = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * k);
        double *w_all = (double *)malloc(sizeof(double) * (size_t)T * k);
        int64_t *cnt = (int64_t *)calloc((size_t)E, sizeof(int64_t));
        keep = (unsigned char *)malloc((size_t)T * k);
        int bad = !sel_all || !w_all || !cnt || !keep;
        if (!bad) {
            if (route_all) {
                for (size_t s = 0; s < (size_t)T * k; ++s) {
                    if (route_all[s] < 0 || route_all[s] >= E) bad = 1;
                    sel_all[s] = route_all[s];
                }
            } else if (oracle_route(T, d, E, k, x, Wg, bias, sel_all, w_all, NULL, NULL, NULL)) {
                bad = 1;
            }
        }
        if (!bad) {
            for (int t = 0; t < T; ++t)
                for (int j = 0; j < k; ++j) {
                    int e = sel_all[(size_t)t * k + j];
                    keep[(size_t)t * k + j] = cnt[e] < cap;
                    cnt[e] += 1;
                }
        }
        free(sel_all);
        free(w_all);
        free(cnt);
        if (bad) {
            free(keep);
            return -1;
        }
    }
    int hmax = dff > dffs ? dff : dffs;
    int err = 0;
#pragma omp parallel
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        double *h = (double *)malloc(sizeof(double) * (size_t)hmax);
        double *y = (double *)malloc(sizeof(double) * (size_t)d);
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        if (!xt || !l || !h || !y || !w || !sel || !taken) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int r = 0; r < n; ++r) {
                int t = tokens ? tokens[r] : r;
                for (int i = 0; i < d; ++i) xt[i] = bf16_bits_to_double(x[(size_t)t * d + i]);
                route_one(d, E, k, xt, Wg, bias, l, sel, w, NULL, taken);
                int ku = k;
                if (forced && w_mode == 3) {
                    /* the forced experts (an unused last slot allowed) with
                     * their tempered probabilities */
                    for (int j = 0; j < k; ++j) sel[j] = forced[(size_t)r * k + j];
                    int ku_own;
                    int32_t e_last = sel[k - 1];
                    if (e_last < 0) sel[k - 1] = sel[0];  /* any valid index; not used */
                    variant_weights(E, k, l, sel, w_mode, w, &ku_own);
                    ku = e_last < 0 ? k - 1 : k;
                } else {
                    if (forced) {
                        /* softmax over the forced experts' logits, in forced order */
                        double m = -INFINITY, s = 0.0;
                        for (int j = 0; j < k; ++j) {
                            sel[j] = forced[(size_t)r * k + j];
                            if (l[sel[j]] > m) m = l[sel[j]];
                        }
                        for (int j = 0; j < k; ++j) {
                            w[j] = exp(l[sel[j]] - m);
                            s += w[j];
                        }
                        for (int j = 0; j < k; ++j) w[j] /= s;
                    }
                    if (w_mode) variant_weights(E, k, l, sel, w_mode, w, &ku);
                }
                double *o = out + (size_t)r * d;
                for (int i = 0; i < d; ++i) o[i] = 0.0;
                for (int j = 0; j < ku; ++j) {
                    if (keep && !keep[(size_t)t * k + j]) continue;
                    int e = sel[j];
                    expert_one(d, dff, W1 + (size_t)e * dff * d, W3 + (size_t)e * dff * d,
                               W2 + (size_t)e * d * dff, xt, h, y, act_mode);
                    for (int i = 0; i < d; ++i) o[i] += w[j] * y[i];
                }
                if (dffs > 0) {
                    expert_one(d, dffs, Ws1, Ws3, Ws2, xt, h, y, act_mode);
                    for (int i = 0; i < d; ++i) o[i] += y[i];
                }
            }
        }
        free(xt);
        free(l);
        free(h);
        free(y);
        free(w);
        free(sel);
        free(taken);
    }
    free(keep);
    return err ? -1 : 0;
}

/* ---------------------------------------------------------------- FP8 experts
 * Expert weights stored as 8-bit floating point codes with one scale per
 * weight row ("Mistral 8x7B SMoE" (jsqmd.com) deployment section:
 * quantised experts, router kept in higher precision): the weight is
 * W[e, r, i] = scale[e, r] * e4m3(code[e, r, i]).  e4m3 is the OCP 8-bit
 * format E4M3 (no infinities): sign bit 7, exponent bits 6..3 with bias 7,
 * mantissa bits 2..0; exponent 0 holds the subnormals 2^-6 * m/8; exponent
 * 15 with mantissa 7 is NaN; the largest finite value is 448. */
static double e4m3_to_double(uint8_t b)
{
    const int sgn = b >> 7, e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7) return NAN;
    const double v = e == 0 ? ldexp((double)m, -9) : ldexp(8.0 + m, e - 10);
    return sgn ? -v : v;
}

double oracle_e4m3_to_double(int code) { return e4m3_to_double((uint8_t)code); }

/* One SwiGLU expert on one token with FP8 weights: rows of W1/W3 [dff, d]
 * and W2 [d, dff] as codes, s1/s3 [dff] and s2 [d] the row scales. */
static void swiglu_one_fp8(int d, int dff, const uint8_t *q1, const double *s1,
                           const uint8_t *q3, const double *s3, const uint8_t *q2,
                           const double *s2, const double *xt, double *h, double *y)
{
    for (int f = 0; f < dff; ++f) {
        const uint8_t *r1 = q1 + (size_t)f * d;
        const uint8_t *r3 = q3 + (size_t)f * d;
        double a = 0.0, b = 0.0;
        for (int i = 0; i < d; ++i) a += s1[f] * e4m3_to_double(r1[i]) * xt[i];
        for (int i = 0; i < d; ++i) b += s3[f] * e4m3_to_double(r3[i]) * xt[i];
        h[f] = silu(a) * b;
    }
    for (int o = 0; o < d; ++o) {
        const uint8_t *r2 = q2 + (size_t)o * dff;
        double acc = 0.0;
        for (int f = 0; f < dff; ++f) acc += s2[o] * e4m3_to_double(r2[f]) * h[f];
        y[o] = acc;
    }
}

/* Layer output for n selected tokens with FP8 experts: the method (router in
 * bf16, top-k, softmax over the selected, weighted sum in slot order) with
 * W1/W3/W2 given as codes q1/q3 [E,dff,d], q2 [E,d,dff] and row scales
 * s1/s3 [E,dff], s2 [E,d].  tokens and forced as in oracle_forward. */
int oracle_forward_fp8(int n, const int32_t *tokens, int T, int d, int E, int dff, int k,
                       const uint16_t *x, const uint16_t *Wg, const double *bias,
                       const uint8_t *q1, const double *s1, const uint8_t *q3, const double *s3,
                       const uint8_t *q2, const double *s2, const int32_t *forced, double *out)
{
    if (n < 0 || T < 1 || d < 1 || E < 1 || dff < 1 || k < 1 || k > E) return -1;
    if (!x || !Wg || !q1 || !s1 || !q3 || !s3 || !q2 || !s2 || !out) return -1;
    for (int r = 0; r < n; ++r) {
        int t = tokens ? tokens[r] : r;
        if (t < 0 || t >= T) return -1;
        if (forced)
            for (int j = 0; j < k; ++j)
                if (forced[(size_t)r * k + j] < 0 || forced[(size_t)r * k + j] >= E) return -1;
    }
    int err = 0;
#pragma omp parallel
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        double *h = (double *)malloc(sizeof(double) * (size_t)dff);
        double *y = (double *)malloc(sizeof(double) * (size_t)d);
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        if (!xt || !l || !h || !y || !w || !sel || !taken) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int r = 0; r < n; ++r) {
                int t = tokens ? tokens[r] : r;
                for (int i = 0; i < d; ++i) xt[i] = bf16_bits_to_double(x[(size_t)t * d + i]);
                route_one(d, E, k, xt, Wg, bias, l, sel, w, NULL, taken);
                if (forced) {
                    double m = -INFINITY, s = 0.0;
                    for (int j = 0; j < k; ++j) {
                        sel[j] = forced[(size_t)r * k + j];
                        if (l[sel[j]] > m) m = l[sel[j]];
                    }
                    for (int j = 0; j < k; ++j) {
                        w[j] = exp(l[sel[j]] - m);
                        s += w[j];
                    }
                    for (int j = 0; j < k; ++j) w[j] /= s;
                }
                double *o = out + (size_t)r * d;
                for (int i = 0; i < d; ++i) o[i] = 0.0;
                for (int j = 0; j < k; ++j) {
                    int e = sel[j];
                    swiglu_one_fp8(d, dff, q1 + (size_t)e * dff * d, s1 + (size_t)e * dff,
                                   q3 + (size_t)e * dff * d, s3 + (size_t)e * dff,
                                   q2 + (size_t)e * d * dff, s2 + (size_t)e * d, xt, h, y);
                    for (int i = 0; i < d; ++i) o[i] += w[j] * y[i];
                }
            }
        }
        free(xt);
        free(l);
        free(h);
        free(y);
        free(w);
        free(sel);
        free(taken);
    }
    return err ? -1 : 0;
}

/* One SwiGLU expert applied to n rows (no routing): out[r] = W2(silu(W1 x_r) * W3 x_r).
 * Used to check the expert FFN by itself. */
int oracle_swiglu(int n, int d, int dff, const uint16_t *x, const uint16_t *W1,
                  const uint16_t *W3, const uint16_t *W2, double *out)
{
    if (n < 0 || d < 1 || dff < 1 || !x || !W1 || !W3 || !W2 || !out) return -1;
    int err = 0;
#pragma omp parallel
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *h = (double *)malloc(sizeof(double) * (size_t)dff);
        if (!xt || !h) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int r = 0; r < n; ++r) {
                for (int i = 0; i < d; ++i) xt[i] = bf16_bits_to_double(x[(size_t)r * d + i]);
                swiglu_one(d, dff, W1, W3, W2, xt, h, out + (size_t)r * d);
            }
        }
        free(xt);
        free(h);
    }
    return err ? -1 : 0;
}

/* Expert parallelism: where every (rank, token, slot) pair lands when the E
 * experts are split over R ranks in contiguous blocks (owner of expert e:
 * e / (E/R)).  The pages place experts on GPUs by hand (jsqmd.com,
 * deployment section, problem 4) and fix no order inside a GPU; the order
 * below is the one this library defines, written out as nested loops:
 *   for each owner q, for each of its experts e in index order,
 *     for each sending rank r in order, for each token t in order, slot j:
 *       if idx_r[t, j] == e, the pair takes the owner's next receive row.
 * T_of[r]: tokens of rank r; idx_all: the R ranks' [T_r, k] arrays back to
 * back; pos_all out (same layout): the receive row of each pair (-1 if its
 * expert is outside [0, E)); offsets out [R][E/R + 1]: each owner's segment
 * starts. */
int oracle_ep_plan(int R, int E, int k, const int32_t *T_of, const int32_t *idx_all,
                   int32_t *pos_all, int32_t *offsets)
{
    if (R < 1 || E < R || E % R != 0 || k < 1 || !T_of || !pos_all || !offsets) return -1;
    const int El = E / R;
    size_t total = 0;
    for (int r = 0; r < R; ++r) {
        if (T_of[r] < 0) return -1;
        total += (size_t)T_of[r] * (size_t)k;
    }
    if (total > 0 && !idx_all) return -1;
    for (size_t i = 0; i < total; ++i) pos_all[i] = -1;
    for (int q = 0; q < R; ++q) {
        int32_t row = 0;
        int32_t *seg = offsets + (size_t)q * (size_t)(El + 1);
        seg[0] = 0;
        for (int e = q * El; e < (q + 1) * El; ++e) {
            size_t first = 0;  /* rank r's first pair in idx_all */
            for (int r = 0; r < R; ++r) {
                for (int t = 0; t < T_of[r]; ++t)
                    for (int j = 0; j < k; ++j) {
                        const size_t i = first + (size_t)t * (size_t)k + (size_t)j;
                        if (idx_all[i] == e) pos_all[i] = row++;
                    }
                first += (size_t)T_of[r] * (size_t)k;
            }
            seg[e - q * El + 1] = row;
        }
    }
    return 0;
}
