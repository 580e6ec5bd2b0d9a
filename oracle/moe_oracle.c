/*
 * moe_oracle.c -- float64 CPU oracle for the sparse Mixture-of-Experts block.
 *
 * TEST INFRASTRUCTURE ONLY.  The parity tests, the smoke check and the
 * benchmark's CPU-baseline leg are the only callers.  The CUDA library never
 * links, loads or calls this file, and this file includes nothing of it: the
 * two implementations share no code, header, table or constant.
 *
 * What it computes, and where the pages say so
 * (page 1 = "qwen36/neural-network.html", the router paragraphs;
 *  page 3 = ".../qwen3-8-max/architecture/", section "La configuration, en
 *  entier", the Mixture-of-Experts keys of config.json;
 *  page 5 = "hyper.ai/fr/stories/...", the Qwen3-Next story, shared expert):
 *
 *   router   l_e = x . W_r[e] (+ b_e)          page 1: a small linear network
 *                                               maps the token to E scores
 *   softmax  p_e = exp(l_e - max l) / sum      page 1: a probability for each
 *                                               expert, softmax top-k
 *   top-k    the k largest p (ties -> lower     page 1; page 3 keys
 *            expert index)                      num_experts / num_experts_per_tok
 *   renorm   w_e = p_e / sum_{kept} p           the block's definition asks for
 *                                               the kept weights renormalised
 *   expert   E_e(x) = W_down[e] (SiLU(W_gate[e] x) * (W_up[e] x))
 *                                               page 3 key hidden_act = silu;
 *                                               moe_intermediate_size = I
 *   shared   S(x), same SwiGLU shape with I_s,  page 1 (one "shared" expert is
 *            always on, weight 1                always active); page 3 key
 *                                               shared_expert_intermediate_size;
 *                                               page 5 (the shared expert treats
 *                                               every input)
 *   output   y = sum_{e kept} w_e E_e(x) + S(x)
 *
 * The block's neighbours (oracle_block_forward; both optional):
 *   norm     x <- x / sqrt(mean_j x_j^2 + eps)   page 5: Qwen3-Next uses a
 *            * (1 + gamma), rounded to the        "zero-centred" RMSNorm whose
 *            activation type (the block's input)  parameters start at zero, so
 *                                                 the applied scale is 1 + gamma;
 *                                                 page 3 key rms_norm_eps = 1e-6
 *   gate     S(x) weighted by sigmoid(x . w_sg)   not on the pages: an option
 *                                                 some implementations carry;
 *                                                 off (weight 1) by default
 *
 * Every function below follows that definition literally, per token, in
 * float64, reading the caller's low-precision values (fp32, bf16 or E4M3 with
 * fp32 block scales) and converting each element as it is used.  There is no
 * blocking, fusion or reordering beyond a plain loop nest.
 *
 * Weight layout (the usual linear-layer convention, out x in, row-major):
 *   W_r [E, d];  W_gate, W_up [E, I, d];  W_down [E, d, I];
 *   shared: [I_s, d], [I_s, d], [d, I_s].
 * E4M3 weights carry one fp32 scale per 128x128 block of each matrix, indexed
 * [row / 128][col / 128]; the weight value is decode(q) * scale.  The packed
 * scale buffer concatenates: gate [E][I/128][d/128], up (same), down
 * [E][d/128][I/128], shared gate [I_s/128][d/128], shared up (same), shared
 * down [d/128][I_s/128].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Element codes used by this file's entry points. */
enum { ODT_F32 = 0, ODT_BF16 = 1, ODT_E4M3 = 2 };

/* bf16 is the upper half of an IEEE binary32. */
static double dec_bf16(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* E4M3 (the "fn" variant: no infinities): 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); the single
 * pattern S.1111.111 is NaN; the largest finite value is 448. */
static double dec_e4m3(uint8_t q)
{
    int s = q >> 7, e = (q >> 3) & 15, m = q & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

static size_t dt_size(int dt) { return dt == ODT_F32 ? 4 : dt == ODT_BF16 ? 2 : 1; }

static double elem(const void *p, int dt, int64_t i)
{
    if (dt == ODT_F32) return (double)((const float *)p)[i];
    if (dt == ODT_BF16) return dec_bf16(((const uint16_t *)p)[i]);
    return dec_e4m3(((const uint8_t *)p)[i]);
}

/* Element (r, c) of a rows x cols weight matrix; E4M3 values are multiplied by
 * the fp32 scale of their 128x128 block. */
static double welem(const void *w, int dt, const float *s, int64_t cols, int64_t r, int64_t c)
{
    double v = elem(w, dt, r * cols + c);
    if (dt == ODT_E4M3) v *= (double)s[(r / 128) * ((cols + 127) / 128) + c / 128];
    return v;
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* v rounded to the nearest value of the activation type (ties to even):
 * bf16 keeps 8 significant bits (quantum 2^(e-8) for v = f 2^e, 1/2 <= |f| < 1;
 * 2^-133 below the normal range); fp32 by the C conversion. */
static double round_act(double v, int dt)
{
    if (dt == ODT_F32) return (double)(float)v;
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    frexp(v, &e);
    int qe = e - 8 < -133 ? -133 : e - 8;
    double q = ldexp(1.0, qe);
    return nearbyint(v / q) * q;
}

/* Zero-centred RMSNorm of one row of d values (read from x at row t):
 * out_j = x_j / sqrt(mean x^2 + eps) * (1 + gamma_j), float64. */
static void rmsnorm_row(int d, const void *x, int act_dt, int64_t t, const void *gamma, double eps, double *out)
{
    double ss = 0.0;
    for (int j = 0; j < d; ++j) {
        double v = elem(x, act_dt, t * d + j);
        ss += v * v;
    }
    double r = 1.0 / sqrt(ss / d + eps);
    for (int j = 0; j < d; ++j) out[j] = elem(x, act_dt, t * d + j) * r * (1.0 + elem(gamma, act_dt, j));
}

/* Zero-centred RMSNorm of T rows, float64 (not rounded). */
int oracle_rmsnorm(int64_t T, int d, int act_dt, const void *x, const void *gamma, double eps, double *out)
{
    if (T < 0 || d <= 0 || !x || !gamma || !(eps >= 0.0)) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) rmsnorm_row(d, x, act_dt, t, gamma, eps, out + t * d);
    return 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int oracle_e4m3_decode(const uint8_t *q, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = dec_e4m3(q[i]);
    return 0;
}

/* Probabilities, top-k set and renormalised weights of one token, from its
 * logits.  Selection is repeated arg-max with a strict '>' so that equal
 * probabilities go to the lower expert index; the k ids come out in
 * descending probability. */
static void route_token(int E, int k, const double *logit, double *p, int32_t *ids, double *w,
                        const int32_t *forced)
{
    double mx = logit[0], z = 0.0, sum = 0.0;
    for (int e = 1; e < E; ++e)
        if (logit[e] > mx) mx = logit[e];
    for (int e = 0; e < E; ++e) {
        p[e] = exp(logit[e] - mx);
        z += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= z;
    if (forced) {
        for (int s = 0; s < k; ++s) ids[s] = forced[s];
    } else {
        char *taken = (char *)calloc((size_t)E, 1);
        for (int s = 0; s < k; ++s) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || p[e] > p[best])) best = e;
            taken[best] = 1;
            ids[s] = best;
        }
        free(taken);
    }
    for (int s = 0; s < k; ++s) sum += p[ids[s]];
    for (int s = 0; s < k; ++s) w[s] = p[ids[s]] / sum;
}

/* Router stage: logits, full softmax, top-k, renormalisation for T tokens.
 * probs [T,E] may be NULL. */
int oracle_router(int64_t T, int d, int E, int k, int act_dt, const void *x, const void *w_r,
                  const float *bias, double *probs, int32_t *topk_ids, double *topk_w)
{
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E) return 1;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = 0; t < T; ++t) {
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        double *p = (double *)malloc(sizeof(double) * (size_t)E);
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j)
                acc += elem(x, act_dt, t * d + j) * elem(w_r, act_dt, (int64_t)e * d + j);
            l[e] = acc + (bias ? (double)bias[e] : 0.0);
        }
        route_token(E, k, l, p, topk_ids + t * k, topk_w + t * k, NULL);
        if (probs) memcpy(probs + t * E, p, sizeof(double) * (size_t)E);
        free(l);
        free(p);
    }
    return 0;
}

/* Dispatch stage: a stable counting sort of the T*k (token, slot) pairs by
 * expert.  Group e holds the rows offs[e] .. offs[e+1]-1 in (token, slot)
 * order; group E (the shared expert) holds every token, in order, at rows
 * T*k .. T*k+T-1.  pos[t*k+j] is the row of pair (t, j); row_slot of a shared
 * row is k. */
int oracle_permute(int64_t T, int E, int k, const int32_t *topk_ids, int32_t *offs,
                   int32_t *row_tok, int32_t *row_slot, int32_t *pos)
{
    int64_t *cnt = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *cur = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    for (int64_t i = 0; i < T * k; ++i) {
        if (topk_ids[i] < 0 || topk_ids[i] >= E) {
            free(cnt);
            free(cur);
            return 1;
        }
        cnt[topk_ids[i]]++;
    }
    int64_t run = 0;
    for (int e = 0; e < E; ++e) {
        offs[e] = (int32_t)run;
        cur[e] = run;
        run += cnt[e];
    }
    offs[E] = (int32_t)(T * k);
    offs[E + 1] = (int32_t)(T * k + T);
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = topk_ids[t * k + j];
            int64_t r = cur[e]++;
            row_tok[r] = (int32_t)t;
            row_slot[r] = j;
            pos[t * k + j] = (int32_t)r;
        }
    for (int64_t t = 0; t < T; ++t) {
        row_tok[T * k + t] = (int32_t)t;
        row_slot[T * k + t] = k;
    }
    free(cnt);
    free(cur);
    return 0;
}

/* One SwiGLU expert on one activation row x (length d, already float64):
 * out[c] = sum_i W_down[c,i] * SiLU(sum_j W_gate[i,j] x_j) * (sum_j W_up[i,j] x_j). */
static void expert_row(int d, int I, const double *x, int w_dt, const void *wg, const void *wu,
                       const void *wd, const float *sg, const float *su, const float *sd,
                       double *h, double *out)
{
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int j = 0; j < d; ++j) {
            g += welem(wg, w_dt, sg, d, i, j) * x[j];
            u += welem(wu, w_dt, su, d, i, j) * x[j];
        }
        h[i] = silu(g) * u;
    }
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += welem(wd, w_dt, sd, I, c, i) * h[i];
        out[c] = acc;
    }
}

/* One expert applied to n rows (row stride x_stride elements) -> out [n, d]. */
int oracle_swiglu_expert(int64_t n, int d, int I, int act_dt, const void *xs, int64_t x_stride,
                         int w_dt, const void *wg, const void *wu, const void *wd, const float *sg,
                         const float *su, const float *sd, double *out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
        double *x = (double *)malloc(sizeof(double) * (size_t)d);
        double *h = (double *)malloc(sizeof(double) * (size_t)(I > 0 ? I : 1));
        for (int j = 0; j < d; ++j) x[j] = elem(xs, act_dt, r * x_stride + j);
        expert_row(d, I, x, w_dt, wg, wu, wd, sg, su, sd, h, out + r * d);
        free(x);
        free(h);
    }
    return 0;
}

/* Offsets (in floats) of the six parts of the packed E4M3 scale buffer. */
static void scale_parts(int d, int E, int I, int I_s, int64_t off[6])
{
    int64_t gd = (d + 127) / 128, gi = (I + 127) / 128, gs = (I_s + 127) / 128;
    off[0] = 0;
    off[1] = off[0] + (int64_t)E * gi * gd;
    off[2] = off[1] + (int64_t)E * gi * gd;
    off[3] = off[2] + (int64_t)E * gd * gi;
    off[4] = off[3] + gs * gd;
    off[5] = off[4] + gs * gd;
}

/* Pointers to expert g's three matrices (g == E: the shared expert). */
static void expert_ptrs(int d, int E, int I, int I_s, int w_dt, const void *wg, const void *wu,
                        const void *wd, const void *s_wg, const void *s_wu, const void *s_wd,
                        const float *scales, int g, const void *p[3], const float *s[3], int *Ig)
{
    size_t b = dt_size(w_dt);
    int64_t off[6];
    scale_parts(d, E, I, I_s, off);
    int64_t gd = (d + 127) / 128, gi = (I + 127) / 128;
    if (g < E) {
        p[0] = (const char *)wg + (size_t)g * I * d * b;
        p[1] = (const char *)wu + (size_t)g * I * d * b;
        p[2] = (const char *)wd + (size_t)g * d * I * b;
        if (scales) {
            s[0] = scales + off[0] + (int64_t)g * gi * gd;
            s[1] = scales + off[1] + (int64_t)g * gi * gd;
            s[2] = scales + off[2] + (int64_t)g * gd * gi;
        }
        *Ig = I;
    } else {
        p[0] = s_wg;
        p[1] = s_wu;
        p[2] = s_wd;
        if (scales) {
            s[0] = scales + off[3];
            s[1] = scales + off[4];
            s[2] = scales + off[5];
        }
        *Ig = I_s;
    }
    if (!scales) s[0] = s[1] = s[2] = NULL;
}

/* The whole block, token by token.  force_ids [T,k] (may be NULL) replaces the
 * router's choice by a given set; the weights are still the renormalised
 * probabilities of that set.  probs [T,E] may be NULL. */
/* The block with its optional neighbours: norm_w (NULL: none) applies the
 * zero-centred RMSNorm to x first, its output rounded to the activation type;
 * gate_w (NULL: none) weights the shared expert by sigmoid(x . gate_w), x being
 * the (normalised) block input.  gate_out (may be NULL) receives that weight. */
int oracle_block_forward(int64_t T, int d, int E, int k, int I, int I_s, int act_dt, int w_dt,
                         const void *x, const void *norm_w, double eps, const void *gate_w,
                         const void *w_r, const float *bias, const void *wg, const void *wu,
                         const void *wd, const void *s_wg, const void *s_wu, const void *s_wd,
                         const float *scales, const int32_t *force_ids, double *y,
                         int32_t *topk_ids, double *topk_w, double *probs, double *gate_out)
{
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || I <= 0 || I_s < 0) return 1;
    if (norm_w && !(eps >= 0.0)) return 1;
    if (w_dt == ODT_E4M3 && !scales) return 1;
    if (force_ids)
        for (int64_t i = 0; i < T * k; ++i)
            if (force_ids[i] < 0 || force_ids[i] >= E) return 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) {
        int Imax = I > I_s ? I : I_s;
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        double *p = (double *)malloc(sizeof(double) * (size_t)E);
        double *h = (double *)malloc(sizeof(double) * (size_t)Imax);
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
        if (norm_w) {
            rmsnorm_row(d, x, act_dt, t, norm_w, eps, xt);
            for (int j = 0; j < d; ++j) xt[j] = round_act(xt[j], act_dt);
        } else {
            for (int j = 0; j < d; ++j) xt[j] = elem(x, act_dt, t * d + j);
        }
        double sgate = 1.0;
        if (gate_w) {
            double z = 0.0;
            for (int j = 0; j < d; ++j) z += xt[j] * elem(gate_w, act_dt, j);
            sgate = 1.0 / (1.0 + exp(-z));
        }
        if (gate_out) gate_out[t] = sgate;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += xt[j] * elem(w_r, act_dt, (int64_t)e * d + j);
            l[e] = acc + (bias ? (double)bias[e] : 0.0);
        }
        route_token(E, k, l, p, topk_ids + t * k, topk_w + t * k,
                    force_ids ? force_ids + t * k : NULL);
        if (probs) memcpy(probs + t * E, p, sizeof(double) * (size_t)E);
        for (int c = 0; c < d; ++c) y[t * d + c] = 0.0;
        for (int s = 0; s <= k; ++s) {
            int g = s < k ? topk_ids[t * k + s] : E;
            double wgt = s < k ? topk_w[t * k + s] : sgate;
            const void *pp[3];
            const float *ss[3];
            int Ig;
            if (g == E && I_s == 0) continue;
            expert_ptrs(d, E, I, I_s, w_dt, wg, wu, wd, s_wg, s_wu, s_wd, scales, g, pp, ss, &Ig);
            expert_row(d, Ig, xt, w_dt, pp[0], pp[1], pp[2], ss[0], ss[1], ss[2], h, o);
            for (int c = 0; c < d; ++c) y[t * d + c] += wgt * o[c];
        }
        free(xt);
        free(l);
        free(p);
        free(h);
        free(o);
    }
    return 0;
}

int oracle_moe_forward(int64_t T, int d, int E, int k, int I, int I_s, int act_dt, int w_dt,
                       const void *x, const void *w_r, const float *bias, const void *wg,
                       const void *wu, const void *wd, const void *s_wg, const void *s_wu,
                       const void *s_wd, const float *scales, const int32_t *force_ids, double *y,
                       int32_t *topk_ids, double *topk_w, double *probs)
{
    return oracle_block_forward(T, d, E, k, I, I_s, act_dt, w_dt, x, NULL, 0.0, NULL, w_r, bias, wg, wu,
                                wd, s_wg, s_wu, s_wd, scales, force_ids, y, topk_ids, topk_w, probs, NULL);
}

/* Expert stage on dispatched rows: group g's rows offs[g] .. offs[g+1]-1 of
 * x_perm [offs[E+1], d] go through expert g (g == E: the shared expert);
 * y_perm [offs[E+1], d] is unweighted. */
int oracle_expert_ffn(int d, int E, int I, int I_s, int act_dt, int w_dt, const void *x_perm,
                      const int32_t *offs, const void *wg, const void *wu, const void *wd,
                      const void *s_wg, const void *s_wu, const void *s_wd, const float *scales,
                      double *y_perm)
{
    size_t ab = dt_size(act_dt);
    for (int g = 0; g <= E; ++g) {
        int64_t r0 = offs[g], n = (int64_t)offs[g + 1] - offs[g];
        const void *pp[3];
        const float *ss[3];
        int Ig;
        if (n <= 0) continue;
        if (g == E && I_s == 0) {
            memset(y_perm + r0 * d, 0, sizeof(double) * (size_t)(n * d));
            continue;
        }
        expert_ptrs(d, E, I, I_s, w_dt, wg, wu, wd, s_wg, s_wu, s_wd, scales, g, pp, ss, &Ig);
        oracle_swiglu_expert(n, d, Ig, act_dt, (const char *)x_perm + (size_t)r0 * d * ab, d, w_dt,
                             pp[0], pp[1], pp[2], ss[0], ss[1], ss[2], y_perm + r0 * d);
    }
    return 0;
}

/* Combine stage: y[t] = sum_j topk_w[t,j] * y_perm[pos[t,j]] + y_perm[offs[E] + t]
 * (the last term only when the shared group is non-empty). */
int oracle_combine(int64_t T, int d, int E, int k, int act_dt, const void *y_perm,
                   const int32_t *pos, const float *topk_w, const int32_t *offs, double *y)
{
    int shared = offs[E + 1] > offs[E];
    for (int64_t t = 0; t < T; ++t)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += (double)topk_w[t * k + j] * elem(y_perm, act_dt, (int64_t)pos[t * k + j] * d + c);
            if (shared) acc += elem(y_perm, act_dt, ((int64_t)offs[E] + t) * d + c);
            y[t * d + c] = acc;
        }
    return 0;
}

/* Parameter bookkeeping of one block: three d x I matrices per routed expert,
 * three d x I_s for the shared expert, and the d x E router.  With active != 0
 * only the k routed experts a token uses are counted. */
int64_t oracle_param_count(int64_t d, int64_t E, int64_t k, int64_t I, int64_t I_s, int active)
{
    int64_t routed = active ? k : E;
    return routed * 3 * d * I + 3 * d * I_s + d * E;
}
