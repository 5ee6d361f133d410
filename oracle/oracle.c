/*
 * oracle.c -- plain fp64 CPU oracle for the LatentMoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library; the two are built separately and neither includes the other.
 *
 * What it computes (per token t, independently; no capacity, no dropping):
 *
 *   1. router logits   l_e = sum_i f_ti * Wr_ei + b_e,  e < N'_tot
 *        f = x (the gate stays at the full width d: "LatentMoE: How MoE Made
 *        a Key Paradigm Leap in 2026", section 2 closing note; Kimi K3 /
 *        Nemotron 3 Super article, "LatentMoE 具体怎么做", closing note), or
 *        f = bf16(z) when the latent-router reading is selected ("routing
 *        happens in the latent", the same sections' second bullet).  The
 *        latent is stored in bf16 before the gate reads it, so the top-K'
 *        decision (an integer decided by floating point) is taken on the same
 *        bf16 input on both sides; everything else stays in fp64.
 *   2. top-K' selection: the K' largest logits, ties to the lower expert id,
 *      slots ordered by (logit descending, id ascending).
 *   3. renormalised softmax over the selected logits
 *        w_k = exp(l_k - l_max) / sum_{j in S} exp(l_j - l_max).
 *   4. z = W_down x  (d -> latent; "How LatentMoE Works" step 1,
 *      Nemotron-3 article section 2.2, Figure 3b), or z = x when the layer
 *      has no projection (the standard MoE of Figure 3a).
 *   5. per selected expert e (experts compute in the latent space,
 *      "How LatentMoE Works" step 2):
 *        FFN expert:   u = W1_e z;  h = relu(u)^2, or h = silu(u[0:m]) * u[m:2m]
 *                      for the gated form; o = W2_e h
 *        zero expert:  o = 0          (MoE++ zero-computation experts,
 *        copy expert:  o = z           Nemotron-3 article section 3.2,
 *        const expert: o = v_c         Figure 1)
 *   6. yl = sum_k w_k o_k   (aggregate in the latent space, Figure 3b)
 *   7. y = x + W_up yl      (project back to d, "How LatentMoE Works"
 *      step 3; the residual add is the plain reading of a layer output),
 *      or y = x + yl without a projection.
 *   8. with a shared expert (hidden width ms > 0), which stays at the full
 *      width d ("LatentMoE: How MoE Made a Key Paradigm Leap in 2026",
 *      section 2 closing note): y += Ws2 act(Ws1 x), act as for the routed
 *      experts, added to the routed output, outside the routing.
 *
 * Everything is computed in double precision on the bf16 inputs widened
 * exactly; nothing is rounded in between.  OpenMP runs tokens in parallel;
 * each token's arithmetic is a straight sequential loop.
 *
 * The counting sort (dispatch) that groups (token, slot) pairs by expert is
 * the single-GPU stand-in for the expert-parallel all-to-all the pages
 * describe; its result is defined as a stable sort of the flat slot index
 * i = t*K' + k by expert id.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t d;             /* model width */
    int32_t latent;        /* latent width (== d when has_proj == 0) */
    int32_t m;             /* expert hidden width */
    int32_t n_ffn;         /* routed FFN experts N' */
    int32_t top_k;         /* K' */
    int32_t act;           /* 0 relu^2, 1 gated silu, 2 identity */
    int32_t n_zero, n_copy, n_const;
    int32_t has_proj;      /* 1: W_down / W_up present */
    int32_t latent_router; /* 1: gate reads z instead of x */
    int32_t shared_m;      /* hidden width of the shared expert at d (0: none) */
} oracle_cfg;

enum { ORACLE_ACT_RELU2 = 0, ORACLE_ACT_SWIGLU = 1, ORACLE_ACT_IDENTITY = 2 };

static double widen(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int n_total(const oracle_cfg *c) { return c->n_ffn + c->n_zero + c->n_copy + c->n_const; }

/* Round to the nearest bfloat16 (ties to even) through binary32, the way a
 * value accumulated in fp32 is stored as bf16.  Used for one input only: the
 * latent the latent-router reading feeds to the gate (see step 1). */
static double round_bf16(double v)
{
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    u &= 0xFFFF0000u;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* out[o] = sum_i W[o*in_dim + i] * v[i] */
static void matvec(int out_dim, int in_dim, const uint16_t *W, const double *v, double *out)
{
    for (int o = 0; o < out_dim; ++o) {
        const uint16_t *row = W + (size_t)o * in_dim;
        double s = 0.0;
        for (int i = 0; i < in_dim; ++i) s += widen(row[i]) * v[i];
        out[o] = s;
    }
}

/* Step 2 + 3 for one token: K' largest logits (ties to the lower id) and the
 * softmax over them.  Returns 0, or -1 on bad sizes. */
int oracle_route_token(int n_tot, int top_k, const double *logits, int32_t *idx, double *w)
{
    if (top_k < 1 || top_k > n_tot) return -1;
    char *taken = (char *)calloc((size_t)n_tot, 1);
    if (!taken) return -1;
    for (int k = 0; k < top_k; ++k) {
        int best = -1;
        for (int e = 0; e < n_tot; ++e) {
            if (taken[e]) continue;
            if (best < 0 || logits[e] > logits[best]) best = e; /* strict: keeps the lower id on ties */
        }
        taken[best] = 1;
        idx[k] = best;
    }
    free(taken);
    double lmax = logits[idx[0]];
    double denom = 0.0;
    for (int k = 0; k < top_k; ++k) denom += exp(logits[idx[k]] - lmax);
    for (int k = 0; k < top_k; ++k) w[k] = exp(logits[idx[k]] - lmax) / denom;
    return 0;
}

/* Routing for T tokens from given logits [T, n_tot]. */
int oracle_route(int T, int n_tot, int top_k, const double *logits, int32_t *idx, double *w)
{
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int t = 0; t < T; ++t)
        bad |= oracle_route_token(n_tot, top_k, logits + (size_t)t * n_tot, idx + (size_t)t * top_k,
                                  w + (size_t)t * top_k) != 0;
    return bad ? -1 : 0;
}

/* Counting sort of the flat slots i = t*K' + k by expert id (stable).
 * counts[e], offsets[e] (exclusive scan, offsets[n_tot] = T*K'), perm[p] = i
 * at sorted position p, inv[i] = p.  Returns -1 on an out-of-range id. */
int oracle_dispatch(int T, int top_k, int n_tot, const int32_t *idx, int32_t *counts, int32_t *offsets,
                    int32_t *perm, int32_t *inv)
{
    const long n = (long)T * top_k;
    for (int e = 0; e < n_tot; ++e) counts[e] = 0;
    for (long i = 0; i < n; ++i) {
        if (idx[i] < 0 || idx[i] >= n_tot) return -1;
        counts[idx[i]] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < n_tot; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_tot > 0 ? n_tot : 1));
    if (!cursor) return -1;
    for (int e = 0; e < n_tot; ++e) cursor[e] = offsets[e];
    for (long i = 0; i < n; ++i) {
        int p = cursor[idx[i]]++;
        perm[p] = (int32_t)i;
        inv[i] = p;
    }
    free(cursor);
    return 0;
}

/* One FFN expert in the latent space: o = W2_e act(W1_e z). */
static void ffn_expert(const oracle_cfg *c, const uint16_t *w1e, const uint16_t *w2e, const double *z,
                       double *u, double *h, double *o)
{
    const int L = c->latent, m = c->m;
    const int up_rows = c->act == ORACLE_ACT_SWIGLU ? 2 * m : m;
    matvec(up_rows, L, w1e, z, u);
    for (int j = 0; j < m; ++j) {
        if (c->act == ORACLE_ACT_RELU2) {
            double r = u[j] > 0.0 ? u[j] : 0.0;
            h[j] = r * r;
        } else if (c->act == ORACLE_ACT_SWIGLU) {
            double a = u[j];
            h[j] = a / (1.0 + exp(-a)) * u[m + j];
        } else {
            h[j] = u[j];
        }
    }
    matvec(L, m, w2e, h, o);
}

/*
 * Whole-layer forward for T tokens.
 *   x [T,d] bf16; w_router [n_tot, fdim] bf16 (fdim = d, or latent with the
 *   latent router); bias [n_tot] fp32 or NULL; w_down [latent,d]; w_up
 *   [d,latent]; w1 [n_ffn, g*m, latent]; w2 [n_ffn, latent, m]; const_vecs
 *   [n_const, latent]; w_shared1 [g*shared_m, d], w_shared2 [d, shared_m]
 *   (NULL without a shared expert)   (all bf16 bit patterns).
 *   idx_in: if non-NULL, [T,K'] routes to use instead of the router's own
 *   choice (the weights are still the renormalised softmax of the router's
 *   logits at those ids, in the given slot order).
 * Outputs (fp64 unless stated; any of the optional ones may be NULL):
 *   y [T,d]; idx_out [T,K'] int32; w_out [T,K']; z_out [T,latent];
 *   yl_out [T,latent]; logits_out [T,n_tot].
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int oracle_forward(const oracle_cfg *c, int T, const uint16_t *x, const uint16_t *w_router, const float *bias,
                   const uint16_t *w_down, const uint16_t *w_up, const uint16_t *w1, const uint16_t *w2,
                   const uint16_t *const_vecs, const uint16_t *w_shared1, const uint16_t *w_shared2,
                   const int32_t *idx_in, double *y, int32_t *idx_out, double *w_out, double *z_out, double *yl_out,
                   double *logits_out)
{
    const int d = c->d, L = c->latent, m = c->m, K = c->top_k, Nt = n_total(c);
    if (T < 0 || K < 1 || K > Nt || d < 1 || L < 1 || m < 1) return -1;
    if (!c->has_proj && L != d) return -1;
    if (c->shared_m < 0 || (c->shared_m > 0 && (!w_shared1 || !w_shared2))) return -1;
    const int ms = c->shared_m;
    const int s_rows = c->act == ORACLE_ACT_SWIGLU ? 2 * ms : ms;
    const int fdim = c->latent_router ? L : d;
    const int up_rows = c->act == ORACLE_ACT_SWIGLU ? 2 * m : m;
    int bad = 0;

#pragma omp parallel reduction(| : bad)
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *z = (double *)malloc(sizeof(double) * (size_t)L);
        double *zr = (double *)malloc(sizeof(double) * (size_t)L);
        double *lg = (double *)malloc(sizeof(double) * (size_t)Nt);
        double *u = (double *)malloc(sizeof(double) * (size_t)up_rows);
        double *h = (double *)malloc(sizeof(double) * (size_t)m);
        double *o = (double *)malloc(sizeof(double) * (size_t)L);
        double *yl = (double *)malloc(sizeof(double) * (size_t)L);
        double *up = (double *)malloc(sizeof(double) * (size_t)d);
        double *w = (double *)malloc(sizeof(double) * (size_t)K);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
        double *su = (double *)malloc(sizeof(double) * (size_t)(s_rows > 0 ? s_rows : 1));
        double *sh = (double *)malloc(sizeof(double) * (size_t)(ms > 0 ? ms : 1));
        double *so = (double *)malloc(sizeof(double) * (size_t)d);
        if (!xt || !z || !zr || !lg || !u || !h || !o || !yl || !up || !w || !sel || !su || !sh || !so) bad = 1;

#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < T; ++t) {
            if (bad) continue;
            for (int i = 0; i < d; ++i) xt[i] = widen(x[(size_t)t * d + i]);
            /* step 4: latent projection (identity for the standard MoE) */
            if (c->has_proj) matvec(L, d, w_down, xt, z);
            else memcpy(z, xt, sizeof(double) * (size_t)d);
            /* step 1: router logits at the full width (or on the bf16 latent) */
            if (c->latent_router) {
                for (int j = 0; j < L; ++j) zr[j] = round_bf16(z[j]);
                matvec(Nt, fdim, w_router, zr, lg);
            } else {
                matvec(Nt, fdim, w_router, xt, lg);
            }
            if (bias)
                for (int e = 0; e < Nt; ++e) lg[e] += (double)bias[e];
            /* steps 2-3 */
            if (idx_in) {
                double lmax = -INFINITY, denom = 0.0;
                for (int k = 0; k < K; ++k) {
                    sel[k] = idx_in[(size_t)t * K + k];
                    if (sel[k] < 0 || sel[k] >= Nt) bad = 1;
                }
                if (bad) continue;
                for (int k = 0; k < K; ++k) lmax = lg[sel[k]] > lmax ? lg[sel[k]] : lmax;
                for (int k = 0; k < K; ++k) denom += exp(lg[sel[k]] - lmax);
                for (int k = 0; k < K; ++k) w[k] = exp(lg[sel[k]] - lmax) / denom;
            } else if (oracle_route_token(Nt, K, lg, sel, w) != 0) {
                bad = 1;
                continue;
            }
            /* steps 5-6: experts in the latent space, aggregated there */
            for (int j = 0; j < L; ++j) yl[j] = 0.0;
            for (int k = 0; k < K; ++k) {
                const int e = sel[k];
                if (e < c->n_ffn) {
                    ffn_expert(c, w1 + (size_t)e * up_rows * L, w2 + (size_t)e * L * m, z, u, h, o);
                } else if (e < c->n_ffn + c->n_zero) {
                    for (int j = 0; j < L; ++j) o[j] = 0.0;
                } else if (e < c->n_ffn + c->n_zero + c->n_copy) {
                    for (int j = 0; j < L; ++j) o[j] = z[j];
                } else {
                    const int cc = e - c->n_ffn - c->n_zero - c->n_copy;
                    for (int j = 0; j < L; ++j) o[j] = widen(const_vecs[(size_t)cc * L + j]);
                }
                for (int j = 0; j < L; ++j) yl[j] += w[k] * o[j];
            }
            /* step 7: back to d, residual add */
            if (c->has_proj) matvec(d, L, w_up, yl, up);
            else memcpy(up, yl, sizeof(double) * (size_t)d);
            for (int i = 0; i < d; ++i) y[(size_t)t * d + i] = xt[i] + up[i];
            /* step 8: the shared expert at the full width, on x */
            if (ms > 0) {
                matvec(s_rows, d, w_shared1, xt, su);
                for (int j = 0; j < ms; ++j) {
                    if (c->act == ORACLE_ACT_RELU2) {
                        double r = su[j] > 0.0 ? su[j] : 0.0;
                        sh[j] = r * r;
                    } else if (c->act == ORACLE_ACT_SWIGLU) {
                        double a = su[j];
                        sh[j] = a / (1.0 + exp(-a)) * su[ms + j];
                    } else {
                        sh[j] = su[j];
                    }
                }
                matvec(d, ms, w_shared2, sh, so);
                for (int i = 0; i < d; ++i) y[(size_t)t * d + i] += so[i];
            }

            if (idx_out)
                for (int k = 0; k < K; ++k) idx_out[(size_t)t * K + k] = sel[k];
            if (w_out)
                for (int k = 0; k < K; ++k) w_out[(size_t)t * K + k] = w[k];
            if (z_out) memcpy(z_out + (size_t)t * L, z, sizeof(double) * (size_t)L);
            if (yl_out) memcpy(yl_out + (size_t)t * L, yl, sizeof(double) * (size_t)L);
            if (logits_out) memcpy(logits_out + (size_t)t * Nt, lg, sizeof(double) * (size_t)Nt);
        }
        free(su); free(sh); free(so);
        free(xt); free(z); free(zr); free(lg); free(u); free(h); free(o); free(yl); free(up); free(w); free(sel);
    }
    return bad ? -1 : 0;
}

/* Threads the OpenMP runtime will use (reported with the CPU baseline). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
