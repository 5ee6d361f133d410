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
 *        f = z (the fp64 latent of step 4) when the latent-router reading is
 *        selected ("routing happens in the latent", the same sections'
 *        second bullet).  The pages say nothing about the latent's precision,
 *        so the gate reads it exactly, like every other step here.
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
 *   9. with block-scaled expert weights (expert_fmt = MXFP8 or MXFP4), W1_e
 *      and W2_e are first encoded in that MX format (see the MX section
 *      below) and used at their encoded values; the inputs of both expert
 *      matrices (z, and the activation h) are stored in bf16 and then
 *      encoded in MXFP8 before the multiply.  With expert_fmt = NVFP4 the
 *      weights and both inputs are NVFP4-encoded instead (see the NVFP4
 *      section).  The router, the projections and the shared expert stay in
 *      bf16.
 *
 * Everything is computed in double precision on the bf16 inputs widened
 * exactly; nothing is rounded in between except the MX encodings of step 9
 * (and the bf16 storage they start from).  OpenMP runs tokens in parallel;
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
    int32_t expert_fmt;    /* 0 bf16 expert weights, 1 MXFP8, 2 MXFP4, 3 NVFP4 */
} oracle_cfg;

enum { ORACLE_ACT_RELU2 = 0, ORACLE_ACT_SWIGLU = 1, ORACLE_ACT_IDENTITY = 2 };
enum { ORACLE_FMT_BF16 = 0, ORACLE_FMT_MXFP8 = 1, ORACLE_FMT_MXFP4 = 2, ORACLE_FMT_NVFP4 = 3 };

static double widen(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int n_total(const oracle_cfg *c) { return c->n_ffn + c->n_zero + c->n_copy + c->n_const; }

/* Round to the nearest bfloat16 (ties to even) through binary32, the way a
 * value accumulated in fp32 is stored as bf16.  Used only where the layer
 * stores a value before an integer decision is taken on it: the expert inputs
 * that are block-scale encoded (step 9). */
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

/* ------------------------------------------------------------------ MX block formats
 *
 * The pages name the formats only: Kimi K3 serves MXFP4 weights after
 * quantisation-aware training (the comparison table of "Two Teams, Two
 * Practices"), and Nemotron 3 Super trains in NVFP4 (the training note of
 * the outlook section).  Their definition is the Open Compute Project's
 * Microscaling (MX) specification, v1.0:
 *   - a block is 32 consecutive values along the reduction (K) axis;
 *   - the block shares one scale X = 2^s, stored as an E8M0 byte s + 127,
 *     with s = floor(log2(max_i |V_i|)) - emax, emax being the exponent of
 *     the element format's largest normal (8 for E4M3, 2 for E2M1); s is
 *     clamped to [-127, 127];
 *   - each element is V_i / X rounded to the nearest value of the element
 *     format (ties to the even mantissa) and saturated to its largest
 *     magnitude (448 for E4M3, 6 for E2M1);
 *   - an all-zero block gets s = -127 and zero elements.
 * E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; normals
 * (1 + m/8) 2^(e-7), subnormals m/8 2^-6; the code 0x7F / 0xFF is NaN and is
 * never produced.  E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit;
 * the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 * Codes are kept one per byte here (E2M1 in the low nibble, sign in bit 3).
 */
static int fmt_mbits(int e2m1) { return e2m1 ? 1 : 3; }
static int fmt_emin(int e2m1) { return e2m1 ? 0 : -6; }   /* exponent of the smallest normal */
static int fmt_emax(int e2m1) { return e2m1 ? 2 : 8; }    /* exponent of the largest normal */
static double fmt_max(int e2m1) { return e2m1 ? 6.0 : 448.0; }

/* Nearest element-format magnitude to a >= 0 (ties to even), saturated. */
static double round_elem(double a, int e2m1)
{
    const double maxv = fmt_max(e2m1);
    if (a >= maxv) return maxv;
    if (a == 0.0) return 0.0;
    int e;
    frexp(a, &e);
    e -= 1; /* a = f 2^e with f in [1, 2) */
    if (e < fmt_emin(e2m1)) e = fmt_emin(e2m1);
    const double quantum = ldexp(1.0, e - fmt_mbits(e2m1));
    const double r = rint(a / quantum) * quantum; /* the default rounding mode: to nearest, ties to even */
    return r > maxv ? maxv : r;
}

/* Code of an element-format magnitude r (exactly representable) and a sign. */
static uint8_t elem_code(double r, int neg, int e2m1)
{
    const int mb = fmt_mbits(e2m1), emin = fmt_emin(e2m1), bias = e2m1 ? 1 : 7;
    unsigned code;
    if (r < ldexp(1.0, emin)) {
        code = (unsigned)(r / ldexp(1.0, emin - mb)); /* subnormal: m quanta of 2^(emin - mbits) */
    } else {
        int e;
        frexp(r, &e);
        e -= 1;
        const unsigned mant = (unsigned)(r / ldexp(1.0, e - mb)) - (1u << mb);
        code = ((unsigned)(e + bias) << mb) | mant;
    }
    if (neg) code |= e2m1 ? 0x8u : 0x80u;
    return (uint8_t)code;
}

/* Value of an element code. */
static double elem_value(uint8_t code, int e2m1)
{
    const int mb = fmt_mbits(e2m1), bias = e2m1 ? 1 : 7;
    const unsigned sign = e2m1 ? (code >> 3) & 1u : (code >> 7) & 1u;
    const unsigned ebits = e2m1 ? (code >> 1) & 3u : (code >> 3) & 15u;
    const unsigned mant = code & ((1u << mb) - 1u);
    double v;
    if (ebits == 0) v = ldexp((double)mant, 1 - bias - mb);
    else v = ldexp((double)((1u << mb) + mant), (int)ebits - bias - mb);
    return sign ? -v : v;
}

/* Encode one block of 32 values. */
static void mx_block(const double *v, int e2m1, uint8_t *codes, uint8_t *scale)
{
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) amax = fabs(v[i]) > amax ? fabs(v[i]) : amax;
    int s = -127;
    if (amax > 0.0) {
        int e;
        frexp(amax, &e);
        s = (e - 1) - fmt_emax(e2m1);
        if (s < -127) s = -127;
        if (s > 127) s = 127;
    }
    *scale = (uint8_t)(s + 127);
    for (int i = 0; i < 32; ++i) {
        const double q = ldexp(v[i], -s); /* exact: a power-of-two scaling */
        codes[i] = elem_code(round_elem(fabs(q), e2m1), signbit(q) != 0, e2m1);
    }
}

/* MX encoding of a bf16 matrix [rows, K] (K a multiple of 32): codes
 * [rows, K] one per byte, scales [rows, K/32] as E8M0 bytes.  fmt is
 * ORACLE_FMT_MXFP8 (E4M3 elements) or ORACLE_FMT_MXFP4 (E2M1 elements).
 * Returns 0, or -1 on bad arguments. */
int oracle_mx_quantize(const uint16_t *w, int rows, int K, int fmt, uint8_t *codes, uint8_t *scales)
{
    if (rows < 0 || K < 32 || K % 32 != 0 || (fmt != ORACLE_FMT_MXFP8 && fmt != ORACLE_FMT_MXFP4)) return -1;
    const int e2m1 = fmt == ORACLE_FMT_MXFP4;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        double v[32];
        for (int b = 0; b < K / 32; ++b) {
            for (int i = 0; i < 32; ++i) v[i] = widen(w[(size_t)r * K + b * 32 + i]);
            mx_block(v, e2m1, codes + (size_t)r * K + b * 32, scales + (size_t)r * (K / 32) + b);
        }
    }
    return 0;
}

/* The values an MX encoding stands for: out = elem(code) * 2^(scale - 127). */
int oracle_mx_dequantize(const uint8_t *codes, const uint8_t *scales, int rows, int K, int fmt, double *out)
{
    if (rows < 0 || K < 32 || K % 32 != 0 || (fmt != ORACLE_FMT_MXFP8 && fmt != ORACLE_FMT_MXFP4)) return -1;
    const int e2m1 = fmt == ORACLE_FMT_MXFP4;
    for (size_t i = 0; i < (size_t)rows * K; ++i)
        out[i] = ldexp(elem_value(codes[i], e2m1), (int)scales[i / 32] - 127);
    return 0;
}

/* An activation vector as the expert GEMMs read it: stored in bf16, then MXFP8-encoded. */
static void mx_activation(const double *v, int n, double *out)
{
    uint8_t codes[32], scale;
    double blk[32];
    for (int b = 0; b < n / 32; ++b) {
        for (int i = 0; i < 32; ++i) blk[i] = round_bf16(v[b * 32 + i]);
        mx_block(blk, 0, codes, &scale);
        for (int i = 0; i < 32; ++i) out[b * 32 + i] = ldexp(elem_value(codes[i], 0), (int)scale - 127);
    }
}

/* ------------------------------------------------------------------ NVFP4
 *
 * The pages name NVFP4 only: Nemotron 3 Super trains in it (the training
 * note of the outlook section).  The definition used is NVIDIA's published
 * two-level one:
 *   - elements are E2M1 (as for MXFP4), codes one per byte;
 *   - a block is 16 consecutive values along K; it shares one positive E4M3
 *     scale sb (a byte with the sign bit clear);
 *   - a whole tensor shares one fp32 scale g.  A weight matrix takes
 *     g = amax / (6 * 448): the block that holds the matrix's largest
 *     magnitude then gets the largest E4M3 scale.  An all-zero matrix takes
 *     g = 1.  Here each expert's W1_e and each W2_e is one tensor.  The
 *     activations take g = 1 (reading R16);
 *   - sb = E4M3(amax_block / (g * 6)), nearest even, saturated at 448;
 *   - element = E2M1(v / (sb * g)), nearest even, saturated at 6;
 *   - a block whose scale rounds to zero encodes zeros;
 *   - the value of an element is element * sb * g.
 * The products g * 6 and sb * g and the two quotients are taken in fp32:
 * they decide integer codes, and the kernels take the same steps in fp32.
 */

/* fp32 tensor scale of a bf16 tensor of n values: amax / (6 * 448), or 1 when all are zero. */
float oracle_nv_tensor_scale(const uint16_t *w, long long n)
{
    float amax = 0.0f;
    for (long long i = 0; i < n; ++i) {
        const float a = (float)fabs(widen(w[i]));
        amax = a > amax ? a : amax;
    }
    return amax == 0.0f ? 1.0f : amax / 2688.0f;
}

/* Encode one block of 16 bf16-exact values with tensor scale g. */
static void nv_block(const double *v, float g, uint8_t *codes, uint8_t *scale)
{
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        const float a = (float)fabs(v[i]);
        amax = a > amax ? a : amax;
    }
    const float d = g * 6.0f;
    const float x = amax / d;
    const double sb = round_elem((double)x, 0); /* E4M3: nearest even, saturated at 448 */
    *scale = elem_code(sb, 0, 0);
    const float sg = (float)sb * g;
    for (int i = 0; i < 16; ++i) {
        if (sb == 0.0) {
            codes[i] = 0;
            continue;
        }
        const float q = (float)v[i] / sg;
        codes[i] = elem_code(round_elem(fabs((double)q), 1), signbit(q) != 0, 1);
    }
}

/* NVFP4 encoding of a bf16 matrix [rows, K] (K a multiple of 16) with tensor
 * scale g > 0: codes [rows, K] one per byte (E2M1), scales [rows, K/16] as
 * E4M3 bytes.  Returns 0, or -1 on bad arguments. */
int oracle_nv_quantize(const uint16_t *w, int rows, int K, float g, uint8_t *codes, uint8_t *scales)
{
    if (rows < 0 || K < 16 || K % 16 != 0 || !(g > 0.0f)) return -1;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        double v[16];
        for (int b = 0; b < K / 16; ++b) {
            for (int i = 0; i < 16; ++i) v[i] = widen(w[(size_t)r * K + b * 16 + i]);
            nv_block(v, g, codes + (size_t)r * K + b * 16, scales + (size_t)r * (K / 16) + b);
        }
    }
    return 0;
}

/* The values an NVFP4 encoding stands for: out = elem(code) * e4m3(scale) * g. */
int oracle_nv_dequantize(const uint8_t *codes, const uint8_t *scales, int rows, int K, float g, double *out)
{
    if (rows < 0 || K < 16 || K % 16 != 0) return -1;
    for (size_t i = 0; i < (size_t)rows * K; ++i)
        out[i] = elem_value(codes[i], 1) * elem_value(scales[i / 16], 0) * (double)g;
    return 0;
}

/* An activation vector as NVFP4 expert GEMMs read it: stored in bf16, then NVFP4-encoded with g = 1. */
static void nv_activation(const double *v, int n, double *out)
{
    uint8_t codes[16], scale;
    double blk[16];
    for (int b = 0; b < n / 16; ++b) {
        for (int i = 0; i < 16; ++i) blk[i] = round_bf16(v[b * 16 + i]);
        nv_block(blk, 1.0f, codes, &scale);
        for (int i = 0; i < 16; ++i) out[b * 16 + i] = elem_value(codes[i], 1) * elem_value(scale, 0);
    }
}

/* A block-scaled weight matrix: codes [rows, in_dim], scales [rows, in_dim / block],
 * with the value of every element code and of every scale byte tabulated
 * (elem_value, and 2^(byte - 127) for MX or the E4M3 value for NVFP4: the
 * same numbers, looked up), and the tensor scale g (1 for MX). */
typedef struct {
    const uint8_t *codes;
    const uint8_t *scales;
    const double *elem; /* 256 entries */
    const double *sval; /* 256 entries */
    int block;          /* 32 (MX) or 16 (NVFP4) */
    double g;
} mx_matrix;

/* out[o] = sum_i value(W[o, i]) * v[i] for a block-scaled W */
static void matvec_mx(int out_dim, int in_dim, mx_matrix W, const double *v, double *out)
{
    for (int o = 0; o < out_dim; ++o) {
        const uint8_t *row = W.codes + (size_t)o * in_dim;
        const uint8_t *sc = W.scales + (size_t)o * (in_dim / W.block);
        double s = 0.0;
        for (int i = 0; i < in_dim; ++i) s += W.elem[row[i]] * W.sval[sc[i / W.block]] * v[i];
        out[o] = s * W.g;
    }
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

/* One FFN expert in the latent space: o = W2_e act(W1_e z).  With MX expert
 * weights (mx1/mx2 non-NULL) the encoded matrices are used and the inputs z
 * and h pass through bf16 storage and the MXFP8 encoding first (step 9);
 * zq and hq are scratch of L and m values. */
static void ffn_expert(const oracle_cfg *c, const uint16_t *w1e, const uint16_t *w2e, const mx_matrix *mx1,
                       const mx_matrix *mx2, const double *z, double *zq, double *u, double *h, double *hq,
                       double *o)
{
    const int L = c->latent, m = c->m;
    const int up_rows = c->act == ORACLE_ACT_SWIGLU ? 2 * m : m;
    if (mx1) {
        if (c->expert_fmt == ORACLE_FMT_NVFP4) nv_activation(z, L, zq);
        else mx_activation(z, L, zq);
        matvec_mx(up_rows, L, *mx1, zq, u);
    } else {
        matvec(up_rows, L, w1e, z, u);
    }
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
    if (mx2) {
        if (c->expert_fmt == ORACLE_FMT_NVFP4) nv_activation(h, m, hq);
        else mx_activation(h, m, hq);
        matvec_mx(L, m, *mx2, hq, o);
    } else {
        matvec(L, m, w2e, h, o);
    }
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
    const int fmt = c->expert_fmt;
    if (fmt != ORACLE_FMT_BF16 && fmt != ORACLE_FMT_MXFP8 && fmt != ORACLE_FMT_MXFP4 && fmt != ORACLE_FMT_NVFP4)
        return -1;
    const int nv = fmt == ORACLE_FMT_NVFP4;
    const int blk = nv ? 16 : 32; /* block length along K */
    if (fmt != ORACLE_FMT_BF16 && (L % blk != 0 || m % blk != 0)) return -1;
    int bad = 0;

    /* step 9: encode the FFN experts' weights once (they are the layer's stored weights) */
    uint8_t *c1 = NULL, *s1 = NULL, *c2 = NULL, *s2 = NULL;
    float *g1 = NULL, *g2 = NULL; /* NVFP4: tensor scale of each expert's W1_e / W2_e */
    double elem_tab[256], sval_tab[256];
    for (int i = 0; i < 256; ++i) {
        const int e2m1 = fmt == ORACLE_FMT_MXFP4 || nv;
        elem_tab[i] = e2m1 ? (i < 16 ? elem_value((uint8_t)i, 1) : 0.0) : elem_value((uint8_t)i, 0);
        sval_tab[i] = nv ? elem_value((uint8_t)i, 0) : ldexp(1.0, i - 127);
    }
    if (fmt != ORACLE_FMT_BF16) {
        const size_t n1 = (size_t)c->n_ffn * up_rows * L, n2 = (size_t)c->n_ffn * L * m;
        c1 = (uint8_t *)malloc(n1 > 0 ? n1 : 1);
        s1 = (uint8_t *)malloc(n1 / blk > 0 ? n1 / blk : 1);
        c2 = (uint8_t *)malloc(n2 > 0 ? n2 : 1);
        s2 = (uint8_t *)malloc(n2 / blk > 0 ? n2 / blk : 1);
        g1 = (float *)malloc(sizeof(float) * (size_t)(c->n_ffn > 0 ? c->n_ffn : 1));
        g2 = (float *)malloc(sizeof(float) * (size_t)(c->n_ffn > 0 ? c->n_ffn : 1));
        int enc_bad = !c1 || !s1 || !c2 || !s2 || !g1 || !g2;
        if (!enc_bad && !nv) {
            enc_bad = oracle_mx_quantize(w1, c->n_ffn * up_rows, L, fmt, c1, s1) != 0 ||
                      oracle_mx_quantize(w2, c->n_ffn * L, m, fmt, c2, s2) != 0;
            for (int e = 0; e < c->n_ffn; ++e) g1[e] = g2[e] = 1.0f;
        }
        for (int e = 0; !enc_bad && nv && e < c->n_ffn; ++e) {
            const size_t o1 = (size_t)e * up_rows * L, o2 = (size_t)e * L * m;
            g1[e] = oracle_nv_tensor_scale(w1 + o1, (long long)up_rows * L);
            g2[e] = oracle_nv_tensor_scale(w2 + o2, (long long)L * m);
            enc_bad = oracle_nv_quantize(w1 + o1, up_rows, L, g1[e], c1 + o1, s1 + o1 / 16) != 0 ||
                      oracle_nv_quantize(w2 + o2, L, m, g2[e], c2 + o2, s2 + o2 / 16) != 0;
        }
        if (enc_bad) {
            free(c1); free(s1); free(c2); free(s2); free(g1); free(g2);
            return -1;
        }
    }

#pragma omp parallel reduction(| : bad)
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *z = (double *)malloc(sizeof(double) * (size_t)L);
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
        double *zq = (double *)malloc(sizeof(double) * (size_t)L);
        double *hq = (double *)malloc(sizeof(double) * (size_t)m);
        if (!xt || !z || !lg || !u || !h || !o || !yl || !up || !w || !sel || !su || !sh || !so || !zq || !hq)
            bad = 1;

#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < T; ++t) {
            if (bad) continue;
            for (int i = 0; i < d; ++i) xt[i] = widen(x[(size_t)t * d + i]);
            /* step 4: latent projection (identity for the standard MoE) */
            if (c->has_proj) matvec(L, d, w_down, xt, z);
            else memcpy(z, xt, sizeof(double) * (size_t)d);
            /* step 1: router logits at the full width (or on the latent) */
            matvec(Nt, fdim, w_router, c->latent_router ? z : xt, lg);
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
                    mx_matrix m1 = {0}, m2 = {0};
                    if (fmt != ORACLE_FMT_BF16) {
                        m1.codes = c1 + (size_t)e * up_rows * L;
                        m1.scales = s1 + (size_t)e * up_rows * (L / blk);
                        m2.codes = c2 + (size_t)e * L * m;
                        m2.scales = s2 + (size_t)e * L * (m / blk);
                        m1.elem = m2.elem = elem_tab;
                        m1.sval = m2.sval = sval_tab;
                        m1.block = m2.block = blk;
                        m1.g = g1[e];
                        m2.g = g2[e];
                    }
                    ffn_expert(c, w1 + (size_t)e * up_rows * L, w2 + (size_t)e * L * m,
                               fmt != ORACLE_FMT_BF16 ? &m1 : NULL, fmt != ORACLE_FMT_BF16 ? &m2 : NULL, z, zq, u, h,
                               hq, o);
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
        free(su); free(sh); free(so); free(zq); free(hq);
        free(xt); free(z); free(lg); free(u); free(h); free(o); free(yl); free(up); free(w); free(sel);
    }
    free(c1); free(s1); free(c2); free(s2); free(g1); free(g2);
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
