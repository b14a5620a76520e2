/*
 * Plain, slow CPU oracle for the JSSA decode step.  TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the CPU-baseline leg of the benchmark
 * may load this library.  The product path (the CUDA library) never calls it and
 * shares no code with it.
 *
 * Everything is single-threaded fp64.  bf16 values travel as their 16-bit
 * patterns (uint16_t), fp32 values (the basis P, score arrays) as float.
 *
 * Source of the method: "Joint Subspace Sparse Attention for Efficient
 * Long-Context Decoding" (Song, Kim, Kim; arXiv 2610.19026v1), as summarised on
 * its paperlayer.ai page:
 *   - Figure 1 and §3.1 (Overview): per KV head, the projected query of the
 *     group's query heads scores a projected-key cache; the top-B positions are
 *     shared by the group's query heads for attention over the original,
 *     full-dimensional keys and values.
 *   - §3.2 (Joint query-key subspace): one orthonormal basis P is applied to both
 *     queries and keys.
 *   - §3.3 (Gather-free indexed attention) and §A.3 (JSSA configuration):
 *     selections are per KV head for GQA and a single set for MLA.
 *   - §3.4 (Projected scoring cache): the projected cache is used for scoring only.
 *   - §E.1 (Component-level latency breakdown): the key of each newly generated
 *     token is projected on write.
 * Conventions the summary leaves open are fixed as follows (each is a reading):
 *   - the group query is the SUM over the group's query heads (the page says
 *     "mean"; the sum ranks identically, being the mean times G > 0);
 *   - a token's score is the dot product of the projected group query with its
 *     projected key; ties in the top-k break toward the lower token index and the
 *     selected indices are reported in ascending order;
 *   - the projected-key cache is stored in bf16, rounded to nearest-even from the
 *     exact value of K.P;
 *   - attention over the selected set is ordinary softmax attention with an
 *     explicit scale (max-subtracted, exact in fp64).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* bf16 encoding, written from the IEEE 754 binary16-"brain" definition:     */
/* 1 sign bit, 8 exponent bits (bias 127), 7 stored mantissa bits.           */
/* ------------------------------------------------------------------------- */

double or_bf16_to_double(uint16_t h)
{
    uint32_t bits = ((uint32_t)h) << 16;   /* bf16 is the top half of an fp32 */
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16, ties to even, in one step (no detour
 * through fp32, which would round twice). */
uint16_t or_double_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0x0000;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int e;
    frexp(a, &e);                 /* a = m * 2^e, 0.5 <= m < 1: leading bit is 2^(e-1) */
    int lead = e - 1;
    if (lead < -126) lead = -126; /* below the normal range the spacing stays 2^-133 */
    double quantum = ldexp(1.0, lead - 7);   /* 7 stored mantissa bits */
    double q = nearbyint(a / quantum);       /* default rounding mode: to nearest, ties even */
    double res = q * quantum;
    if (res >= 0x1p128) return (uint16_t)(sign | 0x7F80);  /* overflow rounds to infinity */
    float f = (float)res;                   /* exact: res has at most 8 significant bits */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(sign | (uint16_t)(bits >> 16));
}

void or_double_to_bf16_array(const double* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = or_double_to_bf16(x[i]);
}

/* ------------------------------------------------------------------------- */
/* Step 1 (projected scoring cache, §3.1 / §3.4 / §E.1):                      */
/*   Kp[t, j] = bf16( sum_i K[t, i] * P[i, j] )                                */
/* K rows are bf16 with row stride k_ld (elements); P is d x r, row-major fp32. */
/* kp_exact (nullable) receives the unrounded fp64 value.                      */
/* ------------------------------------------------------------------------- */
void or_project_rows(const uint16_t* K, int64_t k_ld, int d,
                     const float* P, int r, int64_t n_rows,
                     uint16_t* Kp, int64_t kp_ld, double* kp_exact)
{
    for (int64_t t = 0; t < n_rows; ++t) {
        const uint16_t* krow = K + t * k_ld;
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += or_bf16_to_double(krow[i]) * (double)P[(int64_t)i * r + j];
            Kp[t * kp_ld + j] = or_double_to_bf16(acc);
            if (kp_exact) kp_exact[t * r + j] = acc;
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Step 2 (Figure 1, §3.2): project the group's queries with the same basis:  */
/*   qs[j] = sum_g sum_i P[i, j] * q_g[i]                                      */
/* Q holds the G query heads of one KV group, each of length d (bf16).         */
/* ------------------------------------------------------------------------- */
/* ---------------------------------------------------------------------------------------
 * FP8 E4M3 projected cache (the paper's deployed projected-cache precision, §A.3 / §E.2).
 * Format (OCP 8-bit floating point, "E4M3"): 1 sign bit, 4 exponent bits with bias 7, 3
 * mantissa bits; exponent 0 encodes subnormals m * 2^-9; no infinities; S.1111.111 is NaN, so
 * the largest finite magnitude is 1.75 * 2^8 = 448.  Encoding here: round to nearest, ties to
 * even, and magnitudes that round beyond 448 saturate to 448 (the cache never holds NaN).
 * Unit scale: the stored code is the rounding of the exact product itself.
 * --------------------------------------------------------------------------------------- */
double or_e4m3_to_double(uint8_t c)
{
    const int sign = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double a;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) a = ldexp((double)m, -9);                 /* subnormal: m / 8 * 2^-6 */
    else a = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -a : a;
}

uint8_t or_double_to_e4m3(double x)
{
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (isnan(x)) return 0x7F;
    if (a >= 464.0) return (uint8_t)(sign | 0x7E);        /* 464 = midpoint of 448 and 480 */
    if (a < ldexp(1.0, -6)) {                             /* subnormal spacing 2^-9 */
        double q = nearbyint(a / ldexp(1.0, -9));         /* ties to even (default mode) */
        return (uint8_t)(sign | (uint8_t)q);              /* q = 8 is the smallest normal 0x08 */
    }
    int E;
    frexp(a, &E);                                         /* a = f * 2^E, 0.5 <= f < 1 */
    int e = E - 1;                                        /* a in [2^e, 2^(e+1)) */
    double q = nearbyint((a / ldexp(1.0, e) - 1.0) * 8.0);/* mantissa in eighths, ties even */
    if (q == 8.0) { q = 0.0; e += 1; }
    if (e > 8 || (e == 8 && q == 7.0)) return (uint8_t)(sign | 0x7E);  /* beyond 448: saturate */
    return (uint8_t)(sign | (uint8_t)((e + 7) << 3) | (uint8_t)q);
}

/* Kp8[t, j] = e4m3(sum_i K[t, i] * P[i, j]) from the exact (fp64) product. */
void or_project_rows_e4m3(const uint16_t* K, int64_t k_ld, int d, const float* P, int r, int64_t n,
                          uint8_t* Kp, int64_t kp_ld, double* kp_exact)
{
    for (int64_t t = 0; t < n; ++t) {
        const uint16_t* krow = K + t * k_ld;
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += or_bf16_to_double(krow[i]) * (double)P[(int64_t)i * r + j];
            Kp[t * kp_ld + j] = or_double_to_e4m3(acc);
            if (kp_exact) kp_exact[t * r + j] = acc;
        }
    }
}

/* s[t] = sum_j qs[j] * e4m3_value(Kp8[t, j]) in fp64. */
void or_scores_e4m3(const double* qs, int r, const uint8_t* Kp, int64_t kp_ld, int64_t n, double* s)
{
    for (int64_t t = 0; t < n; ++t) {
        double acc = 0.0;
        for (int j = 0; j < r; ++j) acc += qs[j] * or_e4m3_to_double(Kp[t * kp_ld + j]);
        s[t] = acc;
    }
}

void or_query_proj(const uint16_t* Q, int G, int d, const float* P, int r, double* qs)
{
    for (int j = 0; j < r; ++j) {
        double acc = 0.0;
        for (int g = 0; g < G; ++g)
            for (int i = 0; i < d; ++i)
                acc += (double)P[(int64_t)i * r + j] * or_bf16_to_double(Q[(int64_t)g * d + i]);
        qs[j] = acc;
    }
}

/* ------------------------------------------------------------------------- */
/* Step 3 (Figure 1, §2 "score every candidate position"):                    */
/*   s[t] = sum_j qs[j] * Kp[t, j]       for t in [0, n)                       */
/* ------------------------------------------------------------------------- */
void or_scores(const double* qs, int r, const uint16_t* Kp, int64_t kp_ld,
               int64_t n, double* s)
{
    for (int64_t t = 0; t < n; ++t) {
        double acc = 0.0;
        for (int j = 0; j < r; ++j)
            acc += qs[j] * or_bf16_to_double(Kp[t * kp_ld + j]);
        s[t] = acc;
    }
}

/* ------------------------------------------------------------------------- */
/* Step 4 (Figure 1 "top-B positions", §E.3 per-KV-head selection):           */
/* exact full sort of (score descending, index ascending); the first          */
/* k_eff = min(k, n) entries are returned in ascending index order, and the    */
/* remaining k - k_eff slots of idx are set to -1.  Returns k_eff.             */
/* ------------------------------------------------------------------------- */
typedef struct { double s; int64_t t; } or_scored;

static int or_cmp_desc(const void* a, const void* b)
{
    const or_scored* x = (const or_scored*)a;
    const or_scored* y = (const or_scored*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->t < y->t) ? -1 : (x->t > y->t) ? 1 : 0;
}

static int or_cmp_i32(const void* a, const void* b)
{
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x < y) ? -1 : (x > y) ? 1 : 0;
}

int64_t or_topk(const double* s, int64_t n, int64_t k, int32_t* idx)
{
    int64_t k_eff = (k < n) ? k : n;
    if (k_eff < 0) k_eff = 0;
    if (n > 0) {
        or_scored* all = (or_scored*)malloc((size_t)n * sizeof(or_scored));
        for (int64_t t = 0; t < n; ++t) {
            all[t].s = (s[t] == 0.0) ? 0.0 : s[t];   /* -0 and +0 are one value */
            all[t].t = t;
        }
        qsort(all, (size_t)n, sizeof(or_scored), or_cmp_desc);
        for (int64_t i = 0; i < k_eff; ++i) idx[i] = (int32_t)all[i].t;
        free(all);
        qsort(idx, (size_t)k_eff, sizeof(int32_t), or_cmp_i32);
    }
    for (int64_t i = k_eff; i < k; ++i) idx[i] = -1;
    return k_eff;
}

/* ------------------------------------------------------------------------- */
/* Step 5 (Figure 1, §3.3): softmax attention of G query heads over a given   */
/* token list, reading the original full-dimensional K and V rows:            */
/*   l_t = scale * q . K_t ;  p = softmax(l) ;  O = sum_t p_t V_t              */
/* The list may be in any order and must hold distinct, in-range positions.   */
/* lse (nullable) receives m + log(sum exp(l - m)) per head.  An empty list   */
/* gives O = 0 and lse = -inf.                                                 */
/* ------------------------------------------------------------------------- */
void or_attention(const uint16_t* Q, int G, int dk,
                  const uint16_t* K, int64_t k_ld,
                  const uint16_t* V, int64_t v_ld, int dv,
                  const int64_t* tokens, int64_t n_tok, double scale,
                  double* O, double* lse)
{
    double* logit = (double*)malloc((size_t)(n_tok > 0 ? n_tok : 1) * sizeof(double));
    for (int g = 0; g < G; ++g) {
        const uint16_t* q = Q + (int64_t)g * dk;
        double m = -INFINITY;
        for (int64_t i = 0; i < n_tok; ++i) {
            const uint16_t* krow = K + tokens[i] * k_ld;
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += or_bf16_to_double(q[c]) * or_bf16_to_double(krow[c]);
            logit[i] = scale * acc;
            if (logit[i] > m) m = logit[i];
        }
        double l = 0.0;
        for (int64_t i = 0; i < n_tok; ++i) { logit[i] = exp(logit[i] - m); l += logit[i]; }
        double* o = O + (int64_t)g * dv;
        for (int c = 0; c < dv; ++c) o[c] = 0.0;
        for (int64_t i = 0; i < n_tok; ++i) {
            const uint16_t* vrow = V + tokens[i] * v_ld;
            double w = logit[i] / l;
            for (int c = 0; c < dv; ++c) o[c] += w * or_bf16_to_double(vrow[c]);
        }
        if (lse) lse[g] = (n_tok > 0) ? m + log(l) : -INFINITY;
    }
    free(logit);
}

/* ------------------------------------------------------------------------- */
/* One decode step for one (sequence, KV head) problem, composed from the     */
/* steps above (Figure 1).  Inputs:                                           */
/*   Q     [G, dk]     the group's query heads                                */
/*   K, V  rows [0, T) of this head's cache (row strides k_ld, v_ld)           */
/*   Kp    rows [0, T) of this head's projected cache (row stride kp_ld)       */
/*   P     [dk, r]     this head's basis                                       */
/* Candidates are [0, T - W); the attended list is the selected set followed  */
/* by the window [T - W, T) (W clamped to [0, T]).  Outputs: idx[k] (ascending,*/
/* -1 padded), O [G, dv], lse [G] (nullable), scores [T - W] (nullable).      */
/* Returns k_eff.                                                              */
/* ------------------------------------------------------------------------- */
int64_t or_decode_head(const uint16_t* Q, int G, int dk, int dv,
                       const uint16_t* K, int64_t k_ld,
                       const uint16_t* V, int64_t v_ld,
                       const uint16_t* Kp, int64_t kp_ld,
                       const float* P, int r,
                       int64_t T, int64_t k, int64_t W, double scale,
                       int32_t* idx, double* O, double* lse, double* scores_out)
{
    if (W < 0) W = 0;
    if (W > T) W = T;
    int64_t n = T - W;
    double qs[1024];
    if (r > 1024) return -1;      /* the projected query is held on the stack */
    or_query_proj(Q, G, dk, P, r, qs);
    double* s = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    or_scores(qs, r, Kp, kp_ld, n, s);
    if (scores_out) memcpy(scores_out, s, (size_t)n * sizeof(double));
    int64_t k_eff = or_topk(s, n, k, idx);
    free(s);
    int64_t n_tok = k_eff + W;
    int64_t* list = (int64_t*)malloc((size_t)(n_tok > 0 ? n_tok : 1) * sizeof(int64_t));
    for (int64_t i = 0; i < k_eff; ++i) list[i] = idx[i];
    for (int64_t i = 0; i < W; ++i) list[k_eff + i] = n + i;
    or_attention(Q, G, dk, K, k_ld, V, v_ld, dv, list, n_tok, scale, O, lse);
    free(list);
    return k_eff;
}
