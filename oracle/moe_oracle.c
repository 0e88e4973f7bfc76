/*
 * moe_oracle.c -- plain, slow CPU statement of the MoE expert layer.
 *
 * TEST INFRASTRUCTURE ONLY.  The CUDA library never includes, links or calls
 * this file, and this file shares no code, header, table or helper with it.
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * use it.
 *
 * Sources (web pages on the subject; cited by title and section):
 *  [MoE-latency]  "MoE 少算 FLOPs,延迟反而涨了:慢在搬 token 的路上"
 *                 sections "dense 和 MoE 的差别" (router scores every expert,
 *                 picks top-2, emits two routing weights; only the picked
 *                 experts process the token) and "router 之后还有一串动作"
 *                 (k assignments per token, grouped by expert = dispatch, rows
 *                 sorted by expert = permutation, one matrix per expert in a
 *                 grouped GEMM, inverse mapping back to token order, multiply
 *                 by routing weight, sum = combine / unpermutation).
 *  [FinDEP]       "FinDEP: Efficient MoE Inference with Fine-Grained
 *                 Scheduling of Disaggregated Expert Parallelism", section
 *                 "核心公式", MoE-layer formula: three GEMMs per expert
 *                 (here the SwiGLU form W1, W3, W2); section "问题定义":
 *                 shared experts are always-on experts.
 *  [MoE-latency]  also section "优化从测量开始": quantizing weights (or
 *                 activations) cuts memory bytes, and its numerical error has to
 *                 be measured as an experiment of its own.
 *  [MegaScale]    "MegaScale-Infer: Serving Mixture-of-Experts at Scale with
 *                 Disaggregated Expert Parallelism", section "核心问题"
 *                 (Mixtral 8x22B: 156 tokens over 8 experts at top-2 gives
 *                 39 rows per expert on average).
 *
 * Readings where the pages are silent (each one is a choice, documented in the
 * design notes):
 *  - logits: fp32 W_gate, bf16 x; the oracle sums in fp64 and rounds the logit
 *    to fp32, because the expert choice (an integer decided by floating point)
 *    is taken in the kernel's precision, fp32;
 *  - top-k: larger fp32 logit first; on equal values the lower expert index
 *    wins; picks are listed in that order;
 *  - routing weights: softmax over all E renormalised over the k picks, which
 *    equals a softmax over the k picked logits: w_j = e^(l_j-l_0)/sum_i e^(l_i-l_0);
 *  - dispatch is stable: inside an expert's group, rows follow assignment id
 *    a = t*k + j;
 *  - expert FFN is SwiGLU: h = silu(x W1^T) * (x W3^T), y = h W2^T,
 *    silu(z) = z / (1 + e^-z); all sums in fp64; bf16 rounding (to nearest,
 *    ties to even) at h (the operand of the second GEMM) and at out only: the
 *    expert outputs y and the shared-expert output s stay unrounded through
 *    the combine, so the k-term weighted sum does not amplify a one-ulp
 *    rounding of a term where the terms cancel;
 *  - combine: out[t] = bf16( sum_j w_j * y[row(t,j)] + s[t] ), j in pick order;
 *  - shared experts (optional, Is > 0): one SwiGLU FFN of width Is over every
 *    token, weight 1, added after the routed sum;
 *  - fp8 expert weights (the pages name no format): OCP e4m3 (no infinities,
 *    largest finite 448) with one fp32 scale per output channel (weight row):
 *    s = max|row| / 448 in fp32, q = e4m3(w / s) rounded to nearest even with
 *    magnitudes past 448 kept at 448; the weight the FFN uses is e4m3(q) * s.
 *    Activations, routing, combine and the shared experts are unchanged;
 *  - fp8 activations as well (the same section names activations beside
 *    weights): each row the two routed GEMMs read -- a permuted token row x and
 *    a row of h after its bf16 rounding -- goes through the same per-row
 *    quantizer, and the GEMM uses e4m3(q) * s for it.  Routing, combine and the
 *    shared experts are unchanged.
 *
 * Layouts: x [N,H] bf16 (uint16 storage); W_gate [H,E] fp32; bias [E] fp32 or
 * NULL; W1, W3 [E,I,H] bf16; W2 [E,H,I] bf16; Ws1, Ws3 [Is,H] bf16;
 * Ws2 [H,Is] bf16; all row-major.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* The same file builds two libraries: a serial one, and (with -fopenmp) one whose
 * loops over independent tokens or rows run on several host threads.  A row's or a
 * token's arithmetic is the same in both -- the same operations in the same order on
 * one thread -- so the two give identical bits; only which thread computes a row
 * differs.  oracle_threads(n) sets the thread count (n > 0) and returns the count in
 * use, 1 for the serial build. */
int oracle_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ---------------------------------------------------------------- bf16 ---- */

/* bf16 keeps the top 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double straight to bf16 (8 significant bits, binary32 exponent
 * range), to nearest with ties to even, overflow to infinity.  No detour
 * through fp32, so there is no double rounding. */
uint16_t oracle_round_to_bf16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v)) return 0x7FC0u;
    if (isinf(v)) return (uint16_t)(sign | 0x7F80u);
    double a = fabs(v), q;
    if (a < 0x1p-126) {
        /* subnormal range: the spacing is 2^-133 */
        q = rint(a * 0x1p133) * 0x1p-133;
    } else {
        int ex;
        double m = frexp(a, &ex); /* a = m * 2^ex, 0.5 <= m < 1 */
        q = ldexp(rint(ldexp(m, 8)), ex - 8);
    }
    if (q >= 0x1p128) return (uint16_t)(sign | 0x7F80u);
    float f = (float)q; /* exact: q has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

/* ----------------------------------------------------------------- fp8 ---- */

/* OCP 8-bit float e4m3: sign bit, 4 exponent bits with bias 7, 3 mantissa bits.
 * Exponent field 0 holds subnormals (m/8) * 2^-6; all-ones exponent with all-ones
 * mantissa (0x7F, 0xFF) is NaN; there are no infinities; the largest finite
 * magnitude is 1.75 * 2^8 = 448. */
double oracle_fp8_e4m3_to_double(uint8_t q)
{
    int sign = (q >> 7) & 1, ex = (q >> 3) & 15, m = q & 7;
    double v;
    if (ex == 15 && m == 7) return NAN;
    if (ex == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, ex - 7);
    return sign ? -v : v;
}

/* Nearest e4m3 value to v, ties to the even code (mantissa bit 0 clear);
 * magnitudes at or past 448 give 448 (v must not be NaN). */
uint8_t oracle_fp8_e4m3_from_float(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int e2;
    frexp(a, &e2);       /* a in [2^(e2-1), 2^e2) */
    int E = e2 - 1;      /* unbiased exponent of a */
    if (E < -6) E = -6;  /* subnormal range: spacing 2^-9 */
    double step = ldexp(1.0, E - 3);
    double n = nearbyint(a / step); /* a / step is exact; default rounding: ties to even */
    double r = n * step;            /* at most 448 here */
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -6)) return (uint8_t)(sign | (int)(r / ldexp(1.0, -9)));
    int er;
    frexp(r, &er);
    int Er = er - 1;
    int m = (int)(r / ldexp(1.0, Er - 3)) - 8;
    return (uint8_t)(sign | ((Er + 7) << 3) | m);
}

/* Per output channel quantization of a bf16 weight matrix [rows, K]:
 * s[r] = max_c |W[r,c]| / 448 in fp32 (1 for an all-zero row), q[r,c] =
 * e4m3(float(W[r,c]) / s[r]) with the division in fp32. */
void oracle_quantize_rows_fp8(const uint16_t *W, int64_t rows, int K, uint8_t *q, float *s)
{
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int c = 0; c < K; ++c) {
            float a = fabsf((float)oracle_bf16_to_double(W[r * K + c]));
            if (a > amax) amax = a;
        }
        float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
        s[r] = sc;
        for (int c = 0; c < K; ++c) {
            volatile float t = (float)oracle_bf16_to_double(W[r * K + c]) / sc; /* fp32 quotient */
            q[r * K + c] = oracle_fp8_e4m3_from_float(t);
        }
    }
}

/* -------------------------------------------------------------- router ---- */

/* [MoE-latency] "dense 和 MoE 的差别": the router reads a token's hidden state
 * and scores every expert.  logits[t,e] = sum_h x[t,h] * W_gate[h,e] + bias[e],
 * in fp64. */
void oracle_router_logits(const uint16_t *x, const float *W_gate, const float *bias,
                          int64_t N, int H, int E, double *logits)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t)
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int h = 0; h < H; ++h)
                s += oracle_bf16_to_double(x[t * H + h]) * (double)W_gate[(int64_t)h * E + e];
            if (bias) s += (double)bias[e];
            logits[t * E + e] = s;
        }
}

/* [MoE-latency] "dense 和 MoE 的差别": pick the top-k experts and give k
 * routing weights.  Selection compares fp32 values; ties go to the lower
 * index.  w is the softmax over the k picked logits (equal to the full softmax
 * renormalised over the picks).  Returns 0, or -1 on bad sizes. */
int oracle_topk(const float *logits, int64_t N, int E, int k, int32_t *idx, double *w)
{
    if (E < 1 || k < 1 || k > E) return -1;
    char *taken = (char *)malloc((size_t)E);
    if (!taken) return -1;
    for (int64_t t = 0; t < N; ++t) {
        const float *l = logits + t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict: lower index keeps a tie */
            }
            taken[best] = 1;
            idx[t * k + j] = best;
        }
        double l0 = (double)l[idx[t * k]], den = 0.0;
        for (int j = 0; j < k; ++j) den += exp((double)l[idx[t * k + j]] - l0);
        for (int j = 0; j < k; ++j) w[t * k + j] = exp((double)l[idx[t * k + j]] - l0) / den;
    }
    free(taken);
    return 0;
}

/* ------------------------------------------------------------ dispatch ---- */

/* [MoE-latency] "router 之后还有一串动作": N tokens give N*k assignments;
 * grouping them by expert is dispatch, sorting token rows by expert is the
 * permutation.  counts[e] = #assignments to e; offsets = exclusive scan with
 * offsets[E] = N*k; assignment a = t*k+j lands at row offsets[e] + (number of
 * earlier assignments to e).  Returns 0, or -1 on an index outside [0,E). */
int oracle_dispatch(const int32_t *idx, int64_t N, int E, int k, int32_t *counts,
                    int32_t *offsets, int32_t *row_to_token, int32_t *token_to_row)
{
    if (E < 1 || k < 1 || N < 0) return -1;
    int64_t R = N * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t a = 0; a < R; ++a) {
        if (idx[a] < 0 || idx[a] >= E) return -1;
        counts[idx[a]] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    if (!fill) return -1;
    for (int64_t a = 0; a < R; ++a) {
        int e = idx[a];
        int32_t row = offsets[e] + fill[e]++;
        row_to_token[row] = (int32_t)(a / k);
        token_to_row[a] = row;
    }
    free(fill);
    return 0;
}

/* x_perm[row] = x[row_to_token[row]] (the permuted copy of token rows). */
void oracle_permute_rows(const uint16_t *x, const int32_t *row_to_token, int64_t R, int H,
                         uint16_t *x_perm)
{
    for (int64_t r = 0; r < R; ++r)
        memcpy(x_perm + r * H, x + (int64_t)row_to_token[r] * H, (size_t)H * sizeof(uint16_t));
}

/* ---------------------------------------------------------- expert FFN ---- */

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* One expert weight stack [E*rows, K] (row-major; expert e's rows start at
 * e*rows): bf16 (w8 == NULL), or e4m3 codes with one fp32 scale per row, whose
 * weight is e4m3(q) * s. */
typedef struct {
    const uint16_t *w16;
    const uint8_t *w8;
    const float *sc;
} oracle_wmat;

/* the 256 e4m3 values, filled from oracle_fp8_e4m3_to_double on first use */
static double fp8_value[256];
static int fp8_value_ready = 0;

static double fp8_val(uint8_t q)
{
    if (!fp8_value_ready) {
        for (int i = 0; i < 256; ++i) fp8_value[i] = oracle_fp8_e4m3_to_double((uint8_t)i);
        fp8_value_ready = 1;
    }
    return fp8_value[q];
}

static double wval(const oracle_wmat *m, int64_t row, int K, int c)
{
    if (m->w8) return fp8_val(m->w8[row * K + c]) * (double)m->sc[row];
    return oracle_bf16_to_double(m->w16[row * K + c]);
}

/* The values a GEMM reads for one bf16 activation row of K elements: the row
 * itself, or (quantize != 0) e4m3(q) * s from the per-row quantizer above. */
static void act_row(const uint16_t *row, int K, int quantize, double *d)
{
    if (quantize) {
        uint8_t *q = (uint8_t *)malloc((size_t)K);
        float s;
        oracle_quantize_rows_fp8(row, 1, K, q, &s);
        for (int c = 0; c < K; ++c) d[c] = fp8_val(q[c]) * (double)s;
        free(q);
    } else {
        for (int c = 0; c < K; ++c) d[c] = oracle_bf16_to_double(row[c]);
    }
}

/* [FinDEP] "核心公式": an expert is three GEMMs; here the SwiGLU expert
 * y = W2 (silu(W1 x) * (W3 x)).  One row through the expert whose W1/W3 rows
 * start at r13 and whose W2 rows start at r2.  fp64 sums; h rounded to bf16,
 * y left in fp64.  qa != 0 quantizes the activation rows (x, and h after its
 * rounding) as described at the top.  h_out (may be NULL) receives the bf16 h;
 * h_given (may be NULL) replaces it as the second GEMM's input. */
static void swiglu_row(const uint16_t *xrow, const oracle_wmat *W1, const oracle_wmat *W3,
                       const oracle_wmat *W2, int64_t r13, int64_t r2, int H, int I, int qa,
                       const uint16_t *h_given, uint16_t *h_out, double *yrow)
{
    double *xd = (double *)malloc((size_t)H * sizeof(double));
    double *hd = (double *)malloc((size_t)I * sizeof(double));
    uint16_t *hb = (uint16_t *)malloc((size_t)I * sizeof(uint16_t));
    act_row(xrow, H, qa, xd);
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; ++c) {
            g += xd[c] * wval(W1, r13 + i, H, c);
            u += xd[c] * wval(W3, r13 + i, H, c);
        }
        hb[i] = oracle_round_to_bf16(silu(g) * u);
    }
    if (h_out) memcpy(h_out, hb, (size_t)I * sizeof(uint16_t));
    act_row(h_given ? h_given : hb, I, qa, hd);
    for (int o = 0; o < H; ++o) {
        double y = 0.0;
        for (int i = 0; i < I; ++i) y += hd[i] * wval(W2, r2 + o, I, i);
        yrow[o] = y;
    }
    free(xd);
    free(hd);
    free(hb);
}

/* One row, one expert with bf16 weights: W1, W3 [I,H], W2 [H,I]. */
void oracle_swiglu_ffn(const uint16_t *xrow, const uint16_t *W1, const uint16_t *W3,
                       const uint16_t *W2, int H, int I, double *yrow)
{
    oracle_wmat a = {W1, NULL, NULL}, b = {W3, NULL, NULL}, c = {W2, NULL, NULL};
    swiglu_row(xrow, &a, &b, &c, 0, 0, H, I, 0, NULL, NULL, yrow);
}

/* [MoE-latency] "router 之后还有一串动作": each expert runs its own rows.
 * Rows offsets[e] .. offsets[e+1]-1 of x_perm go through expert e.  h_given
 * and h_out (may be NULL) are [R,I] in the same (permuted) row order. */
static void expert_ffn(const uint16_t *x_perm, const int32_t *offsets, const oracle_wmat *W1,
                       const oracle_wmat *W3, const oracle_wmat *W2, int E, int H, int I, int qa,
                       const uint16_t *h_given, uint16_t *h_out, double *y_perm)
{
    /* every row is independent: row r goes through the expert whose group holds it */
    const int64_t R = offsets[E] > 0 ? offsets[E] : 0;
    int32_t *expert_of = (int32_t *)malloc((size_t)(R > 0 ? R : 1) * sizeof(int32_t));
    if (!expert_of) return;
    for (int64_t r = 0; r < R; ++r) expert_of[r] = -1; /* rows before offsets[0]: no expert */
    for (int e = 0; e < E; ++e)
        for (int64_t r = offsets[e]; r < offsets[e + 1]; ++r)
            if (r >= 0 && r < R) expert_of[r] = e;
    (void)fp8_val(0); /* fill the e4m3 table before the rows run side by side */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        const int e = expert_of[r];
        if (e < 0) continue;
        swiglu_row(x_perm + r * H, W1, W3, W2, (int64_t)e * I, (int64_t)e * H, H, I, qa,
                   h_given ? h_given + r * I : NULL, h_out ? h_out + r * I : NULL,
                   y_perm + r * H);
    }
    free(expert_of);
}

void oracle_expert_ffn(const uint16_t *x_perm, const int32_t *offsets, const uint16_t *W1,
                       const uint16_t *W3, const uint16_t *W2, int E, int H, int I,
                       double *y_perm)
{
    oracle_wmat a = {W1, NULL, NULL}, b = {W3, NULL, NULL}, c = {W2, NULL, NULL};
    expert_ffn(x_perm, offsets, &a, &b, &c, E, H, I, 0, NULL, NULL, y_perm);
}

/* [MoE-latency] "优化从测量开始": the same experts with e4m3 weights q1, q3
 * [E,I,H], q2 [E,H,I] and per-row scales s1, s3 [E,I], s2 [E,H]. */
void oracle_expert_ffn_fp8(const uint16_t *x_perm, const int32_t *offsets, const uint8_t *q1,
                           const float *s1, const uint8_t *q3, const float *s3, const uint8_t *q2,
                           const float *s2, int E, int H, int I, double *y_perm)
{
    oracle_wmat a = {NULL, q1, s1}, b = {NULL, q3, s3}, c = {NULL, q2, s2};
    expert_ffn(x_perm, offsets, &a, &b, &c, E, H, I, 0, NULL, NULL, y_perm);
}

/* The e4m3-weight experts with the two activation options: quantize_acts != 0
 * quantizes every row of x_perm and of h per row as well (e4m3 with one fp32
 * scale, as for the weights).  h_given [R,I] bf16 (may be NULL) replaces the
 * computed h as the second GEMM's input -- so that a caller can hand in h as
 * another implementation rounded it and take the quantization decision on the
 * same values; h_out [R,I] (may be NULL) receives the computed bf16 h. */
void oracle_expert_ffn_fp8_ex(const uint16_t *x_perm, const int32_t *offsets, const uint8_t *q1,
                              const float *s1, const uint8_t *q3, const float *s3,
                              const uint8_t *q2, const float *s2, int E, int H, int I,
                              int quantize_acts, const uint16_t *h_given, double *y_perm,
                              uint16_t *h_out)
{
    oracle_wmat a = {NULL, q1, s1}, b = {NULL, q3, s3}, c = {NULL, q2, s2};
    expert_ffn(x_perm, offsets, &a, &b, &c, E, H, I, quantize_acts != 0, h_given, h_out, y_perm);
}

/* ------------------------------------------------------------- combine ---- */

/* [MoE-latency] "router 之后还有一串动作": inverse mapping back to token
 * order, multiply by the routing weight, add.  out[t] = bf16(sum_j w[t,j] *
 * y_perm[token_to_row[t,j]] + s[t]) in fp64, j in pick order; s may be NULL. */
void oracle_combine(const double *y_perm, const int32_t *token_to_row, const double *w,
                    const double *s, int64_t N, int H, int k, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t)
        for (int o = 0; o < H; ++o) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += w[t * k + j] * y_perm[(int64_t)token_to_row[t * k + j] * H + o];
            if (s) acc += s[t * H + o];
            out[t * H + o] = oracle_round_to_bf16(acc);
        }
}

/* --------------------------------------------------------------- layer ---- */

/* The whole sparse path from given fp32 logits: top-k, dispatch, permuted
 * rows, per-expert SwiGLU, optional shared experts ([FinDEP] "问题定义"),
 * combine.  Optional outputs (may be NULL): idx [N,k], w [N,k], counts [E],
 * offsets [E+1], row_to_token [N*k], token_to_row [N*k], y_perm [N*k,H] (fp64).
 * Returns 0, or -1 on bad arguments / allocation failure. */
static int layer_core(const uint16_t *x, const float *logits, const oracle_wmat *W1,
                      const oracle_wmat *W3, const oracle_wmat *W2, const uint16_t *Ws1,
                      const uint16_t *Ws3, const uint16_t *Ws2, int64_t N, int H, int I, int E, int k,
                      int Is, int qa, const uint16_t *h_given_tok, uint16_t *out, int32_t *idx_out,
                      double *w_out, int32_t *counts_out, int32_t *offsets_out, int32_t *r2t_out,
                      int32_t *t2r_out, double *y_perm_out)
{
    if (N < 0 || H < 1 || I < 1 || E < 1 || k < 1 || k > E || Is < 0) return -1;
    int64_t R = N * k;
    int rc = -1;
    int32_t *idx = (int32_t *)malloc((size_t)(R ? R : 1) * sizeof(int32_t));
    double *w = (double *)malloc((size_t)(R ? R : 1) * sizeof(double));
    int32_t *counts = (int32_t *)malloc((size_t)E * sizeof(int32_t));
    int32_t *offsets = (int32_t *)malloc((size_t)(E + 1) * sizeof(int32_t));
    int32_t *r2t = (int32_t *)malloc((size_t)(R ? R : 1) * sizeof(int32_t));
    int32_t *t2r = (int32_t *)malloc((size_t)(R ? R : 1) * sizeof(int32_t));
    uint16_t *xp = (uint16_t *)malloc((size_t)(R ? R : 1) * H * sizeof(uint16_t));
    double *yp = (double *)malloc((size_t)(R ? R : 1) * H * sizeof(double));
    double *s = NULL;
    uint16_t *hp = NULL;
    if (!idx || !w || !counts || !offsets || !r2t || !t2r || !xp || !yp) goto done;
    if (oracle_topk(logits, N, E, k, idx, w)) goto done;
    if (oracle_dispatch(idx, N, E, k, counts, offsets, r2t, t2r)) goto done;
    oracle_permute_rows(x, r2t, R, H, xp);
    if (h_given_tok) {
        /* given h rows come in assignment order a = t*k + j; the experts read
         * them in permuted order, at row token_to_row[a] */
        hp = (uint16_t *)malloc((size_t)(R ? R : 1) * I * sizeof(uint16_t));
        if (!hp) goto done;
        for (int64_t a = 0; a < R; ++a)
            memcpy(hp + (int64_t)t2r[a] * I, h_given_tok + a * I, (size_t)I * sizeof(uint16_t));
    }
    expert_ffn(xp, offsets, W1, W3, W2, E, H, I, qa, hp, NULL, yp);
    if (Is > 0) {
        s = (double *)malloc((size_t)(N ? N : 1) * H * sizeof(double));
        if (!s) goto done;
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t t = 0; t < N; ++t) oracle_swiglu_ffn(x + t * H, Ws1, Ws3, Ws2, H, Is, s + t * H);
    }
    oracle_combine(yp, t2r, w, s, N, H, k, out);
    if (idx_out) memcpy(idx_out, idx, (size_t)R * sizeof(int32_t));
    if (w_out) memcpy(w_out, w, (size_t)R * sizeof(double));
    if (counts_out) memcpy(counts_out, counts, (size_t)E * sizeof(int32_t));
    if (offsets_out) memcpy(offsets_out, offsets, (size_t)(E + 1) * sizeof(int32_t));
    if (r2t_out) memcpy(r2t_out, r2t, (size_t)R * sizeof(int32_t));
    if (t2r_out) memcpy(t2r_out, t2r, (size_t)R * sizeof(int32_t));
    if (y_perm_out) memcpy(y_perm_out, yp, (size_t)R * H * sizeof(double));
    rc = 0;
done:
    free(idx); free(w); free(counts); free(offsets); free(r2t); free(t2r); free(xp); free(yp);
    free(s); free(hp);
    return rc;
}

int oracle_layer_given_logits(const uint16_t *x, const float *logits, const uint16_t *W1,
                              const uint16_t *W3, const uint16_t *W2, const uint16_t *Ws1,
                              const uint16_t *Ws3, const uint16_t *Ws2, int64_t N, int H, int I,
                              int E, int k, int Is, uint16_t *out, int32_t *idx_out,
                              double *w_out, int32_t *counts_out, int32_t *offsets_out,
                              int32_t *r2t_out, int32_t *t2r_out, double *y_perm_out)
{
    oracle_wmat a = {W1, NULL, NULL}, b = {W3, NULL, NULL}, c = {W2, NULL, NULL};
    return layer_core(x, logits, &a, &b, &c, Ws1, Ws3, Ws2, N, H, I, E, k, Is, 0, NULL, out, idx_out,
                      w_out, counts_out, offsets_out, r2t_out, t2r_out, y_perm_out);
}

/* The same path with e4m3 routed-expert weights (q1, q3 [E,I,H], q2 [E,H,I])
 * and per-row scales (s1, s3 [E,I], s2 [E,H]); shared experts stay bf16. */
int oracle_layer_given_logits_fp8(const uint16_t *x, const float *logits, const uint8_t *q1,
                                  const float *s1, const uint8_t *q3, const float *s3,
                                  const uint8_t *q2, const float *s2, const uint16_t *Ws1,
                                  const uint16_t *Ws3, const uint16_t *Ws2, int64_t N, int H, int I,
                                  int E, int k, int Is, uint16_t *out, double *y_perm_out)
{
    oracle_wmat a = {NULL, q1, s1}, b = {NULL, q3, s3}, c = {NULL, q2, s2};
    return layer_core(x, logits, &a, &b, &c, Ws1, Ws3, Ws2, N, H, I, E, k, Is, 0, NULL, out, NULL,
                      NULL, NULL, NULL, NULL, NULL, y_perm_out);
}

/* The e4m3-weight layer with the activation options of oracle_expert_ffn_fp8_ex:
 * quantize_acts != 0 quantizes the routed experts' activation rows; h_given_tok
 * (may be NULL) is [N*k, I] bf16 in assignment order (row a = t*k + j is the h
 * of token t's j-th pick) and replaces the computed h. */
int oracle_layer_given_logits_fp8_ex(const uint16_t *x, const float *logits, const uint8_t *q1,
                                     const float *s1, const uint8_t *q3, const float *s3,
                                     const uint8_t *q2, const float *s2, const uint16_t *Ws1,
                                     const uint16_t *Ws3, const uint16_t *Ws2, int64_t N, int H,
                                     int I, int E, int k, int Is, int quantize_acts,
                                     const uint16_t *h_given_tok, uint16_t *out, double *y_perm_out)
{
    oracle_wmat a = {NULL, q1, s1}, b = {NULL, q3, s3}, c = {NULL, q2, s2};
    return layer_core(x, logits, &a, &b, &c, Ws1, Ws3, Ws2, N, H, I, E, k, Is, quantize_acts != 0,
                      h_given_tok, out, NULL, NULL, NULL, NULL, NULL, NULL, y_perm_out);
}

/* The whole layer from x: fp64 logits rounded to fp32 (the precision the
 * expert choice is taken in), then the path above.  logits_out [N,E] may be
 * NULL. */
int oracle_layer(const uint16_t *x, const float *W_gate, const float *bias, const uint16_t *W1,
                 const uint16_t *W3, const uint16_t *W2, const uint16_t *Ws1, const uint16_t *Ws3,
                 const uint16_t *Ws2, int64_t N, int H, int I, int E, int k, int Is,
                 uint16_t *out, float *logits_out)
{
    if (N < 0 || H < 1 || E < 1) return -1;
    double *l64 = (double *)malloc((size_t)(N ? N : 1) * E * sizeof(double));
    float *l32 = (float *)malloc((size_t)(N ? N : 1) * E * sizeof(float));
    int rc = -1;
    if (l64 && l32) {
        oracle_router_logits(x, W_gate, bias, N, H, E, l64);
        for (int64_t i = 0; i < N * E; ++i) l32[i] = (float)l64[i];
        rc = oracle_layer_given_logits(x, l32, W1, W3, W2, Ws1, Ws3, Ws2, N, H, I, E, k, Is, out,
                                       NULL, NULL, NULL, NULL, NULL, NULL, NULL);
        if (rc == 0 && logits_out) memcpy(logits_out, l32, (size_t)N * E * sizeof(float));
    }
    free(l64);
    free(l32);
    return rc;
}
