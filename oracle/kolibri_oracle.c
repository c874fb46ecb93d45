/*
 * kolibri_oracle.c -- plain, slow, obviously correct CPU reference for the
 * sigmoid-router + Exact Quantile Balancing (EQB) routing path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * with the CUDA kernels; the two sides were written independently from the
 * method's definition and meet only through seeded inputs.
 *
 * Sources (page, then section):
 *   [KPT]  "Kolibri Pre-Training from Scratch: UniBPE, Hybrid Attention and
 *           Exact Quantile Balancing" -- section 1 (definition of Q_m),
 *           6.1 (routing equations), 6.2 (MaxVio), 7.1 (Quantile Balancing),
 *           7.2 (numerical check), 7.3 (exact quantile by radix selection),
 *           9 (intervention rate).
 *           6.1 also defines the layer output y_t = f_shared(x_t) +
 *           sum_e S_t,e f_e(x_t) that the experts compute.
 *   [K1D]  "Kolibri 1 im Detail: hybride RNoPE-Attention, Sparse MoE und
 *           FP8-Serving" -- section "Routing: Auswahl-Bias und Mischgewichte
 *           sind getrennt" (bf16 router, fp32 logits, two-step rule; every
 *           routed or shared expert a SwiGLU MLP 2560 -> 2 x 512 -> 2560).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - Total order on fp32: the order-preserving key of the bit pattern
 *     (negative values: all bits flipped; non-negative: sign bit set), so
 *     -0.0 sorts below +0.0.  Equal keys are ties.
 *   - Top-K output order: biased score descending, ties to the lower id.
 *   - r = T*K/E is taken as m = floor(N*K/E).
 *   - Centring: fp64 sum of the fp32 biases in ascending expert order,
 *     divided by E in fp64, rounded once to fp32, subtracted in fp32.
 *   - Gate: sigmoid evaluated in fp64 with the exp defined in exp_spec()
 *     below, rounded once to fp32.
 *   - Permutation: experts ascending, and inside an expert the flat slot
 *     index t*K+k ascending (a stable counting sort).
 *   - Experts: the SwiGLU activation h = SiLU(gate) * up is rounded once to
 *     bf16 (the operand of the down projection); everything else is fp64,
 *     and the layer output is rounded once to fp32.
 *
 * Build: plain C11, no fast-math, no FP contraction (the arithmetic must be
 * exactly the operations written).  OpenMP only splits independent rows or
 * columns; it never changes an operation or its order.
 *
 * Parity pins: every function here is pinned in tests/test_oracle_pins.py
 * against values printed on the pages, closed forms, invariants or brute
 * force.  No function is parity-unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- scalars */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the upper half of an fp32 bit pattern. */
static double bf16_value(uint16_t b) { return (double)bits_to_f32((uint32_t)b << 16); }

/* Order-preserving map from fp32 bits to an unsigned key: a < b as keys
 * exactly when a sorts below b in the total order above. */
uint32_t oracle_order_key(float v)
{
    uint32_t u = f32_to_bits(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

/* exp for the gate, in fp64.  Method: Cody & Waite range reduction
 * x = k*ln2 + r with ln2 split into a double-double (hi, lo), then the
 * degree-13 Taylor polynomial of e^r in Horner form with fused multiply-add,
 * then scaling by 2^k assembled from the exponent field.  Domain used here:
 * |x| <= 700 (k stays inside the normal exponent range).  Every step is an
 * IEEE correctly rounded operation, so any IEEE machine that performs the
 * same steps gets the same bits. */
double oracle_exp_spec(double x)
{
    const double inv_ln2 = 1.4426950408889634;            /* 1/ln 2, rounded */
    const double ln2_hi  = 0.69314718055994528623;         /* ln 2, rounded   */
    const double ln2_lo  = 2.3190468138462996e-17;         /* ln 2 - ln2_hi   */
    double k = rint(x * inv_ln2);
    double r = fma(-k, ln2_hi, x);
    r = fma(-k, ln2_lo, r);
    /* Taylor coefficients 1/n!, n = 13 .. 1, each the double nearest 1/n!. */
    double p = 1.0 / 6227020800.0;                         /* 1/13! */
    p = fma(p, r, 1.0 / 479001600.0);                      /* 1/12! */
    p = fma(p, r, 1.0 / 39916800.0);                       /* 1/11! */
    p = fma(p, r, 1.0 / 3628800.0);                        /* 1/10! */
    p = fma(p, r, 1.0 / 362880.0);                         /* 1/9!  */
    p = fma(p, r, 1.0 / 40320.0);                          /* 1/8!  */
    p = fma(p, r, 1.0 / 5040.0);                           /* 1/7!  */
    p = fma(p, r, 1.0 / 720.0);                            /* 1/6!  */
    p = fma(p, r, 1.0 / 120.0);                            /* 1/5!  */
    p = fma(p, r, 1.0 / 24.0);                             /* 1/4!  */
    p = fma(p, r, 1.0 / 6.0);                              /* 1/3!  */
    p = fma(p, r, 0.5);                                    /* 1/2!  */
    p = fma(p, r, 1.0);                                    /* 1/1!  */
    p = fma(p, r, 1.0);                                    /* 1/0!  */
    int64_t ki = (int64_t)k;
    uint64_t scale_bits = (uint64_t)(ki + 1023) << 52;
    double scale;
    memcpy(&scale, &scale_bits, 8);
    return p * scale;
}

/* Gate S = sigma(Z) of [KPT] 6.1: 1 / (1 + e^(-z)) in fp64, rounded once to
 * fp32.  Outside |z| <= 700 the fp32 result is already exactly 0 or 1. */
float oracle_sigmoid_spec(float z)
{
    if (z > 700.0f) return 1.0f;
    if (z < -700.0f) return 0.0f;
    double t = oracle_exp_spec(-(double)z);
    double s = 1.0 / (1.0 + t);
    return (float)s;
}

/* ------------------------------------------------------ a1: router logits */

/* Z[t,e] = sum_i x[t,i] * W[e,i]; x [N,d] bf16, W [E,d] bf16, Z [N,E] fp32
 * ([KPT] 6.1 "the router produces logits Z"; [K1D] routing: bf16 router,
 * [N,2560] tokens to fp32 logits).  Products and the sum are formed in fp64
 * with i ascending and the sum is rounded once to fp32. */
void oracle_router_logits(const uint16_t *x, const uint16_t *w, float *z,
                          int64_t N, int32_t d, int32_t E)
{
    double *wd = (double *)malloc(sizeof(double) * (size_t)E * (size_t)d);
    for (int64_t j = 0; j < (int64_t)E * d; ++j) wd[j] = bf16_value(w[j]);
#pragma omp parallel
    {
        double *xd = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
        for (int64_t t = 0; t < N; ++t) {
            for (int32_t i = 0; i < d; ++i) xd[i] = bf16_value(x[t * d + i]);
            for (int32_t e = 0; e < E; ++e) {
                const double *we = wd + (int64_t)e * d;
                double acc = 0.0;
                for (int32_t i = 0; i < d; ++i) acc += xd[i] * we[i];
                z[t * E + e] = (float)acc;
            }
        }
        free(xd);
    }
    free(wd);
}

/* ------------------------------------------- a2: bias, top-K, gate, alpha */

typedef struct { uint32_t key; int32_t id; } keyed_t;

/* Descending key, then ascending id. */
static int cmp_desc_key_then_id(const void *pa, const void *pb)
{
    const keyed_t *a = (const keyed_t *)pa, *b = (const keyed_t *)pb;
    if (a->key != b->key) return a->key > b->key ? -1 : 1;
    return (a->id > b->id) - (a->id < b->id);
}

/* [KPT] 6.1: B = Z + 1 beta^T (fp32 add), I_t = Top-K(B_t,:), S = sigma(Z)
 * at the chosen ids from the raw logits, never renormalised ([K1D] routing
 * steps 1 and 2).  [KPT] 7.1: alpha_t = -Q_K(Z_t,: + beta), the negated
 * (K+1)-th largest biased score of the row.  Each row is fully sorted.
 * ids/gates are [N,K] in rank order; alpha may be NULL. */
void oracle_select(const float *z, const float *beta, int64_t N, int32_t E, int32_t K,
                   int32_t *ids, float *gates, float *alpha)
{
#pragma omp parallel
    {
        keyed_t *row = (keyed_t *)malloc(sizeof(keyed_t) * (size_t)E);
        float *b = (float *)malloc(sizeof(float) * (size_t)E);
#pragma omp for schedule(static)
        for (int64_t t = 0; t < N; ++t) {
            const float *zt = z + t * E;
            for (int32_t e = 0; e < E; ++e) {
                b[e] = beta ? zt[e] + beta[e] : zt[e];
                row[e].key = oracle_order_key(b[e]);
                row[e].id = e;
            }
            qsort(row, (size_t)E, sizeof(keyed_t), cmp_desc_key_then_id);
            for (int32_t k = 0; k < K; ++k) {
                ids[t * K + k] = row[k].id;
                gates[t * K + k] = oracle_sigmoid_spec(zt[row[k].id]);
            }
            if (alpha) alpha[t] = -b[row[K].id];
        }
        free(b);
        free(row);
    }
}

/* ------------------------------------------------ a3: counts, permutation */

/* Expert loads c_e ([KPT] 6.1, 6.2) and the grouping of the N*K routed slots
 * by expert: a stable counting sort of the flat slot index j = t*K + k by
 * key ids[j].  offsets is the exclusive prefix sum of counts (E+1 entries),
 * perm[p] = j for the p-th slot in grouped order, inv[j] = p (may be NULL). */
void oracle_permute(const int32_t *ids, int64_t N, int32_t E, int32_t K,
                    int32_t *counts, int64_t *offsets, int32_t *perm, int32_t *inv)
{
    int64_t NK = N * K;
    int64_t *cursor = (int64_t *)malloc(sizeof(int64_t) * (size_t)E);
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t j = 0; j < NK; ++j) counts[ids[j]] += 1;
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    for (int32_t e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t j = 0; j < NK; ++j) {
        int64_t p = cursor[ids[j]]++;
        perm[p] = (int32_t)j;
        if (inv) inv[j] = (int32_t)p;
    }
    free(cursor);
}

/* ------------------------------------------------ a4: column quantiles */

static int cmp_u32_desc(const void *pa, const void *pb)
{
    uint32_t a = *(const uint32_t *)pa, b = *(const uint32_t *)pb;
    return (a < b) - (a > b);
}

/* v_e = Q_m(Z_:,e + alpha): the (m+1)-th largest entry of the column after
 * the fp32 add of the token bias ([KPT] 1 for Q_m; 7.1 for the expert
 * update).  Full sort of each column.  alpha may be NULL (plain column). */
void oracle_column_quantiles(const float *z, const float *alpha, int64_t N, int32_t E,
                             int64_t m, float *v)
{
#pragma omp parallel
    {
        uint32_t *col = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int32_t e = 0; e < E; ++e) {
            for (int64_t t = 0; t < N; ++t) {
                float c = alpha ? z[t * E + e] + alpha[t] : z[t * E + e];
                col[t] = oracle_order_key(c);
            }
            qsort(col, (size_t)N, sizeof(uint32_t), cmp_u32_desc);
            uint32_t k = col[m];
            uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
            v[e] = bits_to_f32(u);
        }
        free(col);
    }
}

/* ------------------------------------------------ a5: EQB bias update */

/* [KPT] 7.1: beta_e <- -Q_r(Z_:,e + alpha), then the expert biases are
 * centred (their mean is subtracted); 7.2 shows the order: raw biases, then
 * the mean, then the centred biases. */
void oracle_eqb_bias(const float *v, int32_t E, float *beta_out)
{
    double sum = 0.0;
    for (int32_t e = 0; e < E; ++e) sum += (double)(-v[e]);
    float mean = (float)(sum / (double)E);
    for (int32_t e = 0; e < E; ++e) beta_out[e] = (-v[e]) - mean;
}

/* ------------------------------- the pages' radix selection, step by step */

/* Exact selection by radix digits as in [KPT] 7.3: keys are split into
 * `ndigits` digits of base `radix` (most significant first).  For each digit
 * a histogram of that digit is built over the keys whose higher digits match
 * the prefix chosen so far; bins are scanned from the top until the running
 * count passes the target rank; that bin fixes the digit.  When `nchunks` > 1
 * the keys are the concatenation of chunks (ranks) of the given sizes and
 * each chunk's histogram is summed, which is the all-reduce of 7.3.
 * Returns the selected key (the (m+1)-th largest).  hist_out (nullable,
 * ndigits*radix) receives each pass's summed histogram; bins_out (nullable,
 * ndigits) the chosen bin of each pass. */
uint64_t oracle_radix_select(const uint64_t *keys, const int64_t *chunk_sizes, int32_t nchunks,
                             int64_t m, int64_t radix, int32_t ndigits,
                             int64_t *hist_out, int64_t *bins_out)
{
    int64_t *hist = (int64_t *)malloc(sizeof(int64_t) * (size_t)radix);
    uint64_t place = 1;
    for (int32_t j = 1; j < ndigits; ++j) place *= (uint64_t)radix;
    uint64_t prefix = 0;        /* value of the digits fixed so far          */
    uint64_t span = place * (uint64_t)radix; /* keys matching the prefix lie */
    int64_t rank = m;           /* in [prefix, prefix + span)                */
    for (int32_t j = 0; j < ndigits; ++j) {
        for (int64_t b = 0; b < radix; ++b) hist[b] = 0;
        const uint64_t *base = keys;
        for (int32_t c = 0; c < nchunks; ++c) {            /* one rank each  */
            for (int64_t i = 0; i < chunk_sizes[c]; ++i) {
                uint64_t k = base[i];
                if (k >= prefix && k - prefix < span)
                    hist[(k / place) % (uint64_t)radix] += 1;  /* summed     */
            }
            base += chunk_sizes[c];
        }
        if (hist_out) memcpy(hist_out + (int64_t)j * radix, hist, sizeof(int64_t) * (size_t)radix);
        int64_t b = radix - 1;
        while (b > 0 && hist[b] <= rank) { rank -= hist[b]; --b; } /* from top */
        if (bins_out) bins_out[j] = b;
        prefix += (uint64_t)b * place;
        span = place;
        place /= (uint64_t)radix;
    }
    free(hist);
    return prefix;
}

/* ------------------------------------- bf16 keys, as on the pages (7.3) */

/* The bf16 value nearest to v (ties to the even mantissa), as its 16 bits.
 * Inputs are finite (or infinite); an fp32 value past the largest bf16
 * rounds to infinity, as IEEE rounding does. */
uint16_t oracle_bf16_round(float v)
{
    uint32_t u = f32_to_bits(v);
    uint32_t lsb = (u >> 16) & 1u;              /* last kept bit: ties go to even */
    uint32_t r = u + 0x7fffu + lsb;            /* add just under half, or half */
    return (uint16_t)(r >> 16);
}

/* Order-preserving 16-bit key of a bf16 pattern: the same total order as
 * the fp32 key (negative: all 16 bits flipped; non-negative: sign bit set). */
uint16_t oracle_bf16_key(uint16_t b)
{
    return (b & 0x8000u) ? (uint16_t)(~b & 0xffffu) : (uint16_t)(b | 0x8000u);
}

static int cmp_u16_desc(const void *pa, const void *pb)
{
    uint16_t a = *(const uint16_t *)pa, b = *(const uint16_t *)pb;
    return (a < b) - (a > b);
}

/* [KPT] 7.3 with bfloat16 keys: per column, C = bf16(Z + alpha) (the fp32
 * sum rounded once to bf16), and v_e = the (m+1)-th largest of C in the
 * total order of the keys, returned as its float value.  The plain
 * definition: round, sort, index. */
void oracle_column_quantiles_bf16(const float *z, const float *alpha, int64_t N, int32_t E,
                                  int64_t m, float *v)
{
#pragma omp parallel
    {
        uint16_t *col = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int32_t e = 0; e < E; ++e) {
            for (int64_t t = 0; t < N; ++t) {
                float c = alpha ? z[t * E + e] + alpha[t] : z[t * E + e];
                col[t] = oracle_bf16_key(oracle_bf16_round(c));
            }
            qsort(col, (size_t)N, sizeof(uint16_t), cmp_u16_desc);
            uint16_t k = col[m];
            uint16_t b = (k & 0x8000u) ? (uint16_t)(k & 0x7fffu) : (uint16_t)(~k & 0xffffu);
            v[e] = (float)bf16_value(b);
        }
        free(col);
    }
}

/* ------------------------------------- Load-Error Injection ([KPT] 8) */

/* tanh from the gate's exp: tanh(x) = (1 - e^(-2x)) / (1 + e^(-2x)) for
 * x >= 0, in fp64 IEEE operations (x is a norm, so never negative here). */
double oracle_tanh_spec(double x)
{
    if (x > 350.0) return 1.0;                 /* e^(-2x) < 2^-1000: exactly 1 */
    double t = oracle_exp_spec(-2.0 * x);
    return (1.0 - t) / (1.0 + t);
}

/* The per-expert injection of [KPT] 8 for one microbatch of N tokens:
 *   f_e = c_e / (K N / E),  rho_e = f_e - 1,  xi = max_e |rho_e| / tau,
 *   delta_e = lambda * (tanh(xi) / xi) * rho_e   (the factor is 1 at xi = 0),
 * all in fp64, delta rounded once to fp32.  Every token's score gradient
 * then receives delta: G[t][e] += delta_e in fp32 (g may be NULL to get
 * delta only). */
void oracle_lei_delta(const int32_t *counts, int64_t N, int32_t E, int32_t K, double lambda,
                      double tau, float *delta)
{
    double target = (double)K * (double)N / (double)E;
    double xi = 0.0;
    for (int32_t e = 0; e < E; ++e) {
        double rho = (double)counts[e] / target - 1.0;
        double a = rho < 0.0 ? -rho : rho;
        if (a > xi) xi = a;
    }
    xi = xi / tau;
    double factor = xi == 0.0 ? 1.0 : oracle_tanh_spec(xi) / xi;
    for (int32_t e = 0; e < E; ++e) {
        double rho = (double)counts[e] / target - 1.0;
        delta[e] = (float)(lambda * factor * rho);
    }
}

void oracle_lei_inject(const int32_t *counts, int64_t N, int32_t E, int32_t K, double lambda,
                       double tau, float *g)
{
    float *delta = (float *)malloc(sizeof(float) * (size_t)E);
    oracle_lei_delta(counts, N, E, K, lambda, tau, delta);
    for (int64_t t = 0; t < N; ++t)
        for (int32_t e = 0; e < E; ++e) g[t * E + e] = g[t * E + e] + delta[e];
    free(delta);
}

/* The chain rule to the router logits ([KPT] 8, numerical check):
 * dL/dZ = dL/dS * sigma(Z) (1 - sigma(Z)), with sigma in fp64 from the
 * gate's exp, the product in fp64, rounded once to fp32. */
void oracle_score_grad_to_logits(const float *z, const float *gs, int64_t n, float *gz)
{
    for (int64_t i = 0; i < n; ++i) {
        double s;                                 /* saturates as the gate does */
        if (z[i] > 700.0f) s = 1.0;
        else if (z[i] < -700.0f) s = 0.0;
        else s = 1.0 / (1.0 + oracle_exp_spec(-(double)z[i]));
        gz[i] = (float)((double)gs[i] * (s * (1.0 - s)));
    }
}

/* ------------------------------------------- the experts ([KPT] 6.1) */

/* The bf16 value nearest to the real number v (ties to the even last
 * significand bit), as its 16 bits.  v is rounded once, straight from fp64:
 * an 8-bit significand for normal values, a fixed step of 2^-133 below
 * 2^-126; values at or past the midpoint to 2^128 become infinity. */
uint16_t oracle_bf16_round_f64(double v)
{
    if (v == 0.0) return signbit(v) ? 0x8000u : 0x0000u;
    const double a = fabs(v);
    double r;
    if (a < ldexp(1.0, -126)) {
        r = ldexp(nearbyint(ldexp(a, 133)), -133);
    } else {
        int e;
        const double m = frexp(a, &e);           /* a = m 2^e, 0.5 <= m < 1 */
        r = ldexp(nearbyint(ldexp(m, 8)), e - 8);
    }
    uint16_t b;
    if (r >= ldexp(1.0, 128)) b = 0x7f80u;
    else b = (uint16_t)(f32_to_bits((float)r) >> 16);   /* r has at most 8 significant bits */
    return (uint16_t)(signbit(v) ? (b | 0x8000u) : b);
}

/* SiLU(g) = g sigma(g) with sigma(g) = 1 / (1 + e^(-g)) in fp64, e^x from
 * exp_spec; for g <= -700 the product is 0 (-0 for negative g). */
double oracle_silu_spec(double g)
{
    if (g <= -700.0) return -0.0;
    return g * (1.0 / (1.0 + oracle_exp_spec(-g)));
}

/* One SwiGLU expert of [K1D] ("two projections d -> F form SiLU(gate) x up,
 * then F -> d") applied to one token x [d]:
 *   g_j = sum_i x_i Wg[j,i],  u_j = sum_i x_i Wu[j,i]   (fp64, i ascending)
 *   h_j = bf16(SiLU(g_j) u_j)                          (the activation the
 *                                                       down projection reads)
 *   Y_c = sum_j h_j Wd[c,j]                              (fp64, j ascending)
 * wgu [2F, d]: rows 0..F-1 are Wg, rows F..2F-1 are Wu; wd [d, F].
 * h [F] receives the bf16 bits; mag[c] += scale * sum_j |h_j Wd[c,j]|. */
static void swiglu_expert(const uint16_t *x, const uint16_t *wgu, const uint16_t *wd, int32_t d,
                          int32_t F, uint16_t *h, double *hv, double *y, double *mag,
                          double scale)
{
    for (int32_t j = 0; j < F; ++j) {
        const uint16_t *wg = wgu + (int64_t)j * d, *wu = wgu + (int64_t)(F + j) * d;
        double g = 0.0, u = 0.0;
        for (int32_t i = 0; i < d; ++i) {
            const double xi = bf16_value(x[i]);
            g += xi * bf16_value(wg[i]);
            u += xi * bf16_value(wu[i]);
        }
        h[j] = oracle_bf16_round_f64(oracle_silu_spec(g) * u);
        hv[j] = bf16_value(h[j]);
    }
    for (int32_t c = 0; c < d; ++c) {
        const uint16_t *w = wd + (int64_t)c * F;
        double acc = 0.0, m = 0.0;
        for (int32_t j = 0; j < F; ++j) {
            const double t = hv[j] * bf16_value(w[j]);
            acc += t;
            m += fabs(t);
        }
        y[c] = acc;
        if (mag) mag[c] += scale * m;
    }
}

/* The MoE output of [KPT] 6.1: y_t = f_shared(x_t) + sum_k S_t,k f_e(x_t)
 * over the token's K routed experts e = ids[t,k] with their gates S (the
 * unbiased sigmoid scores, not renormalised).  x [N,d], wgu [E,2F,d],
 * wd [E,d,F] (bf16 bits); the shared expert (wgu_s [2F,d], wd_s [d,F]) is
 * left out when wgu_s is NULL.  The sum is taken in fp64 in the order
 * shared, k = 0..K-1, and rounded once to fp32 into y [N,d].
 * Optional outputs: h [N*K, F] the routed activations in slot order t*K+k,
 * h_s [N, F] the shared ones, mag [N,d] = sum of |each product| weighted by
 * |S| (the scale of the rounding error of any summation order). */
void oracle_expert_ffn(const uint16_t *x, const int32_t *ids, const float *gates,
                       const uint16_t *wgu, const uint16_t *wd, const uint16_t *wgu_s,
                       const uint16_t *wd_s, int64_t N, int32_t d, int32_t F, int32_t E,
                       int32_t K, uint16_t *h, uint16_t *h_s, float *y, double *mag)
{
    #pragma omp parallel
    {
        uint16_t *hb = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)F);
        double *hv = (double *)malloc(sizeof(double) * (size_t)F);
        double *ye = (double *)malloc(sizeof(double) * (size_t)d);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < N; ++t) {
            const uint16_t *xt = x + t * d;
            double *mt = mag ? mag + t * d : NULL;
            if (mt) memset(mt, 0, sizeof(double) * (size_t)d);
            for (int32_t c = 0; c < d; ++c) acc[c] = 0.0;
            if (wgu_s) {
                swiglu_expert(xt, wgu_s, wd_s, d, F, hb, hv, ye, mt, 1.0);
                if (h_s) memcpy(h_s + t * F, hb, sizeof(uint16_t) * (size_t)F);
                for (int32_t c = 0; c < d; ++c) acc[c] += ye[c];
            }
            for (int32_t k = 0; k < K; ++k) {
                const int32_t e = ids[t * K + k];
                if (e < 0 || e >= E) abort();
                const double s = (double)gates[t * K + k];
                swiglu_expert(xt, wgu + (int64_t)e * 2 * F * d, wd + (int64_t)e * d * F, d, F, hb,
                              hv, ye, mt, fabs(s));
                if (h) memcpy(h + (t * K + k) * F, hb, sizeof(uint16_t) * (size_t)F);
                for (int32_t c = 0; c < d; ++c) acc[c] += s * ye[c];
            }
            for (int32_t c = 0; c < d; ++c) y[t * d + c] = (float)acc[c];
        }
        free(hb); free(hv); free(ye); free(acc);
    }
}

/* ------------------------------------------------ measurements */

/* MaxVio of [KPT] 6.2: max_e c_e / (K*N/E) - 1. */
double oracle_maxvio(const int32_t *counts, int32_t E, int64_t N, int32_t K)
{
    double target = (double)K * (double)N / (double)E;
    double worst = -1.0e300;
    for (int32_t e = 0; e < E; ++e) {
        double r = (double)counts[e] / target - 1.0;
        if (r > worst) worst = r;
    }
    return worst;
}

/* Intervention rate of [KPT] 9: mean over tokens of 1 - |I^u_t and I_t| / K,
 * with I^u the router's own top-K (no bias) and I the routed top-K. */
double oracle_intervention_rate(const int32_t *ids_routed, const int32_t *ids_unbiased,
                                int64_t N, int32_t K)
{
    double acc = 0.0;
    for (int64_t t = 0; t < N; ++t) {
        int32_t overlap = 0;
        for (int32_t a = 0; a < K; ++a)
            for (int32_t b = 0; b < K; ++b)
                overlap += ids_routed[t * K + a] == ids_unbiased[t * K + b];
        acc += 1.0 - (double)overlap / (double)K;
    }
    return acc / (double)N;
}

/* The integer at the heart of the intervention rate of [KPT] 9: the total,
 * over tokens, of |I^u_t and I_t|, the routed experts that are also among
 * the router's own top-K.  The ids of one token are distinct, so counting
 * equal pairs counts the intersection.  rate = 1 - overlap / (N K). */
int64_t oracle_intervention_overlap(const int32_t *ids_routed, const int32_t *ids_unbiased,
                                    int64_t N, int32_t K)
{
    int64_t total = 0;
    for (int64_t t = 0; t < N; ++t)
        for (int32_t a = 0; a < K; ++a)
            for (int32_t b = 0; b < K; ++b)
                total += ids_routed[t * K + a] == ids_unbiased[t * K + b];
    return total;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
