/*
 * moe_oracle.c -- plain fp64 CPU oracle for the fused MoE layer forward.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this library.  It shares no source, header, table or
 * helper with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes (the layer sketched by "Decoding the Skew: Distribution-Aware
 * MoE Inference with Adaptive Kernel Dispatch", abstract: a router whose runtime
 * distribution decides the shapes of sparse expert GEMMs; and by "GC-MoE:
 * Overlapping Expert-Parallel Token Dispatch with FP8/FP4 Grouped GEMM via CUDA
 * Green Contexts", abstract: grouped expert GEMMs with a fused SwiGLU, optional
 * shared experts, then a combine step):
 *
 *   1. router logits   L[t,e] = sum_c x[t,c] * Wg[e,c] + b[e]            (fp64)
 *   2. top-k           the k largest fp32 logits of a token, in descending
 *                      order, ties to the lower expert index; gates are the
 *                      softmax over those k logits                        (fp64)
 *   3. histogram       counts[e] = #{pairs routed to e}; offsets = exclusive
 *                      scan; pair q = t*k + j; stable expert-major order
 *                      pos(q) = offsets[e] + #{q' < q routed to e};
 *                      perm[pos] = q, inv_perm[q] = pos
 *   4. expert FFN      per token t and per j: e = idx[t,j];
 *                      h = silu(W1[e] x_t) * (W3[e] x_t), z = W2[e] h,
 *                      y_t += w_j * z; plus the shared expert with gate 1.
 *                      silu(g) = g / (1 + exp(-g)).  Every value is fp64 and
 *                      nothing is rounded in between.
 *
 * Steps the pages leave open and the reading taken here: gates are the softmax
 * over the k selected logits; ties go to the lower expert index; a NaN logit
 * ranks below every number; the order inside an expert's segment is ascending
 * pair id; W1 is the gate projection and W3 the up projection; the shared
 * expert's gate is 1.
 *
 * bf16 inputs arrive as raw 16-bit patterns; a bf16 value is the fp32 whose top
 * 16 bits are that pattern, so the widening below is exact.
 *
 * Every entry point returns 0 on success, ORACLE_EARG on a bad argument,
 * ORACLE_ERANGE when an expert index is out of [0, E) or an expert's weights
 * are missing, ORACLE_ENOMEM when a scratch allocation fails.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_OK 0
#define ORACLE_EARG (-1)
#define ORACLE_ERANGE (-2)
#define ORACLE_ENOMEM (-3)

static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float v;
    memcpy(&v, &u, sizeof v);
    return (double)v;
}

int oracle_default_threads(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* Step 1: router logits in fp64.  x [T,d], Wg [E,d], bias [E] or NULL, L [T,E]. */
int oracle_router_logits(const uint16_t *x, const uint16_t *Wg, const float *bias,
                         int64_t T, int64_t d, int64_t E, double *L)
{
    if (T < 0 || d <= 0 || E <= 0 || (T > 0 && (!x || !Wg || !L)))
        return ORACLE_EARG;
    for (int64_t t = 0; t < T; t++) {
        for (int64_t e = 0; e < E; e++) {
            double s = 0.0;
            for (int64_t c = 0; c < d; c++)
                s += bf16_value(x[t * d + c]) * bf16_value(Wg[e * d + c]);
            if (bias)
                s += (double)bias[e];
            L[t * E + e] = s;
        }
    }
    return ORACLE_OK;
}

/* a ranks before b: larger logit first, NaN below every number, then lower index. */
static int ranks_before(float a, int64_t ia, float b, int64_t ib)
{
    int an = isnan(a), bn = isnan(b);
    if (an != bn)
        return bn;          /* the non-NaN one ranks first */
    if (!an && a != b)
        return a > b;
    return ia < ib;
}

/* Step 2: top-k of fp32 logits L [T,E] -> idx [T,k] (descending), w [T,k] (fp64). */
int oracle_topk(const float *L, int64_t T, int64_t E, int64_t k, int32_t *idx, double *w)
{
    if (T < 0 || E <= 0 || k < 1 || k > E || (T > 0 && (!L || !idx || !w)))
        return ORACLE_EARG;
    unsigned char *taken = (unsigned char *)malloc((size_t)E);
    if (!taken)
        return ORACLE_ENOMEM;
    for (int64_t t = 0; t < T; t++) {
        const float *row = L + t * E;
        memset(taken, 0, (size_t)E);
        /* selection: k rounds, each picks the best expert not yet taken */
        for (int64_t j = 0; j < k; j++) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; e++) {
                if (taken[e])
                    continue;
                if (best < 0 || ranks_before(row[e], e, row[best], best))
                    best = e;
            }
            taken[best] = 1;
            idx[t * k + j] = (int32_t)best;
        }
        /* gates: softmax over the k selected logits, shifted by the largest */
        double top = (double)row[idx[t * k]];
        double z = 0.0;
        for (int64_t j = 0; j < k; j++)
            z += exp((double)row[idx[t * k + j]] - top);
        for (int64_t j = 0; j < k; j++)
            w[t * k + j] = exp((double)row[idx[t * k + j]] - top) / z;
    }
    free(taken);
    return ORACLE_OK;
}

/* Step 3: histogram, offsets [E+1], and the stable expert-major permutation. */
int oracle_permutation(const int32_t *idx, int64_t T, int64_t k, int64_t E,
                       int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm)
{
    if (T < 0 || k < 1 || E <= 0 || !counts || !offsets || (T > 0 && (!idx || !perm || !inv_perm)))
        return ORACLE_EARG;
    int64_t P = T * k;
    for (int64_t e = 0; e < E; e++)
        counts[e] = 0;
    for (int64_t q = 0; q < P; q++) {
        if (idx[q] < 0 || idx[q] >= E)
            return ORACLE_ERANGE;
        counts[idx[q]]++;
    }
    offsets[0] = 0;
    for (int64_t e = 0; e < E; e++)
        offsets[e + 1] = offsets[e] + counts[e];
    int32_t *next = (int32_t *)malloc((size_t)E * sizeof(int32_t));
    if (!next)
        return ORACLE_ENOMEM;
    for (int64_t e = 0; e < E; e++)
        next[e] = offsets[e];
    for (int64_t q = 0; q < P; q++) {      /* ascending q keeps each segment stable */
        int32_t pos = next[idx[q]]++;
        perm[pos] = (int32_t)q;
        inv_perm[q] = pos;
    }
    free(next);
    return ORACLE_OK;
}

/* One SwiGLU expert applied to one token, scaled by gate and added into y:
 * y += gate * W2 (silu(W1 x) * (W3 x)).  W1, W3 [f,d]; W2 [d,f]; h has f doubles. */
static void expert_ffn_add(const uint16_t *W1, const uint16_t *W3, const uint16_t *W2,
                           const uint16_t *xt, int64_t d, int64_t f, double gate,
                           double *h, double *y)
{
    for (int64_t r = 0; r < f; r++) {
        double g = 0.0, u = 0.0;
        for (int64_t c = 0; c < d; c++) {
            double xc = bf16_value(xt[c]);
            g += bf16_value(W1[r * d + c]) * xc;
            u += bf16_value(W3[r * d + c]) * xc;
        }
        h[r] = g / (1.0 + exp(-g)) * u;
    }
    for (int64_t c = 0; c < d; c++) {
        double z = 0.0;
        for (int64_t r = 0; r < f; r++)
            z += bf16_value(W2[c * f + r]) * h[r];
        y[c] += gate * z;
    }
}

typedef struct {
    const uint16_t *x;
    const uint16_t *const *W1, *const *W3, *const *W2;   /* per-expert pointers */
    int64_t d, f, E, k;
    const int32_t *idx;
    const double *w;
    const uint16_t *Ws1, *Ws3, *Ws2;
    int64_t fs;
    const int64_t *tokens;    /* rows of x to evaluate, or NULL for 0..ntok-1 */
    int64_t ntok;
    double *out;              /* [ntok, d] */
    int nthreads, tid;
    int status;
} ffn_job;

static void *ffn_worker(void *arg)
{
    ffn_job *J = (ffn_job *)arg;
    int64_t hlen = J->f > J->fs ? J->f : J->fs;
    double *h = (double *)malloc((size_t)(hlen > 0 ? hlen : 1) * sizeof(double));
    if (!h) {
        J->status = ORACLE_ENOMEM;
        return NULL;
    }
    for (int64_t i = J->tid; i < J->ntok; i += J->nthreads) {
        int64_t t = J->tokens ? J->tokens[i] : i;
        const uint16_t *xt = J->x + t * J->d;
        double *y = J->out + i * J->d;
        for (int64_t c = 0; c < J->d; c++)
            y[c] = 0.0;
        for (int64_t j = 0; j < J->k; j++) {
            int32_t e = J->idx[t * J->k + j];
            if (e < 0 || e >= J->E || !J->W1[e] || !J->W3[e] || !J->W2[e]) {
                J->status = ORACLE_ERANGE;
                free(h);
                return NULL;
            }
            expert_ffn_add(J->W1[e], J->W3[e], J->W2[e], xt, J->d, J->f, J->w[t * J->k + j], h, y);
        }
        if (J->fs > 0)
            expert_ffn_add(J->Ws1, J->Ws3, J->Ws2, xt, J->d, J->fs, 1.0, h, y);
    }
    free(h);
    return NULL;
}

/* Step 4: the routed (and shared) expert FFNs of the listed tokens.
 * x [T,d]; W1[e], W3[e] -> [f,d]; W2[e] -> [d,f] (NULL for experts no listed
 * token uses); idx [T,k]; w [T,k]; Ws* may be NULL when fs == 0;
 * tokens: ntok row ids of x (NULL means rows 0..ntok-1); out [ntok,d].
 * Tokens are split over nthreads threads (<= 0: one per online core); each
 * token is evaluated by one thread in a fixed order, so the result does not
 * depend on the thread count. */
int oracle_moe_ffn(const uint16_t *x,
                   const uint16_t *const *W1, const uint16_t *const *W3, const uint16_t *const *W2,
                   int64_t d, int64_t f, int64_t E,
                   const int32_t *idx, const double *w, int64_t k,
                   const uint16_t *Ws1, const uint16_t *Ws3, const uint16_t *Ws2, int64_t fs,
                   const int64_t *tokens, int64_t ntok, double *out, int nthreads)
{
    if (d <= 0 || f <= 0 || E <= 0 || k < 1 || ntok < 0 || fs < 0)
        return ORACLE_EARG;
    if (ntok == 0)
        return ORACLE_OK;
    if (!x || !W1 || !W3 || !W2 || !idx || !w || !out || (fs > 0 && (!Ws1 || !Ws3 || !Ws2)))
        return ORACLE_EARG;
    if (nthreads <= 0)
        nthreads = oracle_default_threads();
    if (nthreads > ntok)
        nthreads = (int)ntok;
    ffn_job *jobs = (ffn_job *)calloc((size_t)nthreads, sizeof(ffn_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return ORACLE_ENOMEM;
    }
    int started = 0;
    for (int i = 0; i < nthreads; i++) {
        ffn_job J = {x, W1, W3, W2, d, f, E, k, idx, w, Ws1, Ws3, Ws2, fs,
                     tokens, ntok, out, nthreads, i, ORACLE_OK};
        jobs[i] = J;
    }
    for (int i = 1; i < nthreads; i++) {
        if (pthread_create(&th[i], NULL, ffn_worker, &jobs[i]) != 0)
            break;
        started = i;
    }
    /* Threads that could not be started are run on this thread instead. */
    for (int i = started + 1; i < nthreads; i++)
        ffn_worker(&jobs[i]);
    ffn_worker(&jobs[0]);
    for (int i = 1; i <= started; i++)
        pthread_join(th[i], NULL);
    int status = ORACLE_OK;
    for (int i = 0; i < nthreads; i++)
        if (jobs[i].status != ORACLE_OK)
            status = jobs[i].status;
    free(jobs);
    free(th);
    return status;
}

/* ------------------------------------------------------------------------
 * FP8 block-scaled variant (GC-MoE, abstract: an FP8 MoE operator with
 * block-scaled MMA and requantisation; the workload table fixes e4m3 codes
 * with 1x128 activation blocks and 128x128 weight blocks).
 *
 * e4m3 (OCP 8-bit floating point, E4M3 variant): 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits; no infinities; exponent field 15 with mantissa
 * 7 is NaN; largest finite value 1.75 * 2^8 = 448; normal values
 * (1 + m/8) * 2^(e-7) for e = 1..15; subnormals (m/8) * 2^-6.
 *
 * Readings taken: a value is encoded by round-to-nearest, ties to the even
 * code, and magnitudes past 448 saturate to 448.  A block's scale is the
 * smallest power of two s with amax / s <= 448 (amax = 0 gives s = 1), so
 * v / s is exact and the dequantised value of code q is decode(q) * s.
 * ------------------------------------------------------------------------ */

double oracle_e4m3_decode(uint8_t code)
{
    int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Nearest e4m3 code to v (ties to the code with an even mantissa), saturating to 448. */
uint8_t oracle_e4m3_encode(double v)
{
    uint8_t sign = (v < 0 || (v == 0 && signbit(v))) ? 0x80 : 0;
    double a = fabs(v);
    if (isnan(v))
        return 0x7F;
    if (a >= 448.0)
        return sign | 0x7E;   /* 448: exponent field 15, mantissa 6 */
    /* Walk the 127 finite non-negative codes in increasing order; keep the nearest. */
    uint8_t best = 0;
    double best_err = a;      /* code 0 is +0 */
    for (int c = 1; c <= 0x7E; c++) {
        double err = fabs(oracle_e4m3_decode((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = (uint8_t)c;
            best_err = err;
        }
    }
    return sign | best;
}

/* The same rounding computed from the value's binary exponent instead of a
 * walk over every code (the block quantisers use this one; a test checks it
 * against oracle_e4m3_encode on every code, every midpoint and random values). */
uint8_t oracle_e4m3_encode_fast(double v)
{
    uint8_t sign = (v < 0 || (v == 0 && signbit(v))) ? 0x80 : 0;
    double a = fabs(v);
    if (isnan(v))
        return 0x7F;
    if (a >= 448.0)
        return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {                 /* subnormal range: steps of 2^-9 */
        double m = nearbyint(a * 512.0);       /* ties to even (default rounding mode) */
        return sign | (uint8_t)m;              /* m == 8 is the smallest normal, code 0x08 */
    }
    int e;
    double frac = frexp(a, &e);               /* a = frac * 2^e, frac in [0.5, 1) */
    int ex = e - 1;                            /* a = (2 frac) * 2^ex, 2 frac in [1, 2) */
    double m = nearbyint((2.0 * frac - 1.0) * 8.0);
    if (m == 8.0) {
        m = 0.0;
        ex += 1;
    }
    int field = ex + 7;
    if (field > 15 || (field == 15 && m > 6.0))
        return sign | 0x7E;
    return sign | (uint8_t)((field << 3) | (int)m);
}

static double g_e4m3[256];
static pthread_once_t g_e4m3_once = PTHREAD_ONCE_INIT;
static void e4m3_table_init(void)
{
    for (int c = 0; c < 256; c++)
        g_e4m3[c] = oracle_e4m3_decode((uint8_t)c);
}
static double e4m3_value(uint8_t c)
{
    pthread_once(&g_e4m3_once, e4m3_table_init);
    return g_e4m3[c];
}

/* Smallest power of two s with amax / s <= 448 (amax = 0: s = 1), kept in
 * the range of a UE8M0 scale, 2^-127 .. 2^127: the block-scaled MMA takes
 * its scales in that format, so a block whose amax lies below 448 * 2^-128
 * gets the scale 2^-127 (its codes then sit low in the e4m3 range). */
double oracle_fp8_block_scale(double amax)
{
    if (!(amax > 0))
        return 1.0;
    int e = 0;
    while (amax > ldexp(448.0, e) && e < 127)
        e++;
    while (amax <= ldexp(448.0, e - 1) && e > -127)
        e--;
    return ldexp(1.0, e);
}

/* 1 x 128 blocks along each row: x [R, C] bf16 -> q [R, C], s [R, C/128]. C % 128 == 0. */
int oracle_quantize_rows_fp8(const uint16_t *x, int64_t R, int64_t C, uint8_t *q, double *s)
{
    if (R < 0 || C <= 0 || C % 128 || (R > 0 && (!x || !q || !s)))
        return ORACLE_EARG;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t b = 0; b < C / 128; b++) {
            double amax = 0;
            for (int64_t c = 0; c < 128; c++)
                amax = fmax(amax, fabs(bf16_value(x[r * C + b * 128 + c])));
            double sc = oracle_fp8_block_scale(amax);
            s[r * (C / 128) + b] = sc;
            for (int64_t c = 0; c < 128; c++)
                q[r * C + b * 128 + c] = oracle_e4m3_encode_fast(bf16_value(x[r * C + b * 128 + c]) / sc);
        }
    }
    return ORACLE_OK;
}

/* 128 x 128 blocks: W [R, C] bf16 -> q [R, C], s [R/128, C/128].  R, C % 128 == 0. */
int oracle_quantize_blocks_fp8(const uint16_t *W, int64_t R, int64_t C, uint8_t *q, double *s)
{
    if (R <= 0 || C <= 0 || R % 128 || C % 128 || !W || !q || !s)
        return ORACLE_EARG;
    for (int64_t br = 0; br < R / 128; br++) {
        for (int64_t bc = 0; bc < C / 128; bc++) {
            double amax = 0;
            for (int64_t r = 0; r < 128; r++)
                for (int64_t c = 0; c < 128; c++)
                    amax = fmax(amax, fabs(bf16_value(W[(br * 128 + r) * C + bc * 128 + c])));
            double sc = oracle_fp8_block_scale(amax);
            s[br * (C / 128) + bc] = sc;
            for (int64_t r = 0; r < 128; r++)
                for (int64_t c = 0; c < 128; c++) {
                    int64_t i = (br * 128 + r) * C + bc * 128 + c;
                    q[i] = oracle_e4m3_encode_fast(bf16_value(W[i]) / sc);
                }
        }
    }
    return ORACLE_OK;
}

/* The first half of one FP8 SwiGLU expert on one token (fp64 on dequantised
 * values): g = W1^ x^, u = W3^ x^, h = silu(g) * u, then h requantised in
 * 1 x 128 blocks along f -> codes hq [f] and scales sh [f/128].
 * W1q/W3q [f,d] with scales [f/128, d/128]; xq [d] with sx [d/128]; h is
 * scratch of f doubles. */
static void expert_h_fp8(const uint8_t *W1q, const double *s1, const uint8_t *W3q, const double *s3,
                         const uint8_t *xq, const double *sx, int64_t d, int64_t f, double *h, uint8_t *hq,
                         double *sh)
{
    const int64_t db = d / 128, fb = f / 128;
    for (int64_t r = 0; r < f; r++) {
        double g = 0.0, u = 0.0;
        for (int64_t c = 0; c < d; c++) {
            double xc = e4m3_value(xq[c]) * sx[c / 128];
            g += e4m3_value(W1q[r * d + c]) * s1[(r / 128) * db + c / 128] * xc;
            u += e4m3_value(W3q[r * d + c]) * s3[(r / 128) * db + c / 128] * xc;
        }
        h[r] = g / (1.0 + exp(-g)) * u;
    }
    for (int64_t b = 0; b < fb; b++) {          /* requantise h in 1 x 128 blocks */
        double amax = 0;
        for (int64_t r = 0; r < 128; r++)
            amax = fmax(amax, fabs(h[b * 128 + r]));
        double sc = oracle_fp8_block_scale(amax);
        sh[b] = sc;
        for (int64_t r = 0; r < 128; r++)
            hq[b * 128 + r] = oracle_e4m3_encode_fast(h[b * 128 + r] / sc);
    }
}

/* One FP8 SwiGLU expert on one token: h^ from expert_h_fp8, then
 * y += gate * W2^ h^ (W2q [d,f] with scales [d/128, f/128]).  h, hq, sh are
 * scratch of f doubles, f bytes and f/128 doubles. */
static void expert_ffn_fp8_add(const uint8_t *W1q, const double *s1, const uint8_t *W3q, const double *s3,
                               const uint8_t *W2q, const double *s2, const uint8_t *xq, const double *sx,
                               int64_t d, int64_t f, double gate, double *h, uint8_t *hq, double *sh, double *y)
{
    const int64_t fb = f / 128;
    expert_h_fp8(W1q, s1, W3q, s3, xq, sx, d, f, h, hq, sh);
    for (int64_t r = 0; r < f; r++)
        h[r] = e4m3_value(hq[r]) * sh[r / 128];
    for (int64_t c = 0; c < d; c++) {
        double z = 0.0;
        for (int64_t r = 0; r < f; r++)
            z += e4m3_value(W2q[c * f + r]) * s2[(c / 128) * fb + r / 128] * h[r];
        y[c] += gate * z;
    }
}

/* The requantised h of one FP8 expert on one token (the intermediate the
 * down projection reads): codes hq [f] and scales sh [f/128].  W1q/W3q [f,d]
 * with s1/s3 [f/128, d/128]; xq [d] with sx [d/128]; d, f multiples of 128. */
int oracle_expert_h_fp8(const uint8_t *W1q, const double *s1, const uint8_t *W3q, const double *s3,
                        const uint8_t *xq, const double *sx, int64_t d, int64_t f, uint8_t *hq, double *sh)
{
    if (d <= 0 || f <= 0 || d % 128 || f % 128 || !W1q || !s1 || !W3q || !s3 || !xq || !sx || !hq || !sh)
        return ORACLE_EARG;
    double *h = (double *)malloc((size_t)f * sizeof(double));
    if (!h)
        return ORACLE_ENOMEM;
    expert_h_fp8(W1q, s1, W3q, s3, xq, sx, d, f, h, hq, sh);
    free(h);
    return ORACLE_OK;
}

typedef struct {
    const uint8_t *xq;
    const double *sx;
    const uint8_t *const *W1q, *const *W3q, *const *W2q;
    const double *const *s1, *const *s3, *const *s2;
    int64_t d, f, E, k;
    const int32_t *idx;
    const double *w;
    const uint8_t *Ws1q, *Ws3q, *Ws2q;
    const double *ss1, *ss3, *ss2;
    int64_t fs;
    const int64_t *tokens;
    int64_t ntok;
    double *out;
    int nthreads, tid;
    int status;
} ffn8_job;

static void *ffn8_worker(void *arg)
{
    ffn8_job *J = (ffn8_job *)arg;
    int64_t hlen = J->f > J->fs ? J->f : J->fs;
    if (hlen <= 0)
        hlen = 128;
    double *h = (double *)malloc((size_t)hlen * sizeof(double));
    uint8_t *hq = (uint8_t *)malloc((size_t)hlen);
    double *sh = (double *)malloc((size_t)(hlen / 128) * sizeof(double));
    if (!h || !hq || !sh) {
        free(h);
        free(hq);
        free(sh);
        J->status = ORACLE_ENOMEM;
        return NULL;
    }
    const int64_t db = J->d / 128;
    for (int64_t i = J->tid; i < J->ntok; i += J->nthreads) {
        int64_t t = J->tokens ? J->tokens[i] : i;
        const uint8_t *xt = J->xq + t * J->d;
        const double *st = J->sx + t * db;
        double *y = J->out + i * J->d;
        for (int64_t c = 0; c < J->d; c++)
            y[c] = 0.0;
        for (int64_t j = 0; j < J->k; j++) {
            int32_t e = J->idx[t * J->k + j];
            if (e < 0 || e >= J->E || !J->W1q[e] || !J->W3q[e] || !J->W2q[e]) {
                J->status = ORACLE_ERANGE;
                free(h);
                free(hq);
                free(sh);
                return NULL;
            }
            expert_ffn_fp8_add(J->W1q[e], J->s1[e], J->W3q[e], J->s3[e], J->W2q[e], J->s2[e], xt, st, J->d,
                               J->f, J->w[t * J->k + j], h, hq, sh, y);
        }
        if (J->fs > 0)
            expert_ffn_fp8_add(J->Ws1q, J->ss1, J->Ws3q, J->ss3, J->Ws2q, J->ss2, xt, st, J->d, J->fs, 1.0, h, hq,
                               sh, y);
    }
    free(h);
    free(hq);
    free(sh);
    return NULL;
}

/* FP8 expert FFNs of the listed tokens (the FP8 counterpart of oracle_moe_ffn).
 * xq [T,d] e4m3 with sx [T, d/128]; per-expert W1q[e], W3q[e] [f,d] with
 * s1[e], s3[e] [f/128, d/128]; W2q[e] [d,f] with s2[e] [d/128, f/128]; the
 * shared expert likewise (fs > 0).  d, f, fs multiples of 128. */
int oracle_moe_ffn_fp8(const uint8_t *xq, const double *sx,
                       const uint8_t *const *W1q, const double *const *s1,
                       const uint8_t *const *W3q, const double *const *s3,
                       const uint8_t *const *W2q, const double *const *s2,
                       int64_t d, int64_t f, int64_t E, const int32_t *idx, const double *w, int64_t k,
                       const uint8_t *Ws1q, const double *ss1, const uint8_t *Ws3q, const double *ss3,
                       const uint8_t *Ws2q, const double *ss2, int64_t fs,
                       const int64_t *tokens, int64_t ntok, double *out, int nthreads)
{
    if (d <= 0 || f <= 0 || E <= 0 || k < 1 || ntok < 0 || fs < 0 || d % 128 || f % 128 || fs % 128)
        return ORACLE_EARG;
    if (ntok == 0)
        return ORACLE_OK;
    if (!xq || !sx || !W1q || !W3q || !W2q || !s1 || !s3 || !s2 || !idx || !w || !out ||
        (fs > 0 && (!Ws1q || !Ws3q || !Ws2q || !ss1 || !ss3 || !ss2)))
        return ORACLE_EARG;
    if (nthreads <= 0)
        nthreads = oracle_default_threads();
    if (nthreads > ntok)
        nthreads = (int)ntok;
    ffn8_job *jobs = (ffn8_job *)calloc((size_t)nthreads, sizeof(ffn8_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return ORACLE_ENOMEM;
    }
    for (int i = 0; i < nthreads; i++) {
        ffn8_job J = {xq, sx, W1q, W3q, W2q, s1, s3, s2, d, f, E, k, idx, w, Ws1q, Ws3q, Ws2q, ss1, ss3, ss2,
                      fs, tokens, ntok, out, nthreads, i, ORACLE_OK};
        jobs[i] = J;
    }
    int started = 0;
    for (int i = 1; i < nthreads; i++) {
        if (pthread_create(&th[i], NULL, ffn8_worker, &jobs[i]) != 0)
            break;
        started = i;
    }
    for (int i = started + 1; i < nthreads; i++)
        ffn8_worker(&jobs[i]);
    ffn8_worker(&jobs[0]);
    for (int i = 1; i <= started; i++)
        pthread_join(th[i], NULL);
    int status = ORACLE_OK;
    for (int i = 0; i < nthreads; i++)
        if (jobs[i].status != ORACLE_OK)
            status = jobs[i].status;
    free(jobs);
    free(th);
    return status;
}

/* ------------------------------------------------------------------------
 * FP4 expert weights (GC-MoE, abstract: an FP8/FP4 MoE operator with
 * block-scaled MMA).  The pages name FP4 without a layout; the reading taken
 * is the OCP microscaling FP4 element type with 32-element blocks (MXFP4):
 *   e2m1 codes: bit 3 sign, bits 2-1 exponent (bias 1), bit 0 mantissa;
 *   exponent 0 is subnormal (0 or 0.5); no infinities or NaNs; largest 6.
 *   Weights are quantised per row in blocks of 32 consecutive K elements, a
 *   block's scale the smallest power of two s with amax / s <= 6 (s = 1 for
 *   an all-zero block), held to the UE8M0 range; codes are round to nearest,
 *   ties to the even code, saturating at 6.
 * Activations (x, and h before the down projection) stay e4m3 in 1 x 128
 * blocks, as in the FP8 path.
 * ------------------------------------------------------------------------ */

double oracle_e2m1_decode(uint8_t code)
{
    int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -v : v;
}

/* Nearest e2m1 code to v (ties to the code with an even mantissa), saturating to 6. */
uint8_t oracle_e2m1_encode(double v)
{
    uint8_t sign = (v < 0 || (v == 0 && signbit(v))) ? 8 : 0;
    double a = fabs(v);
    if (a >= 6.0)
        return sign | 7;
    uint8_t best = 0;
    double best_err = a;
    for (int c = 1; c <= 7; c++) {
        double err = fabs(oracle_e2m1_decode((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = (uint8_t)c;
            best_err = err;
        }
    }
    return sign | best;
}

/* Smallest power of two s with amax / s <= 6 (amax = 0: s = 1), kept in the UE8M0 range 2^-127 .. 2^127. */
double oracle_fp4_block_scale(double amax)
{
    if (!(amax > 0))
        return 1.0;
    int e = 0;
    while (amax > ldexp(6.0, e) && e < 127)
        e++;
    while (amax <= ldexp(6.0, e - 1) && e > -127)
        e--;
    return ldexp(1.0, e);
}

/* 1 x 32 blocks along each row: W [R, C] bf16 -> codes [R, C] (one e2m1 code per
 * byte, low 4 bits), scales [R, C/32].  C % 32 == 0. */
int oracle_quantize_rows_fp4(const uint16_t *W, int64_t R, int64_t C, uint8_t *q, double *s)
{
    if (R < 0 || C <= 0 || C % 32 || (R > 0 && (!W || !q || !s)))
        return ORACLE_EARG;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t b = 0; b < C / 32; b++) {
            double amax = 0;
            for (int64_t c = 0; c < 32; c++)
                amax = fmax(amax, fabs(bf16_value(W[r * C + b * 32 + c])));
            double sc = oracle_fp4_block_scale(amax);
            s[r * (C / 32) + b] = sc;
            for (int64_t c = 0; c < 32; c++)
                q[r * C + b * 32 + c] = oracle_e2m1_encode(bf16_value(W[r * C + b * 32 + c]) / sc);
        }
    }
    return ORACLE_OK;
}

/* One FP4-weight SwiGLU expert on one token: as expert_ffn_fp8_add with the
 * weights dequantised from e2m1 codes and 1 x 32 scales (W1/W3 [f,d] codes with
 * [f, d/32] scales, W2 [d,f] codes with [d, f/32] scales). */
static void expert_ffn_fp4_add(const uint8_t *W1q, const double *s1, const uint8_t *W3q, const double *s3,
                               const uint8_t *W2q, const double *s2, const uint8_t *xq, const double *sx,
                               int64_t d, int64_t f, double gate, double *h, uint8_t *hq, double *sh, double *y)
{
    const int64_t fb = f / 128;
    for (int64_t r = 0; r < f; r++) {
        double g = 0.0, u = 0.0;
        for (int64_t c = 0; c < d; c++) {
            double xc = e4m3_value(xq[c]) * sx[c / 128];
            g += oracle_e2m1_decode(W1q[r * d + c]) * s1[r * (d / 32) + c / 32] * xc;
            u += oracle_e2m1_decode(W3q[r * d + c]) * s3[r * (d / 32) + c / 32] * xc;
        }
        h[r] = g / (1.0 + exp(-g)) * u;
    }
    for (int64_t b = 0; b < fb; b++) {          /* requantise h in 1 x 128 blocks (e4m3) */
        double amax = 0;
        for (int64_t r = 0; r < 128; r++)
            amax = fmax(amax, fabs(h[b * 128 + r]));
        double sc = oracle_fp8_block_scale(amax);
        sh[b] = sc;
        for (int64_t r = 0; r < 128; r++)
            hq[b * 128 + r] = oracle_e4m3_encode_fast(h[b * 128 + r] / sc);
    }
    for (int64_t r = 0; r < f; r++)
        h[r] = e4m3_value(hq[r]) * sh[r / 128];
    for (int64_t c = 0; c < d; c++) {
        double z = 0.0;
        for (int64_t r = 0; r < f; r++)
            z += oracle_e2m1_decode(W2q[c * f + r]) * s2[c * (f / 32) + r / 32] * h[r];
        y[c] += gate * z;
    }
}

typedef struct {
    const uint8_t *xq;
    const double *sx;
    const uint8_t *const *W1q, *const *W3q, *const *W2q;
    const double *const *s1, *const *s3, *const *s2;
    int64_t d, f, E, k;
    const int32_t *idx;
    const double *w;
    const uint8_t *Ws1q, *Ws3q, *Ws2q;
    const double *ss1, *ss3, *ss2;
    int64_t fs;
    const int64_t *tokens;
    int64_t ntok;
    double *out;
    int nthreads, tid;
    int status;
} ffn4_job;

static void *ffn4_worker(void *arg)
{
    ffn4_job *J = (ffn4_job *)arg;
    int64_t hlen = J->f > J->fs ? J->f : J->fs;
    if (hlen <= 0)
        hlen = 128;
    double *h = (double *)malloc((size_t)hlen * sizeof(double));
    uint8_t *hq = (uint8_t *)malloc((size_t)hlen);
    double *sh = (double *)malloc((size_t)(hlen / 128) * sizeof(double));
    if (!h || !hq || !sh) {
        free(h);
        free(hq);
        free(sh);
        J->status = ORACLE_ENOMEM;
        return NULL;
    }
    const int64_t db = J->d / 128;
    for (int64_t i = J->tid; i < J->ntok; i += J->nthreads) {
        int64_t t = J->tokens ? J->tokens[i] : i;
        const uint8_t *xt = J->xq + t * J->d;
        const double *st = J->sx + t * db;
        double *y = J->out + i * J->d;
        for (int64_t c = 0; c < J->d; c++)
            y[c] = 0.0;
        for (int64_t j = 0; j < J->k; j++) {
            int32_t e = J->idx[t * J->k + j];
            if (e < 0 || e >= J->E || !J->W1q[e] || !J->W3q[e] || !J->W2q[e]) {
                J->status = ORACLE_ERANGE;
                free(h);
                free(hq);
                free(sh);
                return NULL;
            }
            expert_ffn_fp4_add(J->W1q[e], J->s1[e], J->W3q[e], J->s3[e], J->W2q[e], J->s2[e], xt, st, J->d,
                               J->f, J->w[t * J->k + j], h, hq, sh, y);
        }
        if (J->fs > 0)
            expert_ffn_fp4_add(J->Ws1q, J->ss1, J->Ws3q, J->ss3, J->Ws2q, J->ss2, xt, st, J->d, J->fs, 1.0, h, hq,
                               sh, y);
    }
    free(h);
    free(hq);
    free(sh);
    return NULL;
}

/* FP4-weight expert FFNs of the listed tokens (the FP4 counterpart of
 * oracle_moe_ffn_fp8): xq [T,d] e4m3 with sx [T, d/128]; per expert W1q[e],
 * W3q[e] [f,d] e2m1 codes (one per byte) with s1[e], s3[e] [f, d/32];
 * W2q[e] [d,f] with s2[e] [d, f/32]; the shared expert likewise (fs > 0).
 * d, f, fs multiples of 128. */
int oracle_moe_ffn_fp4(const uint8_t *xq, const double *sx,
                       const uint8_t *const *W1q, const double *const *s1,
                       const uint8_t *const *W3q, const double *const *s3,
                       const uint8_t *const *W2q, const double *const *s2,
                       int64_t d, int64_t f, int64_t E, const int32_t *idx, const double *w, int64_t k,
                       const uint8_t *Ws1q, const double *ss1, const uint8_t *Ws3q, const double *ss3,
                       const uint8_t *Ws2q, const double *ss2, int64_t fs,
                       const int64_t *tokens, int64_t ntok, double *out, int nthreads)
{
    if (d <= 0 || f <= 0 || E <= 0 || k < 1 || ntok < 0 || fs < 0 || d % 128 || f % 128 || fs % 128)
        return ORACLE_EARG;
    if (ntok == 0)
        return ORACLE_OK;
    if (!xq || !sx || !W1q || !W3q || !W2q || !s1 || !s3 || !s2 || !idx || !w || !out ||
        (fs > 0 && (!Ws1q || !Ws3q || !Ws2q || !ss1 || !ss3 || !ss2)))
        return ORACLE_EARG;
    if (nthreads <= 0)
        nthreads = oracle_default_threads();
    if (nthreads > ntok)
        nthreads = (int)ntok;
    ffn4_job *jobs = (ffn4_job *)calloc((size_t)nthreads, sizeof(ffn4_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return ORACLE_ENOMEM;
    }
    for (int i = 0; i < nthreads; i++) {
        ffn4_job J = {xq, sx, W1q, W3q, W2q, s1, s3, s2, d, f, E, k, idx, w, Ws1q, Ws3q, Ws2q, ss1, ss3, ss2,
                      fs, tokens, ntok, out, nthreads, i, ORACLE_OK};
        jobs[i] = J;
    }
    int started = 0;
    for (int i = 1; i < nthreads; i++) {
        if (pthread_create(&th[i], NULL, ffn4_worker, &jobs[i]) != 0)
            break;
        started = i;
    }
    for (int i = started + 1; i < nthreads; i++)
        ffn4_worker(&jobs[i]);
    ffn4_worker(&jobs[0]);
    for (int i = 1; i <= started; i++)
        pthread_join(th[i], NULL);
    int status = ORACLE_OK;
    for (int i = 0; i < nthreads; i++)
        if (jobs[i].status != ORACLE_OK)
            status = jobs[i].status;
    free(jobs);
    free(th);
    return status;
}
