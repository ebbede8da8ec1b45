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
