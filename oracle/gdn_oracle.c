/*
 * gdn_oracle.c -- plain fp64 CPU oracle for the Gated DeltaNet (GDN) token mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg use this file.  It shares no code, header, table or helper
 * with the CUDA library; it is the slow, obviously correct definition that the
 * CUDA path is checked against.
 *
 * Source of every formula: "On the design of Qwen3.8-Next architecture:
 * evaluation, efficiency and training stability" (paper-archivist reading of
 * arXiv 2608.30320), section 2.1.1 "Gated Delta recurrence" and
 * "GDN parameterisation", eqs. (1)-(11).
 *
 * Readings taken where the page is silent (each one is listed in the design
 * notes of the repository):
 *   - state orientation: S is dk x dv ("transpose of the original GDN
 *     convention"), stored row-major, dv contiguous; y = S^T q.
 *   - readout uses the updated state S_t (eq. 4 as printed); a scale factor on q
 *     is exposed and is 1 in every workload.
 *   - alpha is passed as g = log(alpha); the oracle forms alpha = exp(g) in fp64.
 *   - ShortConv: width W, no bias, causal, zero history at every sequence start;
 *     tap w[c][W-1] multiplies the current token.
 *   - L2Norm: x / sqrt(sum x^2 + eps), eps = 1e-6, over the head dimension.
 *   - softplus(x) = log(1 + e^x), no threshold.
 *   - RMSNorm is zero-centred: y / sqrt(mean(y^2) + eps) * (1 + w), w shared by
 *     all heads, over dv.
 *
 * parity pins: every function here is pinned by tests that do not re-type it
 * (closed forms, brute force, special cases); see tests/test_oracle_pins.py.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------- */
/* thread pool over independent (sequence, head) units                        */
/* ------------------------------------------------------------------------- */

typedef void (*unit_fn)(void* ctx, long unit);

typedef struct {
    unit_fn fn;
    void* ctx;
    long n_units;
    long next;
    pthread_mutex_t lock;
} pool_t;

static void* pool_worker(void* arg) {
    pool_t* p = (pool_t*)arg;
    for (;;) {
        pthread_mutex_lock(&p->lock);
        long u = p->next++;
        pthread_mutex_unlock(&p->lock);
        if (u >= p->n_units) break;
        p->fn(p->ctx, u);
    }
    return NULL;
}

static int resolve_threads(int nthreads, long n_units) {
    if (nthreads <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = c > 0 ? (int)c : 1;
    }
    if (nthreads > n_units) nthreads = (int)(n_units > 0 ? n_units : 1);
    if (nthreads > 256) nthreads = 256;
    return nthreads;
}

static void run_units(unit_fn fn, void* ctx, long n_units, int nthreads) {
    pool_t p;
    p.fn = fn;
    p.ctx = ctx;
    p.n_units = n_units;
    p.next = 0;
    pthread_mutex_init(&p.lock, NULL);
    int nt = resolve_threads(nthreads, n_units);
    if (nt <= 1) {
        pool_worker(&p);
    } else {
        pthread_t th[256];
        for (int i = 0; i < nt; ++i) pthread_create(&th[i], NULL, pool_worker, &p);
        for (int i = 0; i < nt; ++i) pthread_join(th[i], NULL);
    }
    pthread_mutex_destroy(&p.lock);
}

/* Number of threads a call with this many units would use (reported by the bench). */
int oracle_threads_used(int nthreads, long n_units) { return resolve_threads(nthreads, n_units); }

/* ------------------------------------------------------------------------- */
/* Gated delta rule, eqs. (1)-(4), sequential over tokens                      */
/* ------------------------------------------------------------------------- */

/*
 * One token of the gated delta rule on a dk x dv state S (row-major, dv contiguous):
 *   eq. (1)  S~ = alpha S
 *   eq. (2)  e  = v - S~^T k
 *   eq. (3)  S  = S~ + beta k e^T
 *   eq. (4)  y  = S^T q        (times the exposed scale, 1 by default)
 * e is caller-provided scratch of dv doubles.
 */
static void token_update(double* S, const double* q, const double* k, const double* v, double alpha,
                         double beta, int dk, int dv, double scale, double* y, double* e) {
    for (long i = 0; i < (long)dk * dv; ++i) S[i] *= alpha;
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * k[i];
        e[j] = v[j] - acc;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += beta * k[i] * e[j];
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * q[i];
        y[j] = scale * acc;
    }
}

typedef struct {
    const double *q, *k, *v, *g, *beta, *S0;
    const int64_t* cu;
    int H, dk, dv;
    double scale;
    double *y, *S_T;
} rec_ctx;

static void rec_unit(void* vctx, long unit) {
    rec_ctx* c = (rec_ctx*)vctx;
    const int H = c->H, dk = c->dk, dv = c->dv;
    const long n = unit / H;
    const int h = (int)(unit % H);
    double* S = (double*)calloc((size_t)dk * dv, sizeof(double));
    double* e = (double*)malloc(sizeof(double) * dv);
    if (c->S0) memcpy(S, c->S0 + ((size_t)n * H + h) * dk * dv, sizeof(double) * dk * dv);

    for (int64_t t = c->cu[n]; t < c->cu[n + 1]; ++t) {
        const size_t th = (size_t)t * H + h;
        token_update(S, c->q + th * dk, c->k + th * dk, c->v + th * dv, exp(c->g[th]), c->beta[th],
                     dk, dv, c->scale, c->y + th * dv, e);
    }
    if (c->S_T) memcpy(c->S_T + ((size_t)n * H + h) * dk * dv, S, sizeof(double) * dk * dv);
    free(e);
    free(S);
}

/*
 * q, k: [N, H, dk]; v, y: [N, H, dv]; g (= log alpha), beta: [N, H];
 * S0, S_T: [num_seqs, H, dk, dv] (S0 may be NULL = zeros, S_T may be NULL);
 * cu_seqlens: [num_seqs + 1] token offsets, cu[0] = 0, non-decreasing.
 */
void oracle_recurrence(const double* q, const double* k, const double* v, const double* g,
                       const double* beta, const double* S0, const int64_t* cu_seqlens,
                       int num_seqs, int H, int dk, int dv, double scale, double* y,
                       double* S_T, int nthreads) {
    rec_ctx c = {q, k, v, g, beta, S0, cu_seqlens, H, dk, dv, scale, y, S_T};
    run_units(rec_unit, &c, (long)num_seqs * H, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Reverse-mode derivative of eqs. (1)-(4)                                     */
/* ------------------------------------------------------------------------- */

/*
 * For a loss L with dL/dy_t = dy_t and dL/dS_T = dS_T, the token step of eqs. (1)-(4),
 *   S~ = alpha S,  e = v - S~^T k,  S_t = S~ + beta k e^T,  y = scale S_t^T q,
 * (S = S_{t-1}, alpha = exp(g)) is walked backwards with D = dL/dS_t:
 *   D  += scale q dy^T               dq = scale S_t dy
 *   de  = beta D^T k                 dbeta = k^T D e          dk = beta D e - S~ de
 *   dv  = de                         D~ = D - k de^T          (= dL/dS~)
 *   dg  = alpha sum_ij D~_ij S_ij    D <- alpha D~            (= dL/dS_{t-1})
 * and dS0 is D after the first token.  The states S_{t-1} come from a forward pass that
 * keeps the state at the start of every 64 tokens and recomputes each such block's states
 * before walking it backwards.
 */
typedef struct {
    const double *q, *k, *v, *g, *beta, *S0, *dy, *dS_T;
    const int64_t* cu;
    int H, dk, dv;
    double scale;
    double *dq, *dk_, *dv_, *dg, *dbeta, *dS0;
} bwd_ctx;

enum { BWD_BLOCK = 64 };

static void bwd_unit(void* vctx, long unit) {
    bwd_ctx* c = (bwd_ctx*)vctx;
    const int H = c->H, dk = c->dk, dv = c->dv;
    const long n = unit / H;
    const int h = (int)(unit % H);
    const size_t SZ = (size_t)dk * dv;
    const int64_t t0 = c->cu[n], t1 = c->cu[n + 1];
    const long nb = (long)((t1 - t0 + BWD_BLOCK - 1) / BWD_BLOCK);
    double* ck = (double*)malloc(sizeof(double) * SZ * (nb > 0 ? nb : 1));      /* state at each block start */
    double* st = (double*)malloc(sizeof(double) * SZ * (BWD_BLOCK + 1));        /* one block's states */
    double* S = (double*)calloc(SZ, sizeof(double));
    double* D = (double*)calloc(SZ, sizeof(double));
    double* e = (double*)malloc(sizeof(double) * dv);
    double* de = (double*)malloc(sizeof(double) * dv);
    double* ytmp = (double*)malloc(sizeof(double) * dv);
    if (c->S0) memcpy(S, c->S0 + ((size_t)n * H + h) * SZ, sizeof(double) * SZ);
    for (int64_t t = t0; t < t1; ++t) {
        if ((t - t0) % BWD_BLOCK == 0) memcpy(ck + (size_t)((t - t0) / BWD_BLOCK) * SZ, S, sizeof(double) * SZ);
        const size_t th = (size_t)t * H + h;
        token_update(S, c->q + th * dk, c->k + th * dk, c->v + th * dv, exp(c->g[th]), c->beta[th], dk, dv, c->scale,
                     ytmp, e);
    }
    if (c->dS_T) memcpy(D, c->dS_T + ((size_t)n * H + h) * SZ, sizeof(double) * SZ);
    for (long b = nb - 1; b >= 0; --b) {
        const int64_t tb = t0 + (int64_t)b * BWD_BLOCK, te = tb + BWD_BLOCK < t1 ? tb + BWD_BLOCK : t1;
        memcpy(st, ck + (size_t)b * SZ, sizeof(double) * SZ);
        for (int64_t t = tb; t < te; ++t) {  /* st[i] = S_{tb + i - 1}, the state before token tb + i */
            const size_t th = (size_t)t * H + h;
            double* nxt = st + (size_t)(t - tb + 1) * SZ;
            memcpy(nxt, st + (size_t)(t - tb) * SZ, sizeof(double) * SZ);
            token_update(nxt, c->q + th * dk, c->k + th * dk, c->v + th * dv, exp(c->g[th]), c->beta[th], dk, dv,
                         c->scale, ytmp, e);
        }
        for (int64_t t = te - 1; t >= tb; --t) {
            const size_t th = (size_t)t * H + h;
            const double* q = c->q + th * dk;
            const double* k = c->k + th * dk;
            const double* v = c->v + th * dv;
            const double* dyt = c->dy + th * dv;
            const double alpha = exp(c->g[th]), beta = c->beta[th];
            const double* Sp = st + (size_t)(t - tb) * SZ;      /* S_{t-1} */
            const double* St = st + (size_t)(t - tb + 1) * SZ;  /* S_t */
            for (int j = 0; j < dv; ++j) {                       /* e = v - alpha S_{t-1}^T k */
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += Sp[(size_t)i * dv + j] * k[i];
                e[j] = v[j] - alpha * acc;
            }
            for (int i = 0; i < dk; ++i) {                       /* readout */
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    D[(size_t)i * dv + j] += c->scale * q[i] * dyt[j];
                    acc += St[(size_t)i * dv + j] * dyt[j];
                }
                c->dq[th * dk + i] = c->scale * acc;
            }
            double db = 0.0;
            for (int j = 0; j < dv; ++j) {                       /* de = beta D^T k */
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += D[(size_t)i * dv + j] * k[i];
                de[j] = beta * acc;
                db += acc * e[j];                                /* k^T D e */
            }
            c->dbeta[th] = db;
            for (int i = 0; i < dk; ++i) {                       /* dk = beta D e - S~ de */
                double a = 0.0, b2 = 0.0;
                for (int j = 0; j < dv; ++j) {
                    a += D[(size_t)i * dv + j] * e[j];
                    b2 += alpha * Sp[(size_t)i * dv + j] * de[j];
                }
                c->dk_[th * dk + i] = beta * a - b2;
            }
            for (int j = 0; j < dv; ++j) c->dv_[th * dv + j] = de[j];
            double da = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) {
                    const size_t ij = (size_t)i * dv + j;
                    D[ij] -= k[i] * de[j];                       /* D~ */
                    da += D[ij] * Sp[ij];
                    D[ij] *= alpha;                              /* dL/dS_{t-1} */
                }
            c->dg[th] = alpha * da;
        }
    }
    memcpy(c->dS0 + ((size_t)n * H + h) * SZ, D, sizeof(double) * SZ);
    free(ytmp); free(de); free(e); free(D); free(S); free(st); free(ck);
}

/*
 * Gradients of L through eqs. (1)-(4) for packed sequences.  q, k, dq, dk: [N, H, dk];
 * v, dy, dv: [N, H, dv]; g, beta, dg, dbeta: [N, H]; S0, dS_T, dS0: [num_seqs, H, dk, dv]
 * (S0 and dS_T may be NULL = zeros).  Tokens outside every sequence are not written.
 */
void oracle_backward(const double* q, const double* k, const double* v, const double* g, const double* beta,
                     const double* S0, const int64_t* cu_seqlens, int num_seqs, int H, int dk, int dv, double scale,
                     const double* dy, const double* dS_T, double* dq, double* dk_, double* dv_, double* dg,
                     double* dbeta, double* dS0, int nthreads) {
    bwd_ctx c = {q, k, v, g, beta, S0, dy, dS_T, cu_seqlens, H, dk, dv, scale, dq, dk_, dv_, dg, dbeta, dS0};
    run_units(bwd_unit, &c, (long)num_seqs * H, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Input parameterisation, eqs. (6)-(10)                                       */
/* ------------------------------------------------------------------------- */

static double silu(double x) { return x / (1.0 + exp(-x)); }
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }
static double softplus(double x) { return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x)); }

typedef struct {
    const double *xq, *xk, *xv, *wq, *wk, *wv, *bl, *al, *A, *ba;
    const int64_t* cu;
    int W, H, dk, dv;
    double eps;
    double *q, *k, *v, *g, *beta;
} prep_ctx;

/* ShortConv (causal depthwise, width W, zero history at the sequence start), then SiLU. */
static void conv_silu(const double* x, const double* w, int64_t t, int64_t start, int H, int h,
                      int d, int W, double* out) {
    for (int c = 0; c < d; ++c) {
        const double* wc = w + ((size_t)h * d + c) * W;
        double acc = 0.0;
        for (int j = 0; j < W; ++j) {
            int64_t s = t - (W - 1) + j;
            if (s >= start) acc += wc[j] * x[((size_t)s * H + h) * d + c];
        }
        out[c] = silu(acc);
    }
}

static void l2norm(double* x, int d, double eps) {
    double ss = 0.0;
    for (int i = 0; i < d; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss + eps);
    for (int i = 0; i < d; ++i) x[i] *= inv;
}

static void prep_unit(void* vctx, long unit) {
    prep_ctx* c = (prep_ctx*)vctx;
    const int H = c->H;
    const long n = unit / H;
    const int h = (int)(unit % H);
    for (int64_t t = c->cu[n]; t < c->cu[n + 1]; ++t) {
        double* qt = c->q + ((size_t)t * H + h) * c->dk;
        double* kt = c->k + ((size_t)t * H + h) * c->dk;
        double* vt = c->v + ((size_t)t * H + h) * c->dv;
        conv_silu(c->xq, c->wq, t, c->cu[n], H, h, c->dk, c->W, qt); /* eq. (6) */
        l2norm(qt, c->dk, c->eps);
        conv_silu(c->xk, c->wk, t, c->cu[n], H, h, c->dk, c->W, kt); /* eq. (7) */
        l2norm(kt, c->dk, c->eps);
        conv_silu(c->xv, c->wv, t, c->cu[n], H, h, c->dv, c->W, vt); /* eq. (8) */
        size_t th = (size_t)t * H + h;
        c->beta[th] = sigmoid(c->bl[th]);                                 /* eq. (9) */
        c->g[th] = -exp(c->A[h]) * softplus(c->al[th] + c->ba[h]);        /* eq. (10), log alpha */
    }
}

/*
 * x_q, x_k: [N, H, dk], x_v: [N, H, dv] -- outputs of the input projections;
 * w_q, w_k: [H*dk, W], w_v: [H*dv, W] -- depthwise conv taps, channel c = h*d + i;
 * beta_logit, alpha_logit: [N, H]; A_log, alpha_bias: [H].
 * Outputs q, k: [N, H, dk]; v: [N, H, dv]; g = log alpha and beta: [N, H].
 */
void oracle_prep(const double* x_q, const double* x_k, const double* x_v, const double* w_q,
                 const double* w_k, const double* w_v, int W, const double* beta_logit,
                 const double* alpha_logit, const double* A_log, const double* alpha_bias,
                 const int64_t* cu_seqlens, int num_seqs, int H, int dk, int dv, double eps,
                 double* q, double* k, double* v, double* g, double* beta, int nthreads) {
    prep_ctx c = {x_q, x_k, x_v, w_q, w_k, w_v, beta_logit, alpha_logit, A_log, alpha_bias,
                  cu_seqlens, W, H, dk, dv, eps, q, k, v, g, beta};
    run_units(prep_unit, &c, (long)num_seqs * H, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Output gate, eq. (11) without the output projection W_o                     */
/* ------------------------------------------------------------------------- */

/* out = sigmoid(z) * y / sqrt(mean(y^2) + eps) * (1 + w), per (token, head) over dv. */
void oracle_out_gate(const double* y, const double* z, const double* w, double eps, long N, int H,
                     int dv, double* out) {
    for (long r = 0; r < N * H; ++r) {
        const double* yr = y + (size_t)r * dv;
        const double* zr = z + (size_t)r * dv;
        double ms = 0.0;
        for (int j = 0; j < dv; ++j) ms += yr[j] * yr[j];
        ms /= dv;
        double inv = 1.0 / sqrt(ms + eps);
        for (int j = 0; j < dv; ++j) out[(size_t)r * dv + j] = sigmoid(zr[j]) * yr[j] * inv * (1.0 + w[j]);
    }
}

/* ------------------------------------------------------------------------- */
/* One decode step: eqs. (1)-(4) for one token per row against a given state  */
/* ------------------------------------------------------------------------- */

/*
 * q, k: [B, H, dk]; v, y: [B, H, dv]; g, beta: [B, H];
 * state: [num_slots, H, dk, dv], updated in place; slot: [B] or NULL (row i -> slot i).
 */
typedef struct {
    const double *q, *k, *v, *g, *beta;
    double* state;
    const int64_t* slot;
    int H, dk, dv;
    double scale;
    double* y;
} dec_ctx;

/* One (row, head) unit of a decode step: the same token_update as the prefill oracle. */
static void dec_unit(void* vctx, long unit) {
    dec_ctx* c = (dec_ctx*)vctx;
    const int H = c->H, dk = c->dk, dv = c->dv;
    const long b = unit / H;
    const int h = (int)(unit % H);
    const int64_t s = c->slot ? c->slot[b] : b;
    const size_t bh = (size_t)b * H + h;
    double* e = (double*)malloc(sizeof(double) * dv);
    token_update(c->state + ((size_t)s * H + h) * dk * dv, c->q + bh * dk, c->k + bh * dk, c->v + bh * dv,
                 exp(c->g[bh]), c->beta[bh], dk, dv, c->scale, c->y + bh * dv, e);
    free(e);
}

/* Rows name distinct slots, so the (row, head) units are independent; they run on nthreads
 * threads (0: every hardware thread). */
void oracle_decode_step(const double* q, const double* k, const double* v, const double* g,
                        const double* beta, double* state, const int64_t* slot, int B, int H,
                        int dk, int dv, double scale, double* y, int nthreads) {
    dec_ctx c = {q, k, v, g, beta, state, slot, H, dk, dv, scale, y};
    run_units(dec_unit, &c, (long)B * H, nthreads);
}
