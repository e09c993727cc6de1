/*
 * KDA oracle: plain, slow, fp64 CPU implementation of Kimi Delta Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may include, link or call this file.  Only the
 * tests, the smoke check and the benchmark's CPU-baseline leg use it.  It
 * shares no code, header, table or helper with the CUDA sources.
 *
 * What is computed (per request r, head h, token t = 1..L_r):
 *
 *     S'  = Diag(alpha_t) S_{t-1}            alpha_t = exp(g_t), g_t = log alpha_t
 *     u   = S'^T k_t
 *     d   = beta_t (v_t - u)
 *     S_t = S' + k_t d^T                     == (I - beta k k^T) Diag(alpha) S + beta k v^T
 *     o_t = S_t^T q_t                        (post-update state, no scale factor)
 *
 * Source: the delta-rule linear attention with a channel-wise forget gate
 * ("KimiDelta Attention (KDA)", section 一.1 of the CSDN post analysing the
 * Kimi K3 technical report) and the fixed-size per-request recurrent state
 * ("Kimi K3 开源日来了", Infra section, second layer).  The pages describe the
 * recurrence in words only; the algebraic form above is the plain reading of
 * "delta rule + per-channel decay gate" and is written out token by token,
 * with no chunking, blocking or reordering.
 *
 * Layouts (row-major, all fp64 here; callers widen bf16/fp32 inputs exactly):
 *   q, k, g : [T_total, H, dk]      v, o : [T_total, H, dv]
 *   beta    : [T_total, H]          states : [n, H, dk, dv]  (dv contiguous)
 *   cu_seqlens : [n_req + 1] token offsets of the packed requests
 *   snapshots  : [sum_r floor(L_r / stride), H, dk, dv]; snapshot j (1-based)
 *                of request r is the state after its first j*stride tokens,
 *                stored at dense index (sum_{r'<r} floor(L_r'/stride)) + j - 1
 *                ("Kimi K3 开源日来了", Infra section: KDA state snapshots kept
 *                sparsely at a subset of the 512-token block boundaries).
 *
 * Parity pins (tests/test_oracle_pins.py) check every function here against
 * closed forms, brute-force dense transition products, an independently
 * derived chunked form, hand-worked fixtures and invariants.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

/* ------------------------------------------------------------------------- */
/* A tiny work-sharing pool: workers pull job indices from a shared counter. */
/* ------------------------------------------------------------------------- */

typedef void (*job_fn)(void *ctx, long job);

typedef struct {
    job_fn fn;
    void *ctx;
    long n_jobs;
    long next;
    pthread_mutex_t lock;
} pool_t;

static void *pool_worker(void *arg) {
    pool_t *p = (pool_t *)arg;
    for (;;) {
        long j;
        pthread_mutex_lock(&p->lock);
        j = p->next++;
        pthread_mutex_unlock(&p->lock);
        if (j >= p->n_jobs) break;
        p->fn(p->ctx, j);
    }
    return NULL;
}

static void run_jobs(job_fn fn, void *ctx, long n_jobs, int n_threads) {
    pool_t p;
    pthread_t tids[256];
    int i, nt = n_threads;
    if (nt < 1) nt = 1;
    if (nt > 256) nt = 256;
    if (nt > n_jobs) nt = (int)(n_jobs > 0 ? n_jobs : 1);
    p.fn = fn;
    p.ctx = ctx;
    p.n_jobs = n_jobs;
    p.next = 0;
    pthread_mutex_init(&p.lock, NULL);
    if (nt == 1) {
        pool_worker(&p);
    } else {
        for (i = 0; i < nt; ++i) pthread_create(&tids[i], NULL, pool_worker, &p);
        for (i = 0; i < nt; ++i) pthread_join(tids[i], NULL);
    }
    pthread_mutex_destroy(&p.lock);
}

/* ------------------------------------------------------------------------- */
/* One recurrence step on a dk x dv state, in place.                          */
/* ------------------------------------------------------------------------- */

/* S <- (I - beta k k^T) Diag(exp(g)) S + beta k v^T, written as the four
 * lines of the definition: decay, read-out of the old association, the
 * delta-rule correction, the rank-1 write.  u has room for dv doubles. */
static void kda_step(double *S, int dk, int dv, const double *k, const double *v,
                     const double *g, double beta, double *u) {
    int i, j;
    for (i = 0; i < dk; ++i) {            /* S' = Diag(alpha) S */
        const double a = exp(g[i]);
        double *row = S + (size_t)i * dv;
        for (j = 0; j < dv; ++j) row[j] *= a;
    }
    for (j = 0; j < dv; ++j) u[j] = 0.0;  /* u = S'^T k */
    for (i = 0; i < dk; ++i) {
        const double *row = S + (size_t)i * dv;
        for (j = 0; j < dv; ++j) u[j] += row[j] * k[i];
    }
    for (j = 0; j < dv; ++j) u[j] = beta * (v[j] - u[j]);  /* delta = beta (v - u) */
    for (i = 0; i < dk; ++i) {            /* S = S' + k delta^T */
        double *row = S + (size_t)i * dv;
        for (j = 0; j < dv; ++j) row[j] += k[i] * u[j];
    }
}

/* o = S^T q */
static void kda_readout(const double *S, int dk, int dv, const double *q, double *o) {
    int i, j;
    for (j = 0; j < dv; ++j) o[j] = 0.0;
    for (i = 0; i < dk; ++i) {
        const double *row = S + (size_t)i * dv;
        for (j = 0; j < dv; ++j) o[j] += row[j] * q[i];
    }
}

/* ------------------------------------------------------------------------- */
/* Varlen prefill: every (request, head) chain runs the recurrence from its  */
/* initial state to the end of the request.                                  */
/* ------------------------------------------------------------------------- */

typedef struct {
    int n_req, H, dk, dv, stride;
    const int64_t *cu;
    const int64_t *cu_snap;
    const double *q, *k, *v, *g, *beta, *s0;
    double *o, *s_final, *snaps;
} prefill_ctx;

static void prefill_job(void *vctx, long job) {
    const prefill_ctx *c = (const prefill_ctx *)vctx;
    const int r = (int)(job / c->H), h = (int)(job % c->H);
    const int H = c->H, dk = c->dk, dv = c->dv;
    const size_t ss = (size_t)dk * dv;
    double *S = (double *)malloc(ss * sizeof(double));
    double *u = (double *)malloc((size_t)dv * sizeof(double));
    int64_t t;
    if (!S || !u) { free(S); free(u); return; }
    if (c->s0) memcpy(S, c->s0 + ((size_t)r * H + h) * ss, ss * sizeof(double));
    else memset(S, 0, ss * sizeof(double));
    for (t = c->cu[r]; t < c->cu[r + 1]; ++t) {
        const size_t th = (size_t)t * H + h;
        const int64_t pos = t - c->cu[r] + 1; /* tokens of this request consumed */
        kda_step(S, dk, dv, c->k + th * dk, c->v + th * dv, c->g + th * dk, c->beta[th], u);
        if (c->o) kda_readout(S, dk, dv, c->q + th * dk, c->o + th * dv);
        if (c->snaps && c->stride > 0 && pos % c->stride == 0) {
            const int64_t idx = c->cu_snap[r] + pos / c->stride - 1;
            memcpy(c->snaps + ((size_t)idx * H + h) * ss, S, ss * sizeof(double));
        }
    }
    if (c->s_final) memcpy(c->s_final + ((size_t)r * H + h) * ss, S, ss * sizeof(double));
    free(S);
    free(u);
}

/* Number of snapshots of a request of length len at the given stride. */
long oracle_snapshot_count(long len, long stride) {
    return stride > 0 ? len / stride : 0;
}

int oracle_kda_prefill(int n_req, const int64_t *cu_seqlens, int H, int dk, int dv,
                       const double *q, const double *k, const double *v,
                       const double *g, const double *beta,
                       const double *initial_state, int snapshot_stride,
                       double *o, double *final_state, double *snapshots,
                       int n_threads) {
    prefill_ctx c;
    int64_t *cu_snap;
    int r;
    if (n_req < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens) return ORACLE_EINVAL;
    for (r = 0; r < n_req; ++r)
        if (cu_seqlens[r + 1] < cu_seqlens[r]) return ORACLE_EINVAL;
    cu_snap = (int64_t *)malloc((size_t)(n_req + 1) * sizeof(int64_t));
    if (!cu_snap) return ORACLE_ENOMEM;
    cu_snap[0] = 0;
    for (r = 0; r < n_req; ++r)
        cu_snap[r + 1] = cu_snap[r] + oracle_snapshot_count(cu_seqlens[r + 1] - cu_seqlens[r],
                                                            snapshot_stride);
    c.n_req = n_req; c.H = H; c.dk = dk; c.dv = dv; c.stride = snapshot_stride;
    c.cu = cu_seqlens; c.cu_snap = cu_snap;
    c.q = q; c.k = k; c.v = v; c.g = g; c.beta = beta; c.s0 = initial_state;
    c.o = o; c.s_final = final_state; c.snaps = snapshots;
    run_jobs(prefill_job, &c, (long)n_req * H, n_threads);
    free(cu_snap);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Decode: one token per request against a pool of fixed-size states.       */
/* ------------------------------------------------------------------------- */

typedef struct {
    int H, dk, dv;
    const int64_t *slot;
    const double *q, *k, *v, *g, *beta;
    double *state, *o;
} decode_ctx;

static void decode_job(void *vctx, long job) {
    const decode_ctx *c = (const decode_ctx *)vctx;
    const int n = (int)(job / c->H), h = (int)(job % c->H);
    const int H = c->H, dk = c->dk, dv = c->dv;
    const size_t ss = (size_t)dk * dv, th = (size_t)n * H + h;
    const int64_t s = c->slot ? c->slot[n] : n;
    double *S = c->state + ((size_t)s * H + h) * ss;
    double *u = (double *)malloc((size_t)dv * sizeof(double));
    if (!u) return;
    kda_step(S, dk, dv, c->k + th * dk, c->v + th * dv, c->g + th * dk, c->beta[th], u);
    kda_readout(S, dk, dv, c->q + th * dk, c->o + th * dv);
    free(u);
}

/* One decode step for n requests: request n updates state slot slot[n] (or n
 * when slot is NULL) in place and writes o[n]. */
int oracle_kda_decode_step(int n, int H, int dk, int dv,
                           const double *q, const double *k, const double *v,
                           const double *g, const double *beta,
                           double *state, const int64_t *slot, double *o, int n_threads) {
    decode_ctx c;
    if (n < 0 || H <= 0 || dk <= 0 || dv <= 0 || !state || !o) return ORACLE_EINVAL;
    c.H = H; c.dk = dk; c.dv = dv; c.slot = slot;
    c.q = q; c.k = k; c.v = v; c.g = g; c.beta = beta; c.state = state; c.o = o;
    run_jobs(decode_job, &c, (long)n * H, n_threads);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Context-parallel split ("Kimi K3 开源日来了", Infra section, first layer): */
/* a segment's effect is (i) the state it produces from a zero start and     */
/* (ii) the linear map it applies to an incoming state.  Both are local.     */
/* ------------------------------------------------------------------------- */

typedef struct {
    int H, dk, dv;
    const int64_t *seg;
    const double *k, *v, *g, *beta;
    double *s_loc, *m;
} local_ctx;

static void local_job(void *vctx, long job) {
    const local_ctx *c = (const local_ctx *)vctx;
    const int s = (int)(job / c->H), h = (int)(job % c->H);
    const int H = c->H, dk = c->dk, dv = c->dv;
    double *S = c->s_loc + ((size_t)s * H + h) * dk * dv;
    double *M = c->m + ((size_t)s * H + h) * dk * dk;
    double *u = (double *)malloc((size_t)(dv > dk ? dv : dk) * sizeof(double));
    double *w = (double *)malloc((size_t)dk * sizeof(double));
    int64_t t;
    int i, j;
    if (!u || !w) { free(u); free(w); return; }
    memset(S, 0, (size_t)dk * dv * sizeof(double));           /* zero start */
    for (i = 0; i < dk; ++i)                                   /* M = I */
        for (j = 0; j < dk; ++j) M[(size_t)i * dk + j] = (i == j) ? 1.0 : 0.0;
    for (t = c->seg[s]; t < c->seg[s + 1]; ++t) {
        const size_t th = (size_t)t * H + h;
        const double *kt = c->k + th * dk, *gt = c->g + th * dk;
        const double bt = c->beta[th];
        /* S_loc: the recurrence itself, from zero. */
        kda_step(S, dk, dv, kt, c->v + th * dv, gt, bt, u);
        /* M <- A_t M with A_t = (I - beta k k^T) Diag(alpha): first the
         * diagonal factor, then the projector, applied to every column. */
        for (i = 0; i < dk; ++i) {
            const double a = exp(gt[i]);
            for (j = 0; j < dk; ++j) M[(size_t)i * dk + j] *= a;
        }
        for (j = 0; j < dk; ++j) w[j] = 0.0;                   /* w = k^T M */
        for (i = 0; i < dk; ++i)
            for (j = 0; j < dk; ++j) w[j] += kt[i] * M[(size_t)i * dk + j];
        for (i = 0; i < dk; ++i)                               /* M -= beta k w^T */
            for (j = 0; j < dk; ++j) M[(size_t)i * dk + j] -= bt * kt[i] * w[j];
    }
    free(u);
    free(w);
}

/* Per segment s (token range seg_cu[s]..seg_cu[s+1] of one sequence) and head:
 * S_loc[s] = state after the segment from a zero start, M[s] = A_L ... A_1. */
int oracle_kda_chunk_local_state(int n_seg, const int64_t *seg_cu, int H, int dk, int dv,
                                 const double *k, const double *v, const double *g,
                                 const double *beta, double *s_loc, double *m,
                                 int n_threads) {
    local_ctx c;
    int s;
    if (n_seg < 0 || H <= 0 || dk <= 0 || dv <= 0 || !seg_cu || !s_loc || !m) return ORACLE_EINVAL;
    for (s = 0; s < n_seg; ++s)
        if (seg_cu[s + 1] < seg_cu[s]) return ORACLE_EINVAL;
    c.H = H; c.dk = dk; c.dv = dv; c.seg = seg_cu;
    c.k = k; c.v = v; c.g = g; c.beta = beta; c.s_loc = s_loc; c.m = m;
    run_jobs(local_job, &c, (long)n_seg * H, n_threads);
    return ORACLE_OK;
}

/* The one exchange that recovers every segment's true start state:
 * S_in[0] = S_init (zero when NULL), S_in[s+1] = M[s] S_in[s] + S_loc[s];
 * S_final = S_in[n_seg].  Written as the plain serial product. */
int oracle_kda_state_combine(int n_seg, int H, int dk, int dv, const double *s_loc,
                             const double *m, const double *s_init, double *s_in,
                             double *s_final) {
    const size_t ss = (size_t)dk * dv, mm = (size_t)dk * dk;
    double *cur, *nxt;
    int s, h, i, j, l;
    if (n_seg < 0 || H <= 0 || dk <= 0 || dv <= 0) return ORACLE_EINVAL;
    cur = (double *)malloc(ss * sizeof(double));
    nxt = (double *)malloc(ss * sizeof(double));
    if (!cur || !nxt) { free(cur); free(nxt); return ORACLE_ENOMEM; }
    for (h = 0; h < H; ++h) {
        if (s_init) memcpy(cur, s_init + (size_t)h * ss, ss * sizeof(double));
        else memset(cur, 0, ss * sizeof(double));
        for (s = 0; s < n_seg; ++s) {
            const double *M = m + ((size_t)s * H + h) * mm;
            const double *B = s_loc + ((size_t)s * H + h) * ss;
            if (s_in) memcpy(s_in + ((size_t)s * H + h) * ss, cur, ss * sizeof(double));
            for (i = 0; i < dk; ++i)
                for (j = 0; j < dv; ++j) {
                    double acc = B[(size_t)i * dv + j];
                    for (l = 0; l < dk; ++l) acc += M[(size_t)i * dk + l] * cur[(size_t)l * dv + j];
                    nxt[(size_t)i * dv + j] = acc;
                }
            memcpy(cur, nxt, ss * sizeof(double));
        }
        if (s_final) memcpy(s_final + (size_t)h * ss, cur, ss * sizeof(double));
    }
    free(cur);
    free(nxt);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Backward (training): the vector-Jacobian product of the prefill map.      */
/* FlashKDA also "raises training throughput" ("Kimi K3 开源日来了",          */
/* FlashKDA section), so the derivative of the same map is part of the path. */
/* Given cotangents dO (of o) and dS_final (of the final state), it returns  */
/* dq, dk, dv, dg (of g = log alpha), dbeta and dS_0 (of the initial state). */
/* Snapshots are by-products and take no cotangent.                          */
/*                                                                           */
/* The derivative is taken through the four defining lines of kda_step and   */
/* the read-out, in reverse:                                                 */
/*     o = S_t^T q          ->  dq = S_t dO,   dS += q dO^T                  */
/*     S_t = S' + k d^T     ->  dd = dS^T k,   dk = dS d,   dS' = dS         */
/*     d = beta (v - u)     ->  dv = beta dd,  dbeta = dd . (v - u),         */
/*                              du = -beta dd                                */
/*     u = S'^T k           ->  dS' += k du^T, dk += S' du                   */
/*     S' = Diag(a) S_{t-1} ->  dg_i = a_i sum_j dS'_ij S_{t-1,ij},          */
/*                              dS_{t-1} = Diag(a) dS'                       */
/* The forward states S_{t-1} are recomputed, in the forward order, in       */
/* blocks of 64 tokens from block-start states saved by a first forward      */
/* pass, so memory stays at (L/64 + 65) states per chain.                    */
/* ------------------------------------------------------------------------- */

#define ORACLE_BWD_BLOCK 64

typedef struct {
    int H, dk, dv;
    const int64_t *cu;
    const double *q, *k, *v, *g, *beta, *s0, *d_o, *d_final;
    double *dq, *dk_, *dv_, *dg, *dbeta, *d_init;
} backward_ctx;

/* One reverse step.  S_prev = S_{t-1}; dS holds dL/dS_t on entry and
 * dL/dS_{t-1} on exit.  Sp and dSp are dk x dv scratch, u/dd/du dv scratch. */
static void kda_step_backward(const double *S_prev, double *dS, int dk, int dv,
                              const double *q, const double *k, const double *v,
                              const double *g, double beta, const double *dO,
                              double *dq, double *dk_out, double *dv_out, double *dg,
                              double *dbeta, double *Sp, double *u, double *dd,
                              double *du) {
    int i, j;
    double s, dq_tail = 0.0;
    /* recompute the forward line by line: S', u, d */
    for (i = 0; i < dk; ++i) {
        const double a = exp(g[i]);
        for (j = 0; j < dv; ++j) Sp[(size_t)i * dv + j] = a * S_prev[(size_t)i * dv + j];
    }
    for (j = 0; j < dv; ++j) {
        s = 0.0;
        for (i = 0; i < dk; ++i) s += Sp[(size_t)i * dv + j] * k[i];
        u[j] = s;
    }
    /* d = beta (v - u); d lives in du's slot until du itself is formed below */
    for (j = 0; j < dv; ++j) du[j] = beta * (v[j] - u[j]);
    /* o = S_t^T q with S_t = S' + k d^T:  dq = S' dO + k (d . dO) */
    if (dO) {
        for (j = 0; j < dv; ++j) dq_tail += du[j] * dO[j];
        for (i = 0; i < dk; ++i) {
            s = 0.0;
            for (j = 0; j < dv; ++j) s += Sp[(size_t)i * dv + j] * dO[j];
            dq[i] = s + k[i] * dq_tail;
        }
        for (i = 0; i < dk; ++i)
            for (j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += q[i] * dO[j];
    } else {
        for (i = 0; i < dk; ++i) dq[i] = 0.0;
    }
    /* S_t = S' + k d^T:  dd = dS^T k,  dk = dS d */
    for (j = 0; j < dv; ++j) {
        s = 0.0;
        for (i = 0; i < dk; ++i) s += dS[(size_t)i * dv + j] * k[i];
        dd[j] = s;
    }
    for (i = 0; i < dk; ++i) {
        s = 0.0;
        for (j = 0; j < dv; ++j) s += dS[(size_t)i * dv + j] * du[j];
        dk_out[i] = s;
    }
    /* d = beta (v - u):  dv = beta dd,  dbeta = dd . (v - u),  du = -beta dd */
    s = 0.0;
    for (j = 0; j < dv; ++j) {
        dv_out[j] = beta * dd[j];
        s += dd[j] * (v[j] - u[j]);
        du[j] = -beta * dd[j];
    }
    *dbeta = s;
    /* u = S'^T k:  dS' = dS + k du^T,  dk += S' du */
    for (i = 0; i < dk; ++i) {
        s = 0.0;
        for (j = 0; j < dv; ++j) s += Sp[(size_t)i * dv + j] * du[j];
        dk_out[i] += s;
        for (j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += k[i] * du[j];
    }
    /* S' = Diag(a) S_{t-1}:  dg_i = a_i sum_j dS'_ij S_{t-1,ij};  dS_{t-1} = Diag(a) dS' */
    for (i = 0; i < dk; ++i) {
        const double a = exp(g[i]);
        s = 0.0;
        for (j = 0; j < dv; ++j) s += dS[(size_t)i * dv + j] * S_prev[(size_t)i * dv + j];
        dg[i] = a * s;
        for (j = 0; j < dv; ++j) dS[(size_t)i * dv + j] *= a;
    }
}

static void backward_job(void *vctx, long job) {
    const backward_ctx *c = (const backward_ctx *)vctx;
    const int r = (int)(job / c->H), h = (int)(job % c->H);
    const int H = c->H, dk = c->dk, dv = c->dv;
    const size_t ss = (size_t)dk * dv;
    const int64_t t0 = c->cu[r], L = c->cu[r + 1] - c->cu[r];
    const int64_t n_blk = (L + ORACLE_BWD_BLOCK - 1) / ORACLE_BWD_BLOCK;
    double *ck = (double *)malloc((size_t)(n_blk + 1) * ss * sizeof(double));
    double *blk = (double *)malloc((size_t)(ORACLE_BWD_BLOCK + 1) * ss * sizeof(double));
    double *dS = (double *)malloc(ss * sizeof(double));
    double *Sp = (double *)malloc(ss * sizeof(double));
    double *w = (double *)malloc((size_t)4 * dv * sizeof(double));
    int64_t b, t;
    if (!ck || !blk || !dS || !Sp || !w) goto done;
    /* forward pass: keep the state at every block start */
    if (c->s0) memcpy(ck, c->s0 + ((size_t)r * H + h) * ss, ss * sizeof(double));
    else memset(ck, 0, ss * sizeof(double));
    memcpy(blk, ck, ss * sizeof(double));
    for (t = 0; t < L; ++t) {
        const size_t th = (size_t)(t0 + t) * H + h;
        kda_step(blk, dk, dv, c->k + th * dk, c->v + th * dv, c->g + th * dk, c->beta[th], w);
        if ((t + 1) % ORACLE_BWD_BLOCK == 0)
            memcpy(ck + (size_t)((t + 1) / ORACLE_BWD_BLOCK) * ss, blk, ss * sizeof(double));
    }
    /* reverse pass */
    if (c->d_final) memcpy(dS, c->d_final + ((size_t)r * H + h) * ss, ss * sizeof(double));
    else memset(dS, 0, ss * sizeof(double));
    for (b = n_blk - 1; b >= 0; --b) {
        const int64_t lo = b * ORACLE_BWD_BLOCK;
        const int64_t hi = (lo + ORACLE_BWD_BLOCK < L) ? lo + ORACLE_BWD_BLOCK : L;
        /* blk[i] = S_{lo + i}, recomputed forward from the saved S_lo */
        memcpy(blk, ck + (size_t)b * ss, ss * sizeof(double));
        for (t = lo; t < hi - 1; ++t) {
            const size_t th = (size_t)(t0 + t) * H + h;
            memcpy(blk + (size_t)(t - lo + 1) * ss, blk + (size_t)(t - lo) * ss, ss * sizeof(double));
            kda_step(blk + (size_t)(t - lo + 1) * ss, dk, dv, c->k + th * dk, c->v + th * dv,
                     c->g + th * dk, c->beta[th], w);
        }
        for (t = hi - 1; t >= lo; --t) {
            const size_t th = (size_t)(t0 + t) * H + h;
            kda_step_backward(blk + (size_t)(t - lo) * ss, dS, dk, dv, c->q + th * dk,
                              c->k + th * dk, c->v + th * dv, c->g + th * dk, c->beta[th],
                              c->d_o ? c->d_o + th * dv : NULL, c->dq + th * dk,
                              c->dk_ + th * dk, c->dv_ + th * dv, c->dg + th * dk,
                              c->dbeta + th, Sp, w, w + dv, w + 2 * dv);
        }
    }
    if (c->d_init) memcpy(c->d_init + ((size_t)r * H + h) * ss, dS, ss * sizeof(double));
done:
    free(ck); free(blk); free(dS); free(Sp); free(w);
}

/* Gradients of L = sum(dO * o) + sum(dS_final * S_final) with respect to
 * q, k, v, g, beta and the initial state, for the same packed requests as
 * oracle_kda_prefill.  d_o / d_final / initial_state may be NULL (zeros);
 * d_initial may be NULL (not returned). */
int oracle_kda_prefill_backward(int n_req, const int64_t *cu_seqlens, int H, int dk, int dv,
                                const double *q, const double *k, const double *v,
                                const double *g, const double *beta,
                                const double *initial_state, const double *d_o,
                                const double *d_final, double *dq, double *dk_out,
                                double *dv_out, double *dg, double *dbeta,
                                double *d_initial, int n_threads) {
    backward_ctx c;
    int r;
    if (n_req < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens) return ORACLE_EINVAL;
    if (!dq || !dk_out || !dv_out || !dg || !dbeta) return ORACLE_EINVAL;
    for (r = 0; r < n_req; ++r)
        if (cu_seqlens[r + 1] < cu_seqlens[r]) return ORACLE_EINVAL;
    c.H = H; c.dk = dk; c.dv = dv; c.cu = cu_seqlens;
    c.q = q; c.k = k; c.v = v; c.g = g; c.beta = beta; c.s0 = initial_state;
    c.d_o = d_o; c.d_final = d_final;
    c.dq = dq; c.dk_ = dk_out; c.dv_ = dv_out; c.dg = dg; c.dbeta = dbeta; c.d_init = d_initial;
    run_jobs(backward_job, &c, (long)n_req * H, n_threads);
    return ORACLE_OK;
}
