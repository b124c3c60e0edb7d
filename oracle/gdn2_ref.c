/*
 * gdn2_ref.c -- plain fp64 CPU oracle for the Gated DeltaNet-2 recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code with the
 * CUDA path.
 *
 * What it computes (token form, one (batch, head) at a time, t = 1..T):
 *
 *   alpha_t = exp(g_t)                      channel-wise decay on the key axis
 *   S'      = Diag(alpha_t) S_{t-1}         decay is applied first
 *   e_t     = b_t (.) k_t                   erase gate weights the key used to read
 *   u_t     = w_t (.) v_t - S'^T e_t        write gate weights the candidate value,
 *                                           minus what the erase-weighted key reads
 *   S_t     = S' + k_t u_t^T                outer-product write
 *   o_t     = S_t^T q_t
 *
 * Sources: aixai.ru "Gated DeltaNet-2" post, section "Один скаляр не может
 * решать два разных вопроса" (prose statement of the update: decay first, read
 * by the key, erase gate on the key coordinates of the read, write gate on the
 * candidate value, outer-product write); aiexpert.news article, paragraph on
 * the gate definitions (b_t in [0,1]^{d_k} on the key side, w_t in [0,1]^{d_v}
 * on the value side, exact reduction to KDA when both gates collapse to one
 * scalar).  With b_t = w_t = beta_t 1 this is KDA's
 * S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T, o_t = S_t^T q_t.
 *
 * Layouts (all double, contiguous): q, k, b, g: [B,T,H,Dk]; v, w, o, do:
 * [B,T,H,Dv]; S0, ST, dST, dS0: [B,H,Dk,Dv].  S0 / dST may be NULL (zeros);
 * ST may be NULL (not wanted).
 *
 * The backward is reverse-mode differentiation of the token recurrence above
 * (one token at a time, last token first).  It stores the state every CK
 * tokens and recomputes the states inside a block with exactly the forward's
 * operations, so the recomputed states are bit-identical to the forward's.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define CK 64

typedef struct {
    int B, T, H, Dk, Dv;
    const double *q, *k, *v, *g, *b, *w, *S0, *dout, *dST;
    double *o, *ST;
    double *dq, *dk, *dv, *dg, *db, *dw, *dS0;
    int mode; /* 0 forward, 1 backward */
    int next;  /* next (b,h) index to claim */
    pthread_mutex_t lock;
    int err;
} job_t;

/* One token of the forward recurrence.  S (Dk x Dv, row-major) is updated in
 * place; Sp receives S' = Diag(alpha) S_{t-1}; u receives u_t.  Returns o_t in
 * o (may be NULL). */
static void token_step(int Dk, int Dv, const double *q, const double *k, const double *v,
                       const double *g, const double *b, const double *w,
                       double *S, double *u, double *o)
{
    /* S' = Diag(alpha) S */
    for (int i = 0; i < Dk; ++i) {
        double a = exp(g[i]);
        double *row = S + (size_t)i * Dv;
        for (int j = 0; j < Dv; ++j) row[j] *= a;
    }
    /* u = w.v - S'^T (b.k) */
    for (int j = 0; j < Dv; ++j) u[j] = w[j] * v[j];
    for (int i = 0; i < Dk; ++i) {
        double e = b[i] * k[i];
        const double *row = S + (size_t)i * Dv;
        for (int j = 0; j < Dv; ++j) u[j] -= row[j] * e;
    }
    /* S = S' + k u^T */
    for (int i = 0; i < Dk; ++i) {
        double *row = S + (size_t)i * Dv;
        for (int j = 0; j < Dv; ++j) row[j] += k[i] * u[j];
    }
    /* o = S^T q */
    if (o) {
        for (int j = 0; j < Dv; ++j) o[j] = 0.0;
        for (int i = 0; i < Dk; ++i) {
            const double *row = S + (size_t)i * Dv;
            for (int j = 0; j < Dv; ++j) o[j] += row[j] * q[i];
        }
    }
}

static int fwd_one(job_t *J, int bh)
{
    const int T = J->T, H = J->H, Dk = J->Dk, Dv = J->Dv;
    const int bb = bh / H, hh = bh % H;
    const size_t sk = (size_t)H * Dk, sv = (size_t)H * Dv; /* token strides */
    const size_t offk = ((size_t)bb * T * H + hh) * Dk, offv = ((size_t)bb * T * H + hh) * Dv;
    const size_t offS = (size_t)bh * Dk * Dv;
    double *S = (double *)malloc(sizeof(double) * ((size_t)Dk * Dv + Dv));
    if (!S) return 1;
    double *u = S + (size_t)Dk * Dv;
    if (J->S0) memcpy(S, J->S0 + offS, sizeof(double) * Dk * Dv);
    else memset(S, 0, sizeof(double) * Dk * Dv);
    for (int t = 0; t < T; ++t) {
        token_step(Dk, Dv, J->q + offk + t * sk, J->k + offk + t * sk, J->v + offv + t * sv,
                   J->g + offk + t * sk, J->b + offk + t * sk, J->w + offv + t * sv,
                   S, u, J->o ? J->o + offv + t * sv : NULL);
    }
    if (J->ST) memcpy(J->ST + offS, S, sizeof(double) * Dk * Dv);
    free(S);
    return 0;
}

static int bwd_one(job_t *J, int bh)
{
    const int T = J->T, H = J->H, Dk = J->Dk, Dv = J->Dv;
    const int bb = bh / H, hh = bh % H;
    const size_t sk = (size_t)H * Dk, sv = (size_t)H * Dv;
    const size_t offk = ((size_t)bb * T * H + hh) * Dk, offv = ((size_t)bb * T * H + hh) * Dv;
    const size_t offS = (size_t)bh * Dk * Dv, DD = (size_t)Dk * Dv;
    const int nblk = (T + CK - 1) / CK;
    /* checkpoints: state before each block; block states: state after each token of a block */
    double *ckpt = (double *)malloc(sizeof(double) * DD * (size_t)(nblk > 0 ? nblk : 1));
    double *blk = (double *)malloc(sizeof(double) * DD * (CK + 1));
    double *dS = (double *)malloc(sizeof(double) * DD);
    double *dSp = (double *)malloc(sizeof(double) * DD);
    double *Sp = (double *)malloc(sizeof(double) * DD);
    double *vec = (double *)malloc(sizeof(double) * (size_t)(4 * Dv + 4 * Dk));
    if (!ckpt || !blk || !dS || !dSp || !Sp || !vec) {
        free(ckpt); free(blk); free(dS); free(dSp); free(Sp); free(vec);
        return 1;
    }
    double *u = vec, *du = vec + Dv, *dov = vec + 2 * Dv;
    double *e = vec + 4 * Dv, *de = e + Dk;

    /* forward pass storing block checkpoints */
    double *S = blk; /* running state */
    if (J->S0) memcpy(S, J->S0 + offS, sizeof(double) * DD);
    else memset(S, 0, sizeof(double) * DD);
    for (int t = 0; t < T; ++t) {
        if (t % CK == 0) memcpy(ckpt + (size_t)(t / CK) * DD, S, sizeof(double) * DD);
        token_step(Dk, Dv, J->q + offk + t * sk, J->k + offk + t * sk, J->v + offv + t * sv,
                   J->g + offk + t * sk, J->b + offk + t * sk, J->w + offv + t * sv, S, u, NULL);
    }
    /* dS <- dS_T */
    if (J->dST) memcpy(dS, J->dST + offS, sizeof(double) * DD);
    else memset(dS, 0, sizeof(double) * DD);

    for (int c = nblk - 1; c >= 0; --c) {
        const int t0 = c * CK, t1 = (t0 + CK < T) ? t0 + CK : T;
        /* recompute states after each token of the block: blk[s] = S_{t0+s} (state after t0+s-1) */
        memcpy(blk, ckpt + (size_t)c * DD, sizeof(double) * DD);
        for (int t = t0; t < t1; ++t) {
            double *dst = blk + (size_t)(t - t0 + 1) * DD;
            memcpy(dst, blk + (size_t)(t - t0) * DD, sizeof(double) * DD);
            token_step(Dk, Dv, J->q + offk + t * sk, J->k + offk + t * sk, J->v + offv + t * sv,
                       J->g + offk + t * sk, J->b + offk + t * sk, J->w + offv + t * sv, dst, u, NULL);
        }
        for (int t = t1 - 1; t >= t0; --t) {
            const double *qt = J->q + offk + t * sk, *kt = J->k + offk + t * sk;
            const double *vt = J->v + offv + t * sv, *gt = J->g + offk + t * sk;
            const double *bt = J->b + offk + t * sk, *wt = J->w + offv + t * sv;
            const double *St = blk + (size_t)(t - t0 + 1) * DD;   /* S_t */
            const double *Sm = blk + (size_t)(t - t0) * DD;       /* S_{t-1} */
            for (int j = 0; j < Dv; ++j) dov[j] = J->dout[offv + t * sv + j];
            /* recompute S' = Diag(alpha) S_{t-1}, e, u (same operations as the forward) */
            for (int i = 0; i < Dk; ++i) {
                double a = exp(gt[i]);
                for (int j = 0; j < Dv; ++j) Sp[(size_t)i * Dv + j] = Sm[(size_t)i * Dv + j] * a;
            }
            for (int j = 0; j < Dv; ++j) u[j] = wt[j] * vt[j];
            for (int i = 0; i < Dk; ++i) {
                e[i] = bt[i] * kt[i];
                for (int j = 0; j < Dv; ++j) u[j] -= Sp[(size_t)i * Dv + j] * e[i];
            }
            /* (1) o_t = S_t^T q_t: dS += q do^T, dq = S_t do */
            double *dqt = J->dq + offk + t * sk;
            for (int i = 0; i < Dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < Dv; ++j) {
                    dS[(size_t)i * Dv + j] += qt[i] * dov[j];
                    acc += St[(size_t)i * Dv + j] * dov[j];
                }
                dqt[i] = acc;
            }
            /* (2) S_t = S' + k u^T: dk = dS u, du = dS^T k, dS' = dS */
            double *dkt = J->dk + offk + t * sk;
            for (int j = 0; j < Dv; ++j) du[j] = 0.0;
            for (int i = 0; i < Dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < Dv; ++j) {
                    acc += dS[(size_t)i * Dv + j] * u[j];
                    du[j] += dS[(size_t)i * Dv + j] * kt[i];
                }
                dkt[i] = acc;
            }
            memcpy(dSp, dS, sizeof(double) * DD);
            /* (3) u = w.v - S'^T e: dw, dv; dS' -= e du^T; de = -S' du */
            double *dwt = J->dw + offv + t * sv, *dvt = J->dv + offv + t * sv;
            for (int j = 0; j < Dv; ++j) { dwt[j] = du[j] * vt[j]; dvt[j] = du[j] * wt[j]; }
            for (int i = 0; i < Dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < Dv; ++j) {
                    dSp[(size_t)i * Dv + j] -= e[i] * du[j];
                    acc += Sp[(size_t)i * Dv + j] * du[j];
                }
                de[i] = -acc;
            }
            /* (4) e = b.k: db = de.k, dk += de.b */
            double *dbt = J->db + offk + t * sk;
            for (int i = 0; i < Dk; ++i) { dbt[i] = de[i] * kt[i]; dkt[i] += de[i] * bt[i]; }
            /* (5) S' = Diag(exp g) S_{t-1}: dg_i = sum_j dS'_ij S'_ij; dS_{t-1} = Diag(alpha) dS' */
            double *dgt = J->dg + offk + t * sk;
            for (int i = 0; i < Dk; ++i) {
                double a = exp(gt[i]), acc = 0.0;
                for (int j = 0; j < Dv; ++j) {
                    acc += dSp[(size_t)i * Dv + j] * Sp[(size_t)i * Dv + j];
                    dS[(size_t)i * Dv + j] = a * dSp[(size_t)i * Dv + j];
                }
                dgt[i] = acc;
            }
        }
    }
    memcpy(J->dS0 + offS, dS, sizeof(double) * DD);
    free(ckpt); free(blk); free(dS); free(dSp); free(Sp); free(vec);
    return 0;
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int bh = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (bh >= J->B * J->H) break;
        int rc = J->mode == 0 ? fwd_one(J, bh) : bwd_one(J, bh);
        if (rc) {
            pthread_mutex_lock(&J->lock);
            J->err = rc;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

static int run(job_t *J, int nthreads)
{
    if (J->B < 0 || J->T < 0 || J->H <= 0 || J->Dk <= 0 || J->Dv <= 0) return -2;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > J->B * J->H) nthreads = J->B * J->H > 0 ? J->B * J->H : 1;
    J->next = 0;
    J->err = 0;
    pthread_mutex_init(&J->lock, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -1;
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, worker, J) == 0) ++started;
    if (started == 0) worker(J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return J->err ? -1 : 0;
}

/* Forward: o [B,T,H,Dv] (may be NULL), ST [B,H,Dk,Dv] (may be NULL). */
int gdn2_ref_fwd(int B, int T, int H, int Dk, int Dv,
                 const double *q, const double *k, const double *v, const double *g,
                 const double *b, const double *w, const double *S0,
                 double *o, double *ST, int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof(J));
    J.B = B; J.T = T; J.H = H; J.Dk = Dk; J.Dv = Dv;
    J.q = q; J.k = k; J.v = v; J.g = g; J.b = b; J.w = w; J.S0 = S0;
    J.o = o; J.ST = ST; J.mode = 0;
    return run(&J, nthreads);
}

/* Backward of L = <o, dout> + <S_T, dST> with respect to every input and S0. */
int gdn2_ref_bwd(int B, int T, int H, int Dk, int Dv,
                 const double *q, const double *k, const double *v, const double *g,
                 const double *b, const double *w, const double *S0,
                 const double *dout, const double *dST,
                 double *dq, double *dk, double *dv, double *dg, double *db, double *dw,
                 double *dS0, int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof(J));
    J.B = B; J.T = T; J.H = H; J.Dk = Dk; J.Dv = Dv;
    J.q = q; J.k = k; J.v = v; J.g = g; J.b = b; J.w = w; J.S0 = S0;
    J.dout = dout; J.dST = dST;
    J.dq = dq; J.dk = dk; J.dv = dv; J.dg = dg; J.db = db; J.dw = dw; J.dS0 = dS0;
    J.mode = 1;
    return run(&J, nthreads);
}

/* One decode step for N sequences: S [N,H,Dk,Dv] updated in place, o [N,H,Dv]. */
int gdn2_ref_decode(int N, int H, int Dk, int Dv,
                    const double *q, const double *k, const double *v, const double *g,
                    const double *b, const double *w, double *S, double *o, int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof(J));
    J.B = N; J.T = 1; J.H = H; J.Dk = Dk; J.Dv = Dv;
    J.q = q; J.k = k; J.v = v; J.g = g; J.b = b; J.w = w; J.S0 = S;
    J.o = o; J.ST = S; J.mode = 0;
    return run(&J, nthreads);
}
