/*
 * kda_oracle.c — fp64 CPU oracle for the Kimi Delta Attention (KDA) recurrence.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the independent checker for the CUDA
 * library: only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg may build, load or call it. The product path never routes through it, and
 * it shares no source, header, helper or constant with the CUDA kernels.
 *
 * What it computes (source: "Kimi Linear：让长上下文大模型真正实用的线性注意力架构",
 * juejin.cn, section 三 5️⃣ "Attention 的新解释：在线梯度下降（Delta Rule）", the
 * KDA update rule, with the symbol roles listed right below it: beta = learning
 * rate, alpha = forget rate, S = memory state; section 三 1️⃣ gives one forget
 * rate per channel):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *
 * with S in R^{dk x dv}, alpha_t = exp(log_alpha_t) in (0,1]^{dk} (one rate per
 * key channel, i.e. per ROW of S), beta_t a scalar per token and head. The page
 * prints no read-out; this oracle reads out with the post-update state,
 * o_t = scale * S_t^T q_t, and applies scale to the read-out only.
 *
 * Per token, in the order the equation applies its factors:
 *   1. S' = Diag(alpha_t) S_{t-1}            (row i scaled by alpha_t[i])
 *   2. S_t = S' - beta_t k_t (k_t^T S') + beta_t k_t v_t^T
 *          (the product (I - beta k k^T) S' written out without forming I)
 *   3. o_t = scale * S_t^T q_t
 *
 * Plain token-by-token loops in double precision; no chunking, no blocking, no
 * reordering. Work is split over (sequence, head) units with POSIX threads: the
 * units are independent, so the split does not change any arithmetic.
 *
 * Layouts (all row-major, contiguous, double):
 *   q, k       [B, T, H, dk]       v, o     [B, T, H, dv]
 *   log_alpha  [B, T, H, dk]       beta     [B, T, H]
 *   S0, S_final[N, H, dk, dv]      (N = B, or n_seqs when cu_seqlens is given)
 * With cu_seqlens (int64, n_seqs+1 prefix offsets, B must be 1) sequence n owns
 * tokens [cu_seqlens[n], cu_seqlens[n+1]) of the packed time axis and starts
 * from S0[n]. S0 may be NULL (zero state); S_final may be NULL (not returned).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *S0;
    const int64_t *cu_seqlens;
    int B, T, H, dk, dv, n_seqs;
    double scale;
    double *o, *S_final;
    int n_units;
    int next_unit; /* guarded by lock */
    pthread_mutex_t lock;
} job_t;

/* One token of the recurrence on a single head's state S[dk][dv]. The token's
 * vectors are given by pointer; o_t is written to o (may be NULL). tmp holds dv
 * doubles of scratch. */
static void kda_token(double *S, int dk, int dv, const double *q, const double *k,
                      const double *v, const double *log_alpha, double beta,
                      double scale, double *o, double *tmp)
{
    /* 1. S' = Diag(alpha) S: alpha acts on the key channel (row) index. */
    for (int i = 0; i < dk; ++i) {
        const double a = exp(log_alpha[i]);
        for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;
    }
    /* 2. kS = k^T S' (a row vector over dv), then
     *    S_t = S' - beta k (k^T S') + beta k v^T. */
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += k[i] * S[i * dv + j];
        tmp[j] = acc;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[i * dv + j] += -beta * k[i] * tmp[j] + beta * k[i] * v[j];
    /* 3. o_t = scale * S_t^T q with the updated state. */
    if (o) {
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * q[i];
            o[j] = scale * acc;
        }
    }
}

static void run_unit(job_t *J, int unit, double *S, double *tmp)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const int n = unit / H, h = unit % H;
    int64_t t0, t1;
    if (J->cu_seqlens) {
        t0 = J->cu_seqlens[n];
        t1 = J->cu_seqlens[n + 1];
    } else {
        t0 = (int64_t)n * J->T;
        t1 = t0 + J->T;
    }
    const size_t sidx = ((size_t)n * H + h) * (size_t)dk * dv;
    if (J->S0) memcpy(S, J->S0 + sidx, sizeof(double) * (size_t)dk * dv);
    else memset(S, 0, sizeof(double) * (size_t)dk * dv);
    /* The packed time axis: [B,T,H,d] with B sequences of length T is the same
     * memory as one packed axis of B*T tokens. */
    for (int64_t t = t0; t < t1; ++t) {
        const size_t th = (size_t)t * H + h;
        kda_token(S, dk, dv, J->q + th * dk, J->k + th * dk, J->v + th * dv,
                  J->log_alpha + th * dk, J->beta[th], J->scale,
                  J->o ? J->o + th * dv : NULL, tmp);
    }
    if (J->S_final) memcpy(J->S_final + sidx, S, sizeof(double) * (size_t)dk * dv);
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)J->dk * J->dv);
    double *tmp = (double *)malloc(sizeof(double) * (size_t)J->dv);
    if (!S || !tmp) { free(S); free(tmp); return (void *)1; }
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->n_units) break;
        run_unit(J, u, S, tmp);
    }
    free(S);
    free(tmp);
    return NULL;
}

int kda_oracle_num_threads(int requested)
{
    if (requested > 0) return requested;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* Full-sequence forward. Returns 0 on success, nonzero on bad arguments or
 * allocation failure. n_threads <= 0 uses every online core. */
int kda_oracle_forward(const double *q, const double *k, const double *v,
                       const double *log_alpha, const double *beta, const double *S0,
                       const int64_t *cu_seqlens, int n_seqs, int B, int T, int H,
                       int dk, int dv, double scale, double *o, double *S_final,
                       int n_threads)
{
    if (!q || !k || !v || !log_alpha || !beta || B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1)
        return 1;
    if (cu_seqlens && (B != 1 || n_seqs < 1 || cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != T))
        return 1;
    if (cu_seqlens)
        for (int n = 0; n < n_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
    job_t J;
    J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta; J.S0 = S0;
    J.cu_seqlens = cu_seqlens;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
    J.n_seqs = cu_seqlens ? n_seqs : B;
    J.scale = scale; J.o = o; J.S_final = S_final;
    J.n_units = J.n_seqs * H;
    J.next_unit = 0;
    pthread_mutex_init(&J.lock, NULL);
    int nt = kda_oracle_num_threads(n_threads);
    if (nt > J.n_units) nt = J.n_units;
    if (nt < 1) nt = 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    int rc = th ? 0 : 2;
    int started = 0;
    for (int i = 0; i < nt && rc == 0; ++i) {
        if (pthread_create(&th[i], NULL, worker, &J) != 0) rc = 2;
        else ++started;
    }
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret) rc = 2;
    }
    if (started == 0 && rc == 0) rc = 2;
    free(th);
    pthread_mutex_destroy(&J.lock);
    return rc;
}

/* One recurrent decode step: N independent sequences, one new token each.
 * q, k, log_alpha [N,H,dk]; v, o [N,H,dv]; beta [N,H]; S [N,H,dk,dv] is
 * updated in place. This is the forward with T = 1 and S0 = S_final = S. */
int kda_oracle_decode_step(const double *q, const double *k, const double *v,
                           const double *log_alpha, const double *beta, double *S,
                           int N, int H, int dk, int dv, double scale, double *o,
                           int n_threads)
{
    if (!S) return 1;
    return kda_oracle_forward(q, k, v, log_alpha, beta, S, NULL, 0, N, 1, H, dk, dv,
                              scale, o, S, n_threads);
}

/* ------------------------------------------------------------------ backward
 * Reverse-mode derivatives of
 *     L = <dO, o> + <dS_final, S_final>
 * (dO [B,T,H,dv]; dS_final [N,H,dk,dv] or NULL for zero) with respect to q, k,
 * v, log_alpha, beta and S0, for training; the page states only the forward
 * rule, so this is its derivative, taken step by step. With G = dL/dS_t, the
 * gradient reaching the state after token t, each token's three steps are
 * differentiated in reverse order:
 *   3. o_t = scale S_t^T q_t:   G += scale q_t dO_t^T;   dq_t = scale S_t dO_t
 *   2. S_t = S' + beta k w^T with w = v - S'^T k:
 *        g = G^T k (over dv);  dv_t = beta g;  dbeta_t = g . w;
 *        dk_t = beta (G w - S' g);  dS' = G - beta k g^T
 *   1. S' = Diag(alpha) S_{t-1}: dlog_alpha_t[i] = sum_j dS'_ij S'_ij;
 *        G <- Diag(alpha) dS'  (= dL/dS_{t-1})
 * and dS0 = G once the first token is undone. S_{t-1} and S_t come from a
 * replay of the forward (the same per-token routine): the state is kept every
 * CKPT tokens, and each block of tokens is replayed from its checkpoint,
 * keeping its states, then walked backwards. Gradients have the layouts of
 * their inputs.
 */
#define CKPT 64

typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *S0, *dO, *dS_final;
    const int64_t *cu_seqlens;
    int T, H, dk, dv;
    double scale;
    double *gq, *gk, *gv, *gla, *gbeta, *gS0;
    int n_units;
    int next_unit; /* guarded by lock */
    pthread_mutex_t lock;
} bjob_t;

static int run_bunit(bjob_t *J, int unit)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const size_t dkdv = (size_t)dk * dv;
    const int n = unit / H, h = unit % H;
    int64_t t0, t1;
    if (J->cu_seqlens) {
        t0 = J->cu_seqlens[n];
        t1 = J->cu_seqlens[n + 1];
    } else {
        t0 = (int64_t)n * J->T;
        t1 = t0 + J->T;
    }
    const int64_t L = t1 - t0;
    const int64_t ncp = (L + CKPT - 1) / CKPT;
    const size_t sidx = ((size_t)n * H + h) * dkdv;
    double *ckpt = (double *)malloc(sizeof(double) * dkdv * (size_t)(ncp > 0 ? ncp : 1));
    double *blk = (double *)malloc(sizeof(double) * dkdv * (CKPT + 1));
    double *G = (double *)malloc(sizeof(double) * dkdv);
    double *Sp = (double *)malloc(sizeof(double) * dkdv);
    double *vecs = (double *)malloc(sizeof(double) * (size_t)(3 * dv + dk));
    if (!ckpt || !blk || !G || !Sp || !vecs) {
        free(ckpt); free(blk); free(G); free(Sp); free(vecs);
        return 1;
    }
    double *w = vecs, *g = vecs + dv, *tmp = vecs + 2 * dv, *alpha = vecs + 3 * dv;
    /* forward, keeping the state before every CKPT-th token */
    double *S = blk;
    if (J->S0) memcpy(S, J->S0 + sidx, sizeof(double) * dkdv);
    else memset(S, 0, sizeof(double) * dkdv);
    for (int64_t t = t0; t < t1; ++t) {
        if ((t - t0) % CKPT == 0) memcpy(ckpt + (size_t)((t - t0) / CKPT) * dkdv, S, sizeof(double) * dkdv);
        const size_t th = (size_t)t * H + h;
        kda_token(S, dk, dv, J->q + th * dk, J->k + th * dk, J->v + th * dv,
                  J->log_alpha + th * dk, J->beta[th], J->scale, NULL, tmp);
    }
    if (J->dS_final) memcpy(G, J->dS_final + sidx, sizeof(double) * dkdv);
    else memset(G, 0, sizeof(double) * dkdv);
    for (int64_t b = ncp - 1; b >= 0; --b) {
        const int64_t a = t0 + b * CKPT, e = (a + CKPT < t1) ? a + CKPT : t1;
        /* replay: blk[s] = state before token a + s, blk[e - a] = after the block */
        memcpy(blk, ckpt + (size_t)b * dkdv, sizeof(double) * dkdv);
        for (int64_t t = a; t < e; ++t) {
            double *nx = blk + (size_t)(t - a + 1) * dkdv;
            memcpy(nx, blk + (size_t)(t - a) * dkdv, sizeof(double) * dkdv);
            const size_t th = (size_t)t * H + h;
            kda_token(nx, dk, dv, J->q + th * dk, J->k + th * dk, J->v + th * dv,
                      J->log_alpha + th * dk, J->beta[th], J->scale, NULL, tmp);
        }
        for (int64_t t = e - 1; t >= a; --t) {
            const double *P = blk + (size_t)(t - a) * dkdv;      /* S_{t-1} */
            const double *Q = blk + (size_t)(t - a + 1) * dkdv;  /* S_t */
            const size_t th = (size_t)t * H + h;
            const double *qt = J->q + th * dk, *kt = J->k + th * dk, *vt = J->v + th * dv;
            const double *lat = J->log_alpha + th * dk, *dOt = J->dO + th * dv;
            const double bt = J->beta[th];
            /* 3. read-out */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) G[i * dv + j] += J->scale * qt[i] * dOt[j];
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += Q[i * dv + j] * dOt[j];
                J->gq[th * dk + i] = J->scale * acc;
            }
            /* 2. delta update */
            for (int i = 0; i < dk; ++i) {
                alpha[i] = exp(lat[i]);
                for (int j = 0; j < dv; ++j) Sp[i * dv + j] = alpha[i] * P[i * dv + j];
            }
            double db = 0.0;
            for (int j = 0; j < dv; ++j) {
                double sk = 0.0, gk_ = 0.0;
                for (int i = 0; i < dk; ++i) {
                    sk += Sp[i * dv + j] * kt[i];
                    gk_ += G[i * dv + j] * kt[i];
                }
                w[j] = vt[j] - sk;
                g[j] = gk_;
                J->gv[th * dv + j] = bt * gk_;
                db += gk_ * w[j];
            }
            J->gbeta[th] = db;
            for (int i = 0; i < dk; ++i) {
                double gw = 0.0, sg = 0.0;
                for (int j = 0; j < dv; ++j) {
                    gw += G[i * dv + j] * w[j];
                    sg += Sp[i * dv + j] * g[j];
                }
                J->gk[th * dk + i] = bt * (gw - sg);
            }
            /* dS' = G - beta k g^T, overwriting G; then 1. the decay */
            for (int i = 0; i < dk; ++i) {
                double dl = 0.0;
                for (int j = 0; j < dv; ++j) {
                    const double d = G[i * dv + j] - bt * kt[i] * g[j];
                    dl += d * Sp[i * dv + j];
                    G[i * dv + j] = alpha[i] * d;
                }
                J->gla[th * dk + i] = dl;
            }
        }
    }
    if (J->gS0) memcpy(J->gS0 + sidx, G, sizeof(double) * dkdv);
    free(ckpt); free(blk); free(G); free(Sp); free(vecs);
    return 0;
}

static void *bworker(void *arg)
{
    bjob_t *J = (bjob_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->n_units) break;
        if (run_bunit(J, u)) return (void *)1;
    }
    return NULL;
}

/* Backward of kda_oracle_forward (see above). dO and every gradient array but
 * gS0 must be given; dS_final and gS0 may be NULL. Returns 0 on success,
 * nonzero on bad arguments or allocation failure. */
int kda_oracle_backward(const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *beta, const double *S0,
                        const int64_t *cu_seqlens, int n_seqs, int B, int T, int H, int dk,
                        int dv, double scale, const double *dO, const double *dS_final,
                        double *gq, double *gk, double *gv, double *glog_alpha, double *gbeta,
                        double *gS0, int n_threads)
{
    if (!q || !k || !v || !log_alpha || !beta || !dO || !gq || !gk || !gv || !glog_alpha ||
        !gbeta || B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1)
        return 1;
    if (cu_seqlens && (B != 1 || n_seqs < 1 || cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != T))
        return 1;
    if (cu_seqlens)
        for (int n = 0; n < n_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
    bjob_t J;
    J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta; J.S0 = S0;
    J.dO = dO; J.dS_final = dS_final; J.cu_seqlens = cu_seqlens;
    J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.scale = scale;
    J.gq = gq; J.gk = gk; J.gv = gv; J.gla = glog_alpha; J.gbeta = gbeta; J.gS0 = gS0;
    J.n_units = (cu_seqlens ? n_seqs : B) * H;
    J.next_unit = 0;
    pthread_mutex_init(&J.lock, NULL);
    int nt = kda_oracle_num_threads(n_threads);
    if (nt > J.n_units) nt = J.n_units;
    if (nt < 1) nt = 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    int rc = th ? 0 : 2;
    int started = 0;
    for (int i = 0; i < nt && rc == 0; ++i) {
        if (pthread_create(&th[i], NULL, bworker, &J) != 0) rc = 2;
        else ++started;
    }
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret) rc = 2;
    }
    if (started == 0 && rc == 0) rc = 2;
    free(th);
    pthread_mutex_destroy(&J.lock);
    return rc;
}
