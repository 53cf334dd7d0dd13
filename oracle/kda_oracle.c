/*
 * kda_oracle.c -- plain fp64 CPU oracle for the KDA (Kimi Delta Attention)
 * channel-wise gated delta-rule recurrence.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
 * call this file: only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg use it. It shares no code, header, table or
 * constant with the CUDA library.
 *
 * What it computes (sources are the pages "22580: from GPT-2 to Kimi K3,
 * explained" (temp07.ru), its English original (marvinlee.cn), the Chinese
 * digest (wps.hkprog.org) and the KDA explainer (ai-flip.ru)):
 *
 *   DeltaNet forward with a cache, section "DeltaNet, or Fast Weight
 *   Programmers": read the board at the key (v_old = k S), form the delta
 *   u = beta (v - v_old), write S += k^T u, read out o = q S with no
 *   denominator. The state S is dk x dv (the code's orientation).
 *
 *   Gated DeltaNet, section "Gated Delta Net": a decay alpha multiplies the
 *   previous state before the delta write; alpha = 1 is the pure delta rule,
 *   alpha = 0 clears the memory.
 *
 *   KDA, section "KDA / Kimi Linear" and the ai-flip.ru section on
 *   channel-wise gating: the scalar decay becomes a diagonal matrix, one
 *   decay per key channel.
 *
 * Per sequence and head, for every token t in order:
 *     S'  = Diag(alpha_t) S            alpha_t = exp(log_alpha_t), per key row
 *     r   = S'^T k_t                   (the value the key currently reads)
 *     d   = beta_t (v_t - r)
 *     S   = S' + k_t d^T
 *     o_t = S^T q_t                    (read-out after the write)
 * The read uses the decayed state S' (the only reading under which alpha = 0
 * clears memory and the step equals (I - beta k k^T) Diag(alpha) S + beta k v^T,
 * the transposed Householder form of the "DeltaNet, or Parallelizing Linear
 * Transformers with Delta Rule" section, with the gate inserted).
 *
 * Everything is fp64; exp(-inf) = 0 gives an exact clear. No blocking, no
 * reordering: one token at a time, sums over the key index in index order.
 * Work is split over (sequence, head) pairs with POSIX threads; each pair is
 * independent, so the result does not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *init_state;
    const int64_t *cu_seqlens;
    int n_seq, H, dk, dv;
    double *o, *final_state;
    int next;              /* next (sequence, head) pair to take */
    int failed;
    pthread_mutex_t lock;
} oracle_job;

/* One (sequence, head) chain: the token loop above. */
static int run_chain(oracle_job *job, int seq, int h)
{
    const int H = job->H, dk = job->dk, dv = job->dv;
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *r = (double *)malloc(sizeof(double) * (size_t)dv);
    double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
    if (!S || !r || !alpha) {
        free(S); free(r); free(alpha);
        return -1;
    }
    const size_t state_off = ((size_t)seq * H + h) * (size_t)dk * dv;
    if (job->init_state)
        memcpy(S, job->init_state + state_off, sizeof(double) * (size_t)dk * dv);
    else
        memset(S, 0, sizeof(double) * (size_t)dk * dv);

    for (int64_t t = job->cu_seqlens[seq]; t < job->cu_seqlens[seq + 1]; ++t) {
        const double *qt = job->q + ((size_t)t * H + h) * dk;
        const double *kt = job->k + ((size_t)t * H + h) * dk;
        const double *vt = job->v + ((size_t)t * H + h) * dv;
        const double *lat = job->log_alpha + ((size_t)t * H + h) * dk;
        const double bt = job->beta[(size_t)t * H + h];
        double *ot = job->o + ((size_t)t * H + h) * dv;

        /* S' = Diag(alpha) S */
        for (int a = 0; a < dk; ++a) {
            alpha[a] = exp(lat[a]);
            for (int b = 0; b < dv; ++b)
                S[(size_t)a * dv + b] *= alpha[a];
        }
        /* r = S'^T k */
        for (int b = 0; b < dv; ++b) {
            double acc = 0.0;
            for (int a = 0; a < dk; ++a)
                acc += S[(size_t)a * dv + b] * kt[a];
            r[b] = acc;
        }
        /* S = S' + k (beta (v - r))^T */
        for (int b = 0; b < dv; ++b) {
            const double d = bt * (vt[b] - r[b]);
            for (int a = 0; a < dk; ++a)
                S[(size_t)a * dv + b] += kt[a] * d;
        }
        /* o = S^T q */
        for (int b = 0; b < dv; ++b) {
            double acc = 0.0;
            for (int a = 0; a < dk; ++a)
                acc += S[(size_t)a * dv + b] * qt[a];
            ot[b] = acc;
        }
    }
    if (job->final_state)
        memcpy(job->final_state + state_off, S, sizeof(double) * (size_t)dk * dv);
    free(S); free(r); free(alpha);
    return 0;
}

static void *worker(void *arg)
{
    oracle_job *job = (oracle_job *)arg;
    const int total = job->n_seq * job->H;
    for (;;) {
        pthread_mutex_lock(&job->lock);
        const int idx = job->next++;
        pthread_mutex_unlock(&job->lock);
        if (idx >= total)
            break;
        if (run_chain(job, idx / job->H, idx % job->H) != 0) {
            pthread_mutex_lock(&job->lock);
            job->failed = 1;
            pthread_mutex_unlock(&job->lock);
        }
    }
    return NULL;
}

/*
 * oracle_kda_forward: run the recurrence over packed sequences.
 *   q, k, log_alpha : [T_total, H, dk]   v, o : [T_total, H, dv]
 *   beta            : [T_total, H]
 *   init_state      : [n_seq, H, dk, dv] or NULL (zeros)
 *   final_state     : [n_seq, H, dk, dv] or NULL (not written)
 *   cu_seqlens      : [n_seq + 1], cu[0] = 0, non-decreasing; sequence i owns
 *                     tokens [cu[i], cu[i+1]).
 * A single decode step is the same call with every sequence one token long.
 * Returns 0 on success, -1 on bad arguments, -2 on allocation failure.
 */
int oracle_kda_forward(const double *q, const double *k, const double *v,
                       const double *log_alpha, const double *beta,
                       const double *init_state, const int64_t *cu_seqlens,
                       int n_seq, int H, int dk, int dv,
                       double *o, double *final_state, int n_threads)
{
    if (!q || !k || !v || !log_alpha || !beta || !cu_seqlens || !o)
        return -1;
    if (n_seq < 0 || H <= 0 || dk <= 0 || dv <= 0)
        return -1;
    if (cu_seqlens[0] != 0)
        return -1;
    for (int i = 0; i < n_seq; ++i)
        if (cu_seqlens[i + 1] < cu_seqlens[i])
            return -1;
    if (n_threads < 1)
        n_threads = 1;
    const int total = n_seq * H;
    if (n_threads > total)
        n_threads = total > 0 ? total : 1;

    oracle_job job;
    memset(&job, 0, sizeof(job));
    job.q = q; job.k = k; job.v = v; job.log_alpha = log_alpha; job.beta = beta;
    job.init_state = init_state; job.cu_seqlens = cu_seqlens;
    job.n_seq = n_seq; job.H = H; job.dk = dk; job.dv = dv;
    job.o = o; job.final_state = final_state;
    pthread_mutex_init(&job.lock, NULL);

    pthread_t *tids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!tids) {
        pthread_mutex_destroy(&job.lock);
        return -2;
    }
    int started = 0;
    for (int i = 1; i < n_threads; ++i) {
        if (pthread_create(&tids[i], NULL, worker, &job) != 0)
            break;
        ++started;
    }
    worker(&job); /* the calling thread works too */
    for (int i = 1; i <= started; ++i)
        pthread_join(tids[i], NULL);
    free(tids);
    pthread_mutex_destroy(&job.lock);
    return job.failed ? -2 : 0;
}


/*
 * Reverse mode of the same recurrence (the gradient a training step needs;
 * the pages motivate the chunk-wise form as hardware-efficient training,
 * "DeltaNet, or Parallelizing Linear Transformers with Delta Rule"). For one
 * chain, given dL/do_t for every token and dL/dS_T, it returns dL/dq_t,
 * dL/dk_t, dL/dv_t, dL/dlog_alpha_t, dL/dbeta_t and dL/dS_0.
 *
 * The forward states are recomputed and kept (T + 1 matrices per chain), then
 * the tokens are walked backwards with G = dL/dS_t:
 *     G += q_t do_t^T                 dq_t = S_t do_t            (o_t = S_t^T q_t)
 *     dd = G^T k_t                    dk_t = G d_t               (S_t = S' + k_t d_t^T)
 *     dbeta_t = dd . (v_t - r_t)      dv_t = beta_t dd           (d_t = beta_t (v_t - r_t))
 *     dr = -beta_t dd;  G' = G + k_t dr^T;  dk_t += S' dr         (r_t = S'^T k_t)
 *     dlog_alpha_t[i] = sum_j S'[i][j] G'[i][j]                   (S' = Diag(exp(la)) S_{t-1})
 *     G = Diag(alpha_t) G'
 * and dS_0 is the final G. Plain fp64, one token at a time, sums in index
 * order; threads over independent (sequence, head) chains.
 */
typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *init_state, *d_o, *d_final;
    const int64_t *cu_seqlens;
    int n_seq, H, dk, dv;
    double *dq, *dk_out, *dv_out, *dla, *dbeta, *d_init;
    int next, failed;
    pthread_mutex_t lock;
} oracle_bwd_job;

static int run_chain_bwd(oracle_bwd_job *job, int seq, int h)
{
    const int H = job->H, dk = job->dk, dv = job->dv;
    const int64_t t0 = job->cu_seqlens[seq], t1 = job->cu_seqlens[seq + 1];
    const int64_t L = t1 - t0;
    const size_t SZ = (size_t)dk * dv;
    /* states[0] = S_0, states[t + 1] = S after token t0 + t */
    double *states = (double *)malloc(sizeof(double) * SZ * (size_t)(L + 1));
    double *G = (double *)malloc(sizeof(double) * SZ);
    double *Sp = (double *)malloc(sizeof(double) * SZ);
    double *r = (double *)malloc(sizeof(double) * dv);
    double *d = (double *)malloc(sizeof(double) * dv);
    double *dd = (double *)malloc(sizeof(double) * dv);
    double *dr = (double *)malloc(sizeof(double) * dv);
    double *alpha = (double *)malloc(sizeof(double) * dk);
    if (!states || !G || !Sp || !r || !d || !dd || !dr || !alpha) {
        free(states); free(G); free(Sp); free(r); free(d); free(dd); free(dr); free(alpha);
        return -1;
    }
    const size_t state_off = ((size_t)seq * H + h) * SZ;
    if (job->init_state)
        memcpy(states, job->init_state + state_off, sizeof(double) * SZ);
    else
        memset(states, 0, sizeof(double) * SZ);

    /* forward, keeping every state */
    for (int64_t t = 0; t < L; ++t) {
        const size_t tok = (size_t)(t0 + t) * H + h;
        const double *kt = job->k + tok * dk, *vt = job->v + tok * dv;
        const double *lat = job->log_alpha + tok * dk;
        const double bt = job->beta[tok];
        double *S = states + (size_t)(t + 1) * SZ;
        memcpy(S, states + (size_t)t * SZ, sizeof(double) * SZ);
        for (int a = 0; a < dk; ++a) {
            const double al = exp(lat[a]);
            for (int b = 0; b < dv; ++b) S[(size_t)a * dv + b] *= al;
        }
        for (int b = 0; b < dv; ++b) {
            double acc = 0.0;
            for (int a = 0; a < dk; ++a) acc += S[(size_t)a * dv + b] * kt[a];
            r[b] = acc;
        }
        for (int b = 0; b < dv; ++b) {
            const double db = bt * (vt[b] - r[b]);
            for (int a = 0; a < dk; ++a) S[(size_t)a * dv + b] += kt[a] * db;
        }
    }

    /* backward */
    if (job->d_final)
        memcpy(G, job->d_final + state_off, sizeof(double) * SZ);
    else
        memset(G, 0, sizeof(double) * SZ);
    for (int64_t t = L - 1; t >= 0; --t) {
        const size_t tok = (size_t)(t0 + t) * H + h;
        const double *qt = job->q + tok * dk, *kt = job->k + tok * dk, *vt = job->v + tok * dv;
        const double *lat = job->log_alpha + tok * dk, *dot = job->d_o + tok * dv;
        const double bt = job->beta[tok];
        const double *Sprev = states + (size_t)t * SZ, *S = states + (size_t)(t + 1) * SZ;
        double *dqt = job->dq + tok * dk, *dkt = job->dk_out + tok * dk;
        double *dvt = job->dv_out + tok * dv, *dlat = job->dla + tok * dk;

        /* recompute S' = Diag(alpha) S_{t-1}, r = S'^T k, d = beta (v - r) */
        for (int a = 0; a < dk; ++a) {
            alpha[a] = exp(lat[a]);
            for (int b = 0; b < dv; ++b) Sp[(size_t)a * dv + b] = alpha[a] * Sprev[(size_t)a * dv + b];
        }
        for (int b = 0; b < dv; ++b) {
            double acc = 0.0;
            for (int a = 0; a < dk; ++a) acc += Sp[(size_t)a * dv + b] * kt[a];
            r[b] = acc;
            d[b] = bt * (vt[b] - r[b]);
        }
        /* o_t = S_t^T q_t */
        for (int a = 0; a < dk; ++a)
            for (int b = 0; b < dv; ++b) G[(size_t)a * dv + b] += qt[a] * dot[b];
        for (int a = 0; a < dk; ++a) {
            double acc = 0.0;
            for (int b = 0; b < dv; ++b) acc += S[(size_t)a * dv + b] * dot[b];
            dqt[a] = acc;
        }
        /* S_t = S' + k d^T */
        for (int b = 0; b < dv; ++b) {
            double acc = 0.0;
            for (int a = 0; a < dk; ++a) acc += G[(size_t)a * dv + b] * kt[a];
            dd[b] = acc;
        }
        for (int a = 0; a < dk; ++a) {
            double acc = 0.0;
            for (int b = 0; b < dv; ++b) acc += G[(size_t)a * dv + b] * d[b];
            dkt[a] = acc;
        }
        /* d = beta (v - r) */
        double dbt = 0.0;
        for (int b = 0; b < dv; ++b) {
            dbt += dd[b] * (vt[b] - r[b]);
            dvt[b] = bt * dd[b];
            dr[b] = -bt * dd[b];
        }
        job->dbeta[tok] = dbt;
        /* r = S'^T k: G' = G + k dr^T, dk += S' dr */
        for (int a = 0; a < dk; ++a) {
            double acc = 0.0;
            for (int b = 0; b < dv; ++b) {
                G[(size_t)a * dv + b] += kt[a] * dr[b];
                acc += Sp[(size_t)a * dv + b] * dr[b];
            }
            dkt[a] += acc;
        }
        /* S' = Diag(exp(la)) S_{t-1} */
        for (int a = 0; a < dk; ++a) {
            double acc = 0.0;
            for (int b = 0; b < dv; ++b) acc += Sp[(size_t)a * dv + b] * G[(size_t)a * dv + b];
            dlat[a] = acc;
            for (int b = 0; b < dv; ++b) G[(size_t)a * dv + b] *= alpha[a];
        }
    }
    if (job->d_init)
        memcpy(job->d_init + state_off, G, sizeof(double) * SZ);
    free(states); free(G); free(Sp); free(r); free(d); free(dd); free(dr); free(alpha);
    return 0;
}

static void *worker_bwd(void *arg)
{
    oracle_bwd_job *job = (oracle_bwd_job *)arg;
    const int total = job->n_seq * job->H;
    for (;;) {
        pthread_mutex_lock(&job->lock);
        const int idx = job->next++;
        pthread_mutex_unlock(&job->lock);
        if (idx >= total)
            break;
        if (run_chain_bwd(job, idx / job->H, idx % job->H) != 0) {
            pthread_mutex_lock(&job->lock);
            job->failed = 1;
            pthread_mutex_unlock(&job->lock);
        }
    }
    return NULL;
}

/*
 * oracle_kda_backward: gradients of a loss through oracle_kda_forward.
 *   inputs as oracle_kda_forward, plus
 *   d_o      : [T_total, H, dv]     dL/do
 *   d_final  : [n_seq, H, dk, dv] or NULL (zero)   dL/dS_final
 *   outputs dq, dk_out, dla : [T_total, H, dk]; dv_out : [T_total, H, dv];
 *   dbeta : [T_total, H]; d_init : [n_seq, H, dk, dv] or NULL.
 * Returns 0 on success, -1 on bad arguments, -2 on allocation failure.
 */
int oracle_kda_backward(const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *beta,
                        const double *init_state, const int64_t *cu_seqlens,
                        int n_seq, int H, int dk, int dv,
                        const double *d_o, const double *d_final,
                        double *dq, double *dk_out, double *dv_out, double *dla,
                        double *dbeta, double *d_init, int n_threads)
{
    if (!q || !k || !v || !log_alpha || !beta || !cu_seqlens || !d_o)
        return -1;
    if (!dq || !dk_out || !dv_out || !dla || !dbeta)
        return -1;
    if (n_seq < 0 || H <= 0 || dk <= 0 || dv <= 0 || cu_seqlens[0] != 0)
        return -1;
    for (int i = 0; i < n_seq; ++i)
        if (cu_seqlens[i + 1] < cu_seqlens[i])
            return -1;
    if (n_threads < 1)
        n_threads = 1;
    const int total = n_seq * H;
    if (n_threads > total)
        n_threads = total > 0 ? total : 1;
    oracle_bwd_job job;
    memset(&job, 0, sizeof(job));
    job.q = q; job.k = k; job.v = v; job.log_alpha = log_alpha; job.beta = beta;
    job.init_state = init_state; job.d_o = d_o; job.d_final = d_final;
    job.cu_seqlens = cu_seqlens; job.n_seq = n_seq; job.H = H; job.dk = dk; job.dv = dv;
    job.dq = dq; job.dk_out = dk_out; job.dv_out = dv_out; job.dla = dla;
    job.dbeta = dbeta; job.d_init = d_init;
    pthread_mutex_init(&job.lock, NULL);
    pthread_t *tids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!tids) {
        pthread_mutex_destroy(&job.lock);
        return -2;
    }
    int started = 0;
    for (int i = 1; i < n_threads; ++i) {
        if (pthread_create(&tids[i], NULL, worker_bwd, &job) != 0)
            break;
        ++started;
    }
    worker_bwd(&job);
    for (int i = 1; i <= started; ++i)
        pthread_join(tids[i], NULL);
    free(tids);
    pthread_mutex_destroy(&job.lock);
    return job.failed ? -2 : 0;
}
