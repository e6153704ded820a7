/*
 * kda_oracle.c -- plain fp64 CPU oracle for the KDA (Kimi Delta Attention)
 * token recurrence.  TEST INFRASTRUCTURE ONLY: tests, the smoke check and the
 * CPU-baseline leg of the benchmark call this file.  The product library never
 * links, loads or calls it, and it shares no code with the CUDA path.
 *
 * What it computes (one token step, for one sequence and one head).  The rule
 * is the "Stage 3: KDA's fused design" equation of "Hybrid Linear Attention
 * Architectures: Breaking Through the Long-Context Engineering Bottleneck in
 * LLMs", repeated as section 2.5 "KDA: Fine-Grained Gated DeltaNet (Final
 * Form)" of "Linear Attention KDA Gating in a 3:1 Hybrid Architecture":
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * with S a d_k x d_v matrix (rows indexed by key channel), alpha_t =
 * exp(log_alpha_t) a per-channel forget gate and beta_t a scalar write
 * strength.  The pages print the write term as "beta v k^T"; with S being
 * d_k x d_v and the erase matrix (I - beta k k^T) acting from the left it must
 * be k v^T (the same pages' section 3.1 gives U in R^{d_k x d_v}, and the
 * gated-recurrence listing of "Linear Attention + Sparse Attention", section
 * 2, writes the update as k (x) v with the read y_t = q_t . S_t).  Section 2.5
 * says the diagonal decay acts on the memory first and the key-direction
 * overwrite second, so the erase sees the decayed state; the output is read
 * after the write (section 3.2: token i sees tokens j <= i).  No scale is
 * applied to q: the pages never mention one.
 *
 * Written out step by step, the body of the loop below is
 *     S'  = Diag(alpha_t) S               (per-channel decay)
 *     r   = S'^T k_t                      (what the decayed memory returns for k_t)
 *     S   = S' + beta_t k_t (v_t - r)^T   (= (I - beta k k^T) S' + beta k v^T)
 *     o_t = S^T q_t
 * which is the plain expansion of the matrix form above; every product is a
 * plain loop in fp64 with no blocking or reordering.
 *
 * Layouts (row-major, all fp64):
 *   q, k, log_alpha  [B, T, H, d_k]     v, out  [B, T, H, d_v]     beta [B, T, H]
 *   state            [N, H, d_k, d_v]   (N = B, or num_seqs when cu_seqlens is given)
 * With cu_seqlens (int64 [num_seqs + 1], ascending, first entry 0) the batch
 * dimension must be 1 and sequence n covers tokens cu_seqlens[n] ..
 * cu_seqlens[n+1]-1 of the packed token axis; each sequence starts from its
 * own initial state and chunks never cross sequences.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *init_state;
    const int64_t *cu_seqlens;
    int64_t num_seqs, B, T, H, dk, dv;
    double *out, *final_state;
    int64_t next_task;           /* work counter over (sequence, head) pairs */
    pthread_mutex_t lock;
} oracle_job;

/* One recurrence step on one head's state S (d_k x d_v), in place.
 * Returns nothing; writes o (d_v) when o != NULL. */
static void kda_step(double *S, const double *q, const double *k, const double *v,
                     const double *log_alpha, double beta, int64_t dk, int64_t dv,
                     double *o, double *r /* scratch d_v */) {
    /* S' = Diag(alpha) S */
    for (int64_t i = 0; i < dk; ++i) {
        double a = exp(log_alpha[i]);
        for (int64_t j = 0; j < dv; ++j) S[i * dv + j] *= a;
    }
    /* r = S'^T k */
    for (int64_t j = 0; j < dv; ++j) r[j] = 0.0;
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * k[i];
    /* S = S' + beta k (v - r)^T */
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) S[i * dv + j] += beta * k[i] * (v[j] - r[j]);
    /* o = S^T q */
    if (o) {
        for (int64_t j = 0; j < dv; ++j) o[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) o[j] += S[i * dv + j] * q[i];
    }
}

static void run_task(oracle_job *jb, int64_t task, double *S, double *r) {
    const int64_t H = jb->H, dk = jb->dk, dv = jb->dv;
    const int64_t n = task / H, h = task % H;
    int64_t t0, t1, b;
    if (jb->cu_seqlens) {
        b = 0;
        t0 = jb->cu_seqlens[n];
        t1 = jb->cu_seqlens[n + 1];
    } else {
        b = n;
        t0 = 0;
        t1 = jb->T;
    }
    if (jb->init_state)
        memcpy(S, jb->init_state + (n * H + h) * dk * dv, sizeof(double) * dk * dv);
    else
        memset(S, 0, sizeof(double) * dk * dv);
    for (int64_t t = t0; t < t1; ++t) {
        const int64_t row = (b * jb->T + t) * H + h; /* token-head row index */
        kda_step(S, jb->q + row * dk, jb->k + row * dk, jb->v + row * dv,
                 jb->log_alpha + row * dk, jb->beta[row], dk, dv,
                 jb->out ? jb->out + row * dv : NULL, r);
    }
    if (jb->final_state)
        memcpy(jb->final_state + (n * H + h) * dk * dv, S, sizeof(double) * dk * dv);
}

static void *worker(void *arg) {
    oracle_job *jb = (oracle_job *)arg;
    const int64_t ntask = jb->num_seqs * jb->H;
    double *S = (double *)malloc(sizeof(double) * (size_t)(jb->dk * jb->dv));
    double *r = (double *)malloc(sizeof(double) * (size_t)jb->dv);
    for (;;) {
        pthread_mutex_lock(&jb->lock);
        int64_t task = jb->next_task++;
        pthread_mutex_unlock(&jb->lock);
        if (task >= ntask) break;
        run_task(jb, task, S, r);
    }
    free(S);
    free(r);
    return NULL;
}

/* Full token recurrence over every (sequence, head) pair, fanned out over
 * `nthreads` host threads (each pair is independent).  Returns 0 on success,
 * -1 on bad arguments.  out / final_state may be NULL to skip them. */
int kda_oracle_recurrent(const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta,
                         const double *init_state, const int64_t *cu_seqlens,
                         int64_t num_seqs, int64_t B, int64_t T, int64_t H,
                         int64_t dk, int64_t dv, double *out, double *final_state,
                         int nthreads) {
    if (!q || !k || !v || !log_alpha || !beta) return -1;
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return -1;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 1) return -1;
        if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T) return -1;
        for (int64_t n = 0; n < num_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    } else {
        num_seqs = B;
    }
    oracle_job jb;
    jb.q = q; jb.k = k; jb.v = v; jb.log_alpha = log_alpha; jb.beta = beta;
    jb.init_state = init_state; jb.cu_seqlens = cu_seqlens; jb.num_seqs = num_seqs;
    jb.B = B; jb.T = T; jb.H = H; jb.dk = dk; jb.dv = dv;
    jb.out = out; jb.final_state = final_state; jb.next_task = 0;
    pthread_mutex_init(&jb.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > num_seqs * H) nthreads = (int)(num_seqs * H);
    pthread_t th[256];
    int started = 0;
    for (int i = 1; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, worker, &jb) == 0) ++started; else break;
    worker(&jb); /* the calling thread works too */
    for (int i = 1; i <= started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&jb.lock);
    return 0;
}

/* One decode step: one iteration of the recurrence body for every (b, h),
 * updating state [B, H, d_k, d_v] in place and writing out [B, H, d_v].
 * Inputs are laid out [B, H, d] (one token per sequence). */
int kda_oracle_decode_step(const double *q, const double *k, const double *v,
                           const double *log_alpha, const double *beta,
                           double *state, double *out, int64_t B, int64_t H,
                           int64_t dk, int64_t dv) {
    if (!q || !k || !v || !log_alpha || !beta || !state) return -1;
    if (B < 1 || H < 1 || dk < 1 || dv < 1) return -1;
    double *r = (double *)malloc(sizeof(double) * (size_t)dv);
    for (int64_t bh = 0; bh < B * H; ++bh)
        kda_step(state + bh * dk * dv, q + bh * dk, k + bh * dk, v + bh * dv,
                 log_alpha + bh * dk, beta[bh], dk, dv, out ? out + bh * dv : NULL, r);
    free(r);
    return 0;
}

/*
 * Gradient of the same recurrence (reverse mode).  The pages describe
 * training with the chunked form (the "Implementation checklist" of "Hybrid
 * Linear Attention Architectures: Breaking Through the Long-Context
 * Engineering Bottleneck in LLMs" asks for FP32 intermediates and gradient
 * clipping; "Linear Attention KDA Gating in a 3:1 Hybrid Architecture",
 * section 3, asks for gradient checks when choosing the chunk size) but print
 * no backward pass, so this is the plain adjoint of the forward step above.
 * With the step written as
 *     S'  = Diag(a) S_prev,  a = exp(g)
 *     w   = S'^T k
 *     u   = beta (v - w)
 *     S   = S' + k u^T
 *     o   = S^T q
 * and dX denoting dLoss/dX, one reverse step (given dS, the gradient with
 * respect to the state after the token, and do) is
 *     dS   += q do^T                 dq = S do
 *     du    = dS^T k                 dk = dS u
 *     dbeta = du . (v - w)           dv = beta du
 *     dS'   = dS - beta k du^T       dk -= beta S' du
 *     dg    = rowsum(dS' * S')       (d a * a)
 *     dS_prev = Diag(a) dS'
 * The forward states are kept for the whole sequence (plain and slow: memory
 * grows with T), then the tokens are visited in reverse.  dfinal (the
 * gradient with respect to the final state) seeds dS, and the last dS_prev is
 * the gradient with respect to the initial state.
 *
 * Layouts as for kda_oracle_recurrent; dout [B, T, H, d_v]; dq, dk, dlog_alpha
 * [B, T, H, d_k]; dv [B, T, H, d_v]; dbeta [B, T, H]; dfinal, dinit
 * [N, H, d_k, d_v] (dfinal may be NULL: zero; dinit may be NULL: skipped).
 */
typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *init_state, *dout, *dfinal;
    const int64_t *cu_seqlens;
    int64_t num_seqs, B, T, H, dk, dv;
    double *dq, *dkk, *dvv, *dla, *dbeta, *dinit;
    int64_t next_task;
    int failed;
    pthread_mutex_t lock;
} oracle_bwd_job;

static int run_bwd_task(oracle_bwd_job *jb, int64_t task) {
    const int64_t H = jb->H, dk = jb->dk, dv = jb->dv, kv = dk * dv;
    const int64_t n = task / H, h = task % H;
    int64_t t0, t1, b;
    if (jb->cu_seqlens) {
        b = 0;
        t0 = jb->cu_seqlens[n];
        t1 = jb->cu_seqlens[n + 1];
    } else {
        b = n;
        t0 = 0;
        t1 = jb->T;
    }
    const int64_t L = t1 - t0;
    double *Ss = (double *)malloc(sizeof(double) * (size_t)((L + 1) * kv));
    double *dS = (double *)malloc(sizeof(double) * (size_t)kv);
    double *Sp = (double *)malloc(sizeof(double) * (size_t)kv);
    double *w = (double *)malloc(sizeof(double) * (size_t)dv);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    double *du = (double *)malloc(sizeof(double) * (size_t)dv);
    double *a = (double *)malloc(sizeof(double) * (size_t)dk);
    if (!Ss || !dS || !Sp || !w || !u || !du || !a) {
        free(Ss); free(dS); free(Sp); free(w); free(u); free(du); free(a);
        return -1;
    }
    /* forward, keeping the state after every token: Ss[t] = state after t tokens */
    if (jb->init_state)
        memcpy(Ss, jb->init_state + (n * H + h) * kv, sizeof(double) * kv);
    else
        memset(Ss, 0, sizeof(double) * kv);
    for (int64_t t = 0; t < L; ++t) {
        const int64_t row = (b * jb->T + t0 + t) * H + h;
        memcpy(Ss + (t + 1) * kv, Ss + t * kv, sizeof(double) * kv);
        kda_step(Ss + (t + 1) * kv, jb->q + row * dk, jb->k + row * dk, jb->v + row * dv,
                 jb->log_alpha + row * dk, jb->beta[row], dk, dv, NULL, w);
    }
    /* reverse */
    if (jb->dfinal)
        memcpy(dS, jb->dfinal + (n * H + h) * kv, sizeof(double) * kv);
    else
        memset(dS, 0, sizeof(double) * kv);
    for (int64_t t = L - 1; t >= 0; --t) {
        const int64_t row = (b * jb->T + t0 + t) * H + h;
        const double *q = jb->q + row * dk, *k = jb->k + row * dk, *v = jb->v + row * dv;
        const double *g = jb->log_alpha + row * dk, *dout = jb->dout + row * dv;
        const double beta = jb->beta[row];
        const double *Sprev = Ss + t * kv, *Snew = Ss + (t + 1) * kv;
        double *dq = jb->dq + row * dk, *dkr = jb->dkk + row * dk, *dvr = jb->dvv + row * dv;
        double *dg = jb->dla + row * dk;
        /* recompute the step's intermediates: S' and w = S'^T k, u = beta (v - w) */
        for (int64_t i = 0; i < dk; ++i) {
            a[i] = exp(g[i]);
            for (int64_t j = 0; j < dv; ++j) Sp[i * dv + j] = a[i] * Sprev[i * dv + j];
        }
        for (int64_t j = 0; j < dv; ++j) {
            w[j] = 0.0;
            for (int64_t i = 0; i < dk; ++i) w[j] += Sp[i * dv + j] * k[i];
            u[j] = beta * (v[j] - w[j]);
        }
        /* o = S^T q */
        for (int64_t i = 0; i < dk; ++i) {
            dq[i] = 0.0;
            for (int64_t j = 0; j < dv; ++j) {
                dS[i * dv + j] += q[i] * dout[j];
                dq[i] += Snew[i * dv + j] * dout[j];
            }
        }
        /* S = S' + k u^T */
        for (int64_t j = 0; j < dv; ++j) {
            du[j] = 0.0;
            for (int64_t i = 0; i < dk; ++i) du[j] += dS[i * dv + j] * k[i];
        }
        for (int64_t i = 0; i < dk; ++i) {
            dkr[i] = 0.0;
            for (int64_t j = 0; j < dv; ++j) dkr[i] += dS[i * dv + j] * u[j];
        }
        /* u = beta (v - w) */
        double db = 0.0;
        for (int64_t j = 0; j < dv; ++j) {
            db += du[j] * (v[j] - w[j]);
            dvr[j] = beta * du[j];
        }
        jb->dbeta[row] = db;
        /* w = S'^T k: dw = -beta du */
        for (int64_t i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int64_t j = 0; j < dv; ++j) {
                dS[i * dv + j] -= beta * k[i] * du[j]; /* now dS' */
                acc += Sp[i * dv + j] * du[j];
            }
            dkr[i] -= beta * acc;
        }
        /* S' = Diag(a) S_prev */
        for (int64_t i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int64_t j = 0; j < dv; ++j) {
                acc += dS[i * dv + j] * Sp[i * dv + j];
                dS[i * dv + j] *= a[i]; /* now dS_prev */
            }
            dg[i] = acc;
        }
    }
    if (jb->dinit) memcpy(jb->dinit + (n * H + h) * kv, dS, sizeof(double) * kv);
    free(Ss); free(dS); free(Sp); free(w); free(u); free(du); free(a);
    return 0;
}

static void *bwd_worker(void *arg) {
    oracle_bwd_job *jb = (oracle_bwd_job *)arg;
    const int64_t ntask = jb->num_seqs * jb->H;
    for (;;) {
        pthread_mutex_lock(&jb->lock);
        int64_t task = jb->next_task++;
        pthread_mutex_unlock(&jb->lock);
        if (task >= ntask) break;
        if (run_bwd_task(jb, task) != 0) {
            pthread_mutex_lock(&jb->lock);
            jb->failed = 1;
            pthread_mutex_unlock(&jb->lock);
        }
    }
    return NULL;
}

/* Gradients of every input of kda_oracle_recurrent given dout (and dfinal).
 * Returns 0 on success, -1 on bad arguments, -2 if memory ran out. */
int kda_oracle_backward(const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *beta,
                        const double *init_state, const int64_t *cu_seqlens,
                        int64_t num_seqs, int64_t B, int64_t T, int64_t H,
                        int64_t dk, int64_t dv, const double *dout, const double *dfinal,
                        double *dq, double *dkk, double *dvv, double *dlog_alpha,
                        double *dbeta, double *dinit, int nthreads) {
    if (!q || !k || !v || !log_alpha || !beta || !dout) return -1;
    if (!dq || !dkk || !dvv || !dlog_alpha || !dbeta) return -1;
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return -1;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 1) return -1;
        if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T) return -1;
        for (int64_t n = 0; n < num_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    } else {
        num_seqs = B;
    }
    oracle_bwd_job jb;
    jb.q = q; jb.k = k; jb.v = v; jb.log_alpha = log_alpha; jb.beta = beta;
    jb.init_state = init_state; jb.dout = dout; jb.dfinal = dfinal; jb.cu_seqlens = cu_seqlens;
    jb.num_seqs = num_seqs; jb.B = B; jb.T = T; jb.H = H; jb.dk = dk; jb.dv = dv;
    jb.dq = dq; jb.dkk = dkk; jb.dvv = dvv; jb.dla = dlog_alpha; jb.dbeta = dbeta; jb.dinit = dinit;
    jb.next_task = 0; jb.failed = 0;
    pthread_mutex_init(&jb.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > num_seqs * H) nthreads = (int)(num_seqs * H);
    pthread_t th[256];
    int started = 0;
    for (int i = 1; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, bwd_worker, &jb) == 0) ++started; else break;
    bwd_worker(&jb);
    for (int i = 1; i <= started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&jb.lock);
    return jb.failed ? -2 : 0;
}
