/*
 * CKDA fp64 CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * This file is the slow, obviously correct reference for the Complex Kimi
 * Delta Attention (CKDA) recurrence.  Only the test suite, the package's
 * smoke check and the CPU-baseline leg of the benchmark may load it.  It
 * shares no code with the CUDA path and includes no CUDA header.
 *
 * What it computes (per sequence n and head h, all arithmetic in fp64):
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = S_t^T q_t                         (read-out after the update)
 *
 * Sources:
 *  - "Complex KDA: Kimi Delta Attention Mimarisinin Ifade Gucunu Anlamak ve
 *    Gelistirmek", section "Complex KDA (CKDA) Mimarisi ve Parametre
 *    Genislemesi": per-channel gate alpha in [-1, 1], delta coefficient
 *    beta in [0, 2], diagonal-plus-rank-one transition.
 *  - "Gated DeltaNet-2" technical summary, Methodology section 1, the state
 *    equation S_t = (I - k_t (b_t . k_t)^T) D_t S_{t-1} + k_t (w_t . v_t)^T
 *    with D_t = Diag(alpha_t); tying b_t = w_t = beta_t gives the form above.
 *  - "Semidirect Fourier Delta Attention (SFDA)" technical summary,
 *    "Arquitectura Central" equation with zero phase (Lambda_t = diag(alpha_t)).
 *  The read-out o_t = S_t^T q_t is not printed on those pages; the plainest
 *  reading (post-update state, no query scale) is used.
 *
 * The per-token body is written exactly in the order of the equation:
 *   1. S <- Diag(alpha) S            (scale row i by alpha_i)
 *   2. r <- S^T k                    (read the current association of k)
 *   3. S <- S + beta k (v - r)^T     ((I - beta k k^T) S' + beta k v^T)
 *   4. o <- S^T q
 *
 * Layouts (row-major, contiguous):
 *   q, k, alpha : [T_total, H, dk]     v, out : [T_total, H, dv]
 *   beta        : [T_total, H]
 *   S0, S_final : [N, H, dk, dv]       (S0 may be NULL: zero initial state)
 *   cu_seqlens  : int64 [N + 1], sequence n spans tokens [cu[n], cu[n+1])
 *
 * The Gated DeltaNet-2 form (ckda_oracle_gdn2_forward) replaces the scalar
 * beta_t by an erase gate b_t in [0, 1]^dk on the key side and a write gate
 * w_t in [0, 1]^dv on the value side ("Gated DeltaNet-2" technical summary,
 * Methodology section 1):
 *
 *   S_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T
 *
 * with the same read-out; its body, in the order of that equation:
 *   1. S <- Diag(alpha) S
 *   2. r <- S^T e,  e = b . k         (the erased read)
 *   3. S <- S + k (z - r)^T,  z = w . v
 *   4. o <- S^T q
 *   b : [T_total, H, dk]   w : [T_total, H, dv]
 *
 * The SFDA form (ckda_oracle_sfda_forward) replaces the real diagonal gate by
 * a phase-decay gate ("Semidirect Fourier Delta Attention (SFDA)" technical
 * summary, "Arquitectura Central"): in complex coordinates
 * Lambda_t = diag(alpha_t . e^{i theta_t}); in real coordinates, the form
 * used here, Lambda_t is the direct sum of 2x2 rotation-decay blocks, block
 * p acting on the state rows (2p, 2p+1) as
 *
 *   alpha_p * [[cos theta_p, -sin theta_p], [sin theta_p, cos theta_p]]
 *
 * (row 2p is the real part, row 2p+1 the imaginary part of channel p), and
 *
 *   S_t = (I - beta_t k_t k_t^T) Lambda_t S_{t-1} + beta_t k_t v_t^T,
 *
 * i.e. the transition Lambda_t - u_t r_t^T with u_t = beta_t k_t and
 * r_t = Lambda_t^T k_t ("El Teorema de Chunk-WY Constructivo").  Keys,
 * queries, values and the state are real.  Its body:
 *   1. S <- Lambda S                  (rotate and scale each row pair)
 *   2. r <- S^T k
 *   3. S <- S + beta k (v - r)^T
 *   4. o <- S^T q
 *   alpha, theta : [T_total, H, dk / 2]   (dk even)
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t n_seqs, H, dk, dv;
    const int64_t *cu;
    const double *q, *k, *v, *alpha, *beta, *S0;
    const double *eg, *wg; /* Gated DeltaNet-2 gates (NULL for the beta form) */
    const double *theta;   /* SFDA phases (NULL unless the SFDA form) */
    double *out, *S_final;
    int64_t next_unit; /* shared work counter (guarded by lock) */
    pthread_mutex_t lock;
} oracle_job;

/* One (sequence, head) unit: the sequential recurrence, token by token. */
static void run_unit(const oracle_job *J, int64_t n, int64_t h, double *S,
                     double *r) {
    const int64_t H = J->H, dk = J->dk, dv = J->dv;
    if (J->S0) {
        memcpy(S, J->S0 + ((n * H + h) * dk) * dv, sizeof(double) * dk * dv);
    } else {
        memset(S, 0, sizeof(double) * dk * dv);
    }
    for (int64_t t = J->cu[n]; t < J->cu[n + 1]; ++t) {
        const double *q = J->q + (t * H + h) * dk;
        const double *k = J->k + (t * H + h) * dk;
        const double *a = J->alpha + (t * H + h) * dk;
        const double *v = J->v + (t * H + h) * dv;
        const double b = J->beta[t * H + h];
        double *o = J->out + (t * H + h) * dv;

        /* 1. S <- Diag(alpha) S */
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) S[i * dv + j] *= a[i];
        /* 2. r <- S^T k */
        for (int64_t j = 0; j < dv; ++j) r[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * k[i];
        /* 3. S <- S + beta k (v - r)^T */
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j)
                S[i * dv + j] += b * k[i] * (v[j] - r[j]);
        /* 4. o <- S^T q */
        for (int64_t j = 0; j < dv; ++j) o[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) o[j] += S[i * dv + j] * q[i];
    }
    if (J->S_final)
        memcpy(J->S_final + ((n * H + h) * dk) * dv, S,
               sizeof(double) * dk * dv);
}

/* One (sequence, head) unit of the Gated DeltaNet-2 recurrence. */
static void run_unit_gdn2(const oracle_job *J, int64_t n, int64_t h, double *S,
                          double *r) {
    const int64_t H = J->H, dk = J->dk, dv = J->dv;
    if (J->S0) {
        memcpy(S, J->S0 + ((n * H + h) * dk) * dv, sizeof(double) * dk * dv);
    } else {
        memset(S, 0, sizeof(double) * dk * dv);
    }
    for (int64_t t = J->cu[n]; t < J->cu[n + 1]; ++t) {
        const double *q = J->q + (t * H + h) * dk;
        const double *k = J->k + (t * H + h) * dk;
        const double *a = J->alpha + (t * H + h) * dk;
        const double *b = J->eg + (t * H + h) * dk;
        const double *v = J->v + (t * H + h) * dv;
        const double *w = J->wg + (t * H + h) * dv;
        double *o = J->out + (t * H + h) * dv;

        /* 1. S <- Diag(alpha) S */
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) S[i * dv + j] *= a[i];
        /* 2. r <- S^T (b . k) */
        for (int64_t j = 0; j < dv; ++j) r[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * (b[i] * k[i]);
        /* 3. S <- S + k (w . v - r)^T */
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j)
                S[i * dv + j] += k[i] * (w[j] * v[j] - r[j]);
        /* 4. o <- S^T q */
        for (int64_t j = 0; j < dv; ++j) o[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) o[j] += S[i * dv + j] * q[i];
    }
    if (J->S_final)
        memcpy(J->S_final + ((n * H + h) * dk) * dv, S,
               sizeof(double) * dk * dv);
}

/* One (sequence, head) unit of the SFDA recurrence (phase-decay blocks). */
static void run_unit_sfda(const oracle_job *J, int64_t n, int64_t h, double *S,
                          double *r) {
    const int64_t H = J->H, dk = J->dk, dv = J->dv, np = dk / 2;
    if (J->S0) {
        memcpy(S, J->S0 + ((n * H + h) * dk) * dv, sizeof(double) * dk * dv);
    } else {
        memset(S, 0, sizeof(double) * dk * dv);
    }
    for (int64_t t = J->cu[n]; t < J->cu[n + 1]; ++t) {
        const double *q = J->q + (t * H + h) * dk;
        const double *k = J->k + (t * H + h) * dk;
        const double *a = J->alpha + (t * H + h) * np;
        const double *th = J->theta + (t * H + h) * np;
        const double *v = J->v + (t * H + h) * dv;
        const double b = J->beta[t * H + h];
        double *o = J->out + (t * H + h) * dv;

        /* 1. S <- Lambda S: rows (2p, 2p+1) times alpha_p R(theta_p) */
        for (int64_t p = 0; p < np; ++p) {
            const double c = a[p] * cos(th[p]), sn = a[p] * sin(th[p]);
            double *x = S + (2 * p) * dv, *y = S + (2 * p + 1) * dv;
            for (int64_t j = 0; j < dv; ++j) {
                const double xr = x[j], yr = y[j];
                x[j] = c * xr - sn * yr;
                y[j] = sn * xr + c * yr;
            }
        }
        /* 2. r <- S^T k */
        for (int64_t j = 0; j < dv; ++j) r[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * k[i];
        /* 3. S <- S + beta k (v - r)^T */
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j)
                S[i * dv + j] += b * k[i] * (v[j] - r[j]);
        /* 4. o <- S^T q */
        for (int64_t j = 0; j < dv; ++j) o[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) o[j] += S[i * dv + j] * q[i];
    }
    if (J->S_final)
        memcpy(J->S_final + ((n * H + h) * dk) * dv, S,
               sizeof(double) * dk * dv);
}

static void *worker(void *arg) {
    oracle_job *J = (oracle_job *)arg;
    double *S = (double *)malloc(sizeof(double) * J->dk * J->dv);
    double *r = (double *)malloc(sizeof(double) * J->dv);
    const int64_t n_units = J->n_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= n_units) break;
        if (J->theta)
            run_unit_sfda(J, u / J->H, u % J->H, S, r);
        else if (J->eg)
            run_unit_gdn2(J, u / J->H, u % J->H, S, r);
        else
            run_unit(J, u / J->H, u % J->H, S, r);
    }
    free(S);
    free(r);
    return NULL;
}

/* Share the (sequence, head) units of a job out to n_threads host threads. */
static void run_job(oracle_job *J, int n_threads) {
    J->next_unit = 0;
    pthread_mutex_init(&J->lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    pthread_t tid[256];
    int started = 0;
    for (int i = 1; i < n_threads; ++i)
        if (pthread_create(&tid[started], NULL, worker, J) == 0) ++started;
    worker(J);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    pthread_mutex_destroy(&J->lock);
}

/*
 * Sequential CKDA forward over a packed batch.  Returns 0 on success, -1 on
 * an argument error (bad sizes or offsets).  Units of (sequence, head) are
 * independent and are shared out to `n_threads` host threads; the result
 * does not depend on the thread count.
 */
int ckda_oracle_forward(int64_t n_seqs, int64_t H, int64_t dk, int64_t dv,
                        const int64_t *cu_seqlens, const double *q,
                        const double *k, const double *v, const double *alpha,
                        const double *beta, const double *S0, double *out,
                        double *S_final, int n_threads) {
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens)
        return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int64_t n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    oracle_job J;
    J.n_seqs = n_seqs;
    J.H = H;
    J.dk = dk;
    J.dv = dv;
    J.cu = cu_seqlens;
    J.q = q;
    J.k = k;
    J.v = v;
    J.alpha = alpha;
    J.beta = beta;
    J.eg = NULL;
    J.wg = NULL;
    J.theta = NULL;
    J.S0 = S0;
    J.out = out;
    J.S_final = S_final;
    run_job(&J, n_threads);
    return 0;
}

/*
 * Sequential Gated DeltaNet-2 forward over a packed batch (layouts as
 * above, with the gates b [T_total, H, dk] and w [T_total, H, dv] in place
 * of beta).  Returns 0 on success, -1 on an argument error.
 */
int ckda_oracle_gdn2_forward(int64_t n_seqs, int64_t H, int64_t dk, int64_t dv,
                             const int64_t *cu_seqlens, const double *q,
                             const double *k, const double *v,
                             const double *alpha, const double *b,
                             const double *w, const double *S0, double *out,
                             double *S_final, int n_threads) {
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens || !b || !w)
        return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int64_t n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    oracle_job J;
    J.n_seqs = n_seqs;
    J.H = H;
    J.dk = dk;
    J.dv = dv;
    J.cu = cu_seqlens;
    J.q = q;
    J.k = k;
    J.v = v;
    J.alpha = alpha;
    J.beta = NULL;
    J.eg = b;
    J.wg = w;
    J.theta = NULL;
    J.S0 = S0;
    J.out = out;
    J.S_final = S_final;
    run_job(&J, n_threads);
    return 0;
}

/*
 * Sequential SFDA forward over a packed batch (layouts as above, with the
 * decays alpha and phases theta both [T_total, H, dk / 2] and dk even).
 * Returns 0 on success, -1 on an argument error.
 */
int ckda_oracle_sfda_forward(int64_t n_seqs, int64_t H, int64_t dk, int64_t dv,
                             const int64_t *cu_seqlens, const double *q,
                             const double *k, const double *v,
                             const double *alpha, const double *theta,
                             const double *beta, const double *S0, double *out,
                             double *S_final, int n_threads) {
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || (dk & 1) || !cu_seqlens ||
        !theta)
        return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int64_t n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    oracle_job J;
    J.n_seqs = n_seqs;
    J.H = H;
    J.dk = dk;
    J.dv = dv;
    J.cu = cu_seqlens;
    J.q = q;
    J.k = k;
    J.v = v;
    J.alpha = alpha;
    J.beta = beta;
    J.eg = NULL;
    J.wg = NULL;
    J.theta = theta;
    J.S0 = S0;
    J.out = out;
    J.S_final = S_final;
    run_job(&J, n_threads);
    return 0;
}

/*
 * Backward of the CKDA forward (the gradient of a scalar loss through the
 * recurrence), for one (sequence, head) unit, in fp64.  Given the upstream
 * gradients dO = dL/do_t and dS_T = dL/dS_final it returns dL/dq, dL/dk,
 * dL/dv, dL/dalpha, dL/dbeta and dL/dS0.  It is the adjoint of the per-token
 * body above, taken step by step in reverse order:
 *
 *   forward:  S' = Diag(a) S_prev;  r = S'^T k;  u = b (v - r);
 *             S = S' + k u^T;  o = S^T q
 *   reverse (dS = dL/dS after token t, accumulated from later tokens):
 *     dq = S do;            dS += q do^T          (o = S^T q)
 *     du = dS^T k;          dk = dS u             (S = S' + k u^T)
 *     dbeta = du . (v - r); dv = b du;  dr = -b du  (u = b (v - r))
 *     dS' = dS + k dr^T;    dk += S' dr           (r = S'^T k, S' direct)
 *     dalpha = rowsum(dS' . S_prev);  dS = Diag(a) dS'  (S' = Diag(a) S_prev)
 *   and finally dS0 = dS.
 *
 * The states S_prev of every token are recomputed: the forward pass keeps
 * the state at every kSeg-th token, and the reverse pass re-runs each
 * segment from its checkpoint before walking it backwards.
 */
enum { kSeg = 64 };

typedef struct {
    int64_t n_seqs, H, dk, dv;
    const int64_t *cu;
    const double *q, *k, *v, *alpha, *beta, *S0, *dO, *dSf;
    double *dq, *dk_out, *dv_out, *dalpha, *dbeta, *dS0;
    int64_t next_unit;
    pthread_mutex_t lock;
} oracle_bwd_job;

/* One forward token step on S (in place); keeps r and u when asked. */
static void fwd_token(int64_t dk, int64_t dv, const double *k, const double *a,
                      const double *v, double b, double *S, double *r,
                      double *u) {
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) S[i * dv + j] *= a[i];
    for (int64_t j = 0; j < dv; ++j) r[j] = 0.0;
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * k[i];
    for (int64_t j = 0; j < dv; ++j) u[j] = b * (v[j] - r[j]);
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) S[i * dv + j] += k[i] * u[j];
}

static void run_unit_bwd(const oracle_bwd_job *J, int64_t n, int64_t h) {
    const int64_t H = J->H, dk = J->dk, dv = J->dv, sz = dk * dv;
    const int64_t t0 = J->cu[n], t1 = J->cu[n + 1], L = t1 - t0;
    const int64_t nseg = (L + kSeg - 1) / kSeg;
    double *ck = (double *)malloc(sizeof(double) * sz * (nseg > 0 ? nseg : 1));
    double *St = (double *)malloc(sizeof(double) * sz * (kSeg + 1));
    double *rr = (double *)malloc(sizeof(double) * dv * kSeg);
    double *uu = (double *)malloc(sizeof(double) * dv * kSeg);
    double *dS = (double *)malloc(sizeof(double) * sz);
    double *du = (double *)malloc(sizeof(double) * dv);
    double *tmp = (double *)malloc(sizeof(double) * dv);
    double *S = St; /* scratch for the checkpoint pass */

    /* forward pass: the state at the start of every segment */
    if (J->S0)
        memcpy(S, J->S0 + (n * H + h) * sz, sizeof(double) * sz);
    else
        memset(S, 0, sizeof(double) * sz);
    for (int64_t g = 0; g < nseg; ++g) {
        memcpy(ck + g * sz, S, sizeof(double) * sz);
        const int64_t e = (g + 1) * kSeg < L ? (g + 1) * kSeg : L;
        for (int64_t t = t0 + g * kSeg; t < t0 + e; ++t)
            fwd_token(dk, dv, J->k + (t * H + h) * dk, J->alpha + (t * H + h) * dk,
                      J->v + (t * H + h) * dv, J->beta[t * H + h], S, tmp, du);
    }

    /* reverse pass */
    if (J->dSf)
        memcpy(dS, J->dSf + (n * H + h) * sz, sizeof(double) * sz);
    else
        memset(dS, 0, sizeof(double) * sz);
    for (int64_t g = nseg - 1; g >= 0; --g) {
        const int64_t ts = t0 + g * kSeg;
        const int64_t te = (g + 1) * kSeg < L ? t0 + (g + 1) * kSeg : t1;
        /* St[m] = state after token ts + m - 1 (St[0] = segment start) */
        memcpy(St, ck + g * sz, sizeof(double) * sz);
        for (int64_t t = ts; t < te; ++t) {
            const int64_t m = t - ts;
            memcpy(St + (m + 1) * sz, St + m * sz, sizeof(double) * sz);
            fwd_token(dk, dv, J->k + (t * H + h) * dk, J->alpha + (t * H + h) * dk,
                      J->v + (t * H + h) * dv, J->beta[t * H + h], St + (m + 1) * sz,
                      rr + m * dv, uu + m * dv);
        }
        for (int64_t t = te - 1; t >= ts; --t) {
            const int64_t m = t - ts;
            const double *q = J->q + (t * H + h) * dk;
            const double *k = J->k + (t * H + h) * dk;
            const double *a = J->alpha + (t * H + h) * dk;
            const double *v = J->v + (t * H + h) * dv;
            const double b = J->beta[t * H + h];
            const double *dO = J->dO + (t * H + h) * dv;
            const double *Sp = St + m * sz;       /* S_prev */
            const double *Sc = St + (m + 1) * sz; /* S after the token */
            const double *r = rr + m * dv, *u = uu + m * dv;
            double *dq = J->dq + (t * H + h) * dk;
            double *dkk = J->dk_out + (t * H + h) * dk;
            double *dvv = J->dv_out + (t * H + h) * dv;
            double *da = J->dalpha + (t * H + h) * dk;

            /* o = S^T q */
            for (int64_t i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < dv; ++j) acc += Sc[i * dv + j] * dO[j];
                dq[i] = acc;
            }
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) dS[i * dv + j] += q[i] * dO[j];
            /* S = S' + k u^T */
            for (int64_t j = 0; j < dv; ++j) du[j] = 0.0;
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) du[j] += dS[i * dv + j] * k[i];
            for (int64_t i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < dv; ++j) acc += dS[i * dv + j] * u[j];
                dkk[i] = acc;
            }
            /* u = b (v - r) */
            double db = 0.0;
            for (int64_t j = 0; j < dv; ++j) db += du[j] * (v[j] - r[j]);
            J->dbeta[t * H + h] = db;
            for (int64_t j = 0; j < dv; ++j) dvv[j] = b * du[j];
            for (int64_t j = 0; j < dv; ++j) tmp[j] = -b * du[j]; /* dr */
            /* r = S'^T k, with S' = Diag(a) S_prev */
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) dS[i * dv + j] += k[i] * tmp[j];
            for (int64_t i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < dv; ++j) acc += a[i] * Sp[i * dv + j] * tmp[j];
                dkk[i] += acc;
            }
            /* S' = Diag(a) S_prev */
            for (int64_t i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < dv; ++j) acc += dS[i * dv + j] * Sp[i * dv + j];
                da[i] = acc;
                for (int64_t j = 0; j < dv; ++j) dS[i * dv + j] *= a[i];
            }
        }
    }
    if (J->dS0) memcpy(J->dS0 + (n * H + h) * sz, dS, sizeof(double) * sz);
    free(ck);
    free(St);
    free(rr);
    free(uu);
    free(dS);
    free(du);
    free(tmp);
}

static void *worker_bwd(void *arg) {
    oracle_bwd_job *J = (oracle_bwd_job *)arg;
    const int64_t n_units = J->n_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= n_units) break;
        run_unit_bwd(J, u / J->H, u % J->H);
    }
    return NULL;
}

/*
 * Backward of the sequential CKDA forward over a packed batch (layouts as
 * for ckda_oracle_forward; dO like out, dS_final like S_final, either may be
 * NULL = zero; gradients dq, dk, dalpha [T_total, H, dk], dv [T_total, H, dv],
 * dbeta [T_total, H], dS0 [N, H, dk, dv] (may be NULL)).  Returns 0 on
 * success, -1 on an argument error.
 */
int ckda_oracle_backward(int64_t n_seqs, int64_t H, int64_t dk, int64_t dv,
                         const int64_t *cu_seqlens, const double *q,
                         const double *k, const double *v, const double *alpha,
                         const double *beta, const double *S0, const double *dO,
                         const double *dS_final, double *dq, double *dk_out,
                         double *dv_out, double *dalpha, double *dbeta,
                         double *dS0, int n_threads) {
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens || !dO)
        return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int64_t n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    oracle_bwd_job J;
    J.n_seqs = n_seqs;
    J.H = H;
    J.dk = dk;
    J.dv = dv;
    J.cu = cu_seqlens;
    J.q = q;
    J.k = k;
    J.v = v;
    J.alpha = alpha;
    J.beta = beta;
    J.S0 = S0;
    J.dO = dO;
    J.dSf = dS_final;
    J.dq = dq;
    J.dk_out = dk_out;
    J.dv_out = dv_out;
    J.dalpha = dalpha;
    J.dbeta = dbeta;
    J.dS0 = dS0;
    J.next_unit = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    pthread_t tid[256];
    int started = 0;
    for (int i = 1; i < n_threads; ++i)
        if (pthread_create(&tid[started], NULL, worker_bwd, &J) == 0) ++started;
    worker_bwd(&J);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/*
 * One recurrent decode step for B independent sequences: the same body as
 * above applied to a single token, with the state updated in place.
 * ("Complex KDA ...", section "Yazilim Gelistirme Acisindan Pratik
 * Cikarimlar": constant-size state at inference.)
 *   q, k, alpha : [B, H, dk]   v, out : [B, H, dv]   beta : [B, H]
 *   S_inout     : [B, H, dk, dv]
 */
int ckda_oracle_decode_step(int64_t B, int64_t H, int64_t dk, int64_t dv,
                            const double *q, const double *k, const double *v,
                            const double *alpha, const double *beta,
                            double *S_inout, double *out, int n_threads) {
    if (B < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    int64_t *cu = (int64_t *)malloc(sizeof(int64_t) * (B + 1));
    for (int64_t b = 0; b <= B; ++b) cu[b] = b;
    int rc = ckda_oracle_forward(B, H, dk, dv, cu, q, k, v, alpha, beta,
                                 S_inout, out, S_inout, n_threads);
    free(cu);
    return rc;
}
