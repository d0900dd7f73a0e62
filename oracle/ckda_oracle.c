/*
 * ckda_oracle.c -- fp64 CPU oracle for the gated delta-rule recurrence
 * (KDA and Complex-KDA forms).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, sequential
 * statement of what the CUDA path computes.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header, table or helper with the CUDA library and includes no CUDA header.
 *
 * What it computes (per sequence n and head h, tokens in order):
 *
 *   alpha_t = sigma(a_t)            beta_t = sigma(b_t)       (KDA,  signed_gate = 0)
 *   alpha_t = 2 sigma(a_t) - 1      beta_t = 2 sigma(b_t)     (CKDA, signed_gate = 1)
 *   alpha_t = a_t                   beta_t = b_t              (raw,  signed_gate = 2)
 *   alpha_t = 2 sigma(a_t) - 1      beta_t = sigma(b_t)       (gate range only, 3)
 *   alpha_t = sigma(a_t)            beta_t = 2 sigma(b_t)     (strength range only, 4)
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = S_t^T q_t
 *
 * Sources:
 *   - transition A_t = (I - beta k k^T) Diag(alpha): "Complex KDA: Understanding
 *     and Enhancing the Expressivity of Kimi Delta Attention" (paper review page),
 *     section "Diagonal-plus-rank-one (DPR1) transition";
 *   - ranges alpha = 2 sigma(a) - 1 in [-1,1], beta = 2 sigma(b) in [0,2]: same
 *     page, "Method steps", step 1; the standard KDA ranges (sigma) are the
 *     un-extended ones of the same section ("standard gates are non-negative");
 *   - write term beta k v^T: the delta rule S + k (v - S^T k)^T of the CyFA
 *     blog ("No delta rule needed ...", section 2.2) with gate and strength;
 *     expanding (I - beta k k^T) Diag(alpha) S + beta k v^T gives
 *     Diag(alpha) S + beta k (v - (Diag(alpha) S)^T k)^T, i.e. that rule;
 *   - state S in R^{dk x dv} (row = key channel) and key-side read S^T q:
 *     "Dual DeltaNet" abstract.
 *
 * The recurrence has no 1/sqrt(dk) scale on q (none appears on the pages);
 * o_t uses the state after token t's update.
 *
 * Layouts (all dense, row-major, float64):
 *   q, k, a : [B, T, H, dk]      v, o : [B, T, H, dv]     b : [B, T, H]
 *   S0, S_T : [N, H, dk, dv]     N = B, or n_seqs when cu_seqlens != NULL
 *   cu_seqlens (optional): N+1 non-decreasing offsets into T, B must be 1.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_SEQLENS (-2)
#define ORACLE_ERR_NOMEM (-3)

/* sigma(x) = 1 / (1 + e^{-x}); exact 1 at +inf and 0 at -inf. */
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/*
 * Gate activation, "Method steps" step 1 of the CKDA review (both ranges widened),
 * and the single-range variants of its "Experimental results" (Figure 6): the gate
 * range alone (3) or the strength range alone (4).  Per form: the gate is
 * sigma (0, 4), 2 sigma - 1 (1, 3) or the raw value (2); the strength is sigma
 * (0, 3), 2 sigma (1, 4) or the raw value (2).
 */
static int alpha_form(int signed_gate) {
    return signed_gate == 3 ? 1 : (signed_gate == 4 ? 0 : signed_gate);
}
static int beta_form(int signed_gate) {
    return signed_gate == 3 ? 0 : (signed_gate == 4 ? 1 : signed_gate);
}
static void gate_values(const double *a, double b, int n, int signed_gate,
                        double *alpha, double *beta) {
    const int af = alpha_form(signed_gate), bf = beta_form(signed_gate);
    for (int i = 0; i < n; ++i) {
        if (af == 0)
            alpha[i] = sigmoid(a[i]);
        else if (af == 1)
            alpha[i] = 2.0 * sigmoid(a[i]) - 1.0;
        else
            alpha[i] = a[i];
    }
    if (bf == 0)
        *beta = sigmoid(b);
    else if (bf == 1)
        *beta = 2.0 * sigmoid(b);
    else
        *beta = b;
}

/* Elementwise activation of n_a gate logits and n_b strength logits. */
void oracle_gates(const double *a, const double *b, int n_a, int n_b,
                  int signed_gate, double *alpha, double *beta) {
    if (n_a > 0) {
        double unused;
        gate_values(a, 0.0, n_a, signed_gate, alpha, &unused);
    }
    for (int i = 0; i < n_b; ++i) {
        double unused;
        gate_values(NULL, b[i], 0, signed_gate, &unused, &beta[i]);
    }
}

/*
 * One token on one head, in place on S [dk][dv]:
 *   S <- Diag(alpha) S ;  p = S^T k ;  S <- S + beta k (v - p)^T ;  o = S^T q
 * which is S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T, o_t = S_t^T q.
 */
static void token_step(double *S, const double *q, const double *k, const double *v,
                       const double *alpha, double beta, int dk, int dv,
                       double *o, double *p) {
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= alpha[i];
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += k[i] * S[(size_t)i * dv + j];
        p[j] = acc;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += beta * k[i] * (v[j] - p[j]);
    if (o) {
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += q[i] * S[(size_t)i * dv + j];
            o[j] = acc;
        }
    }
}

typedef struct {
    const double *q, *k, *v, *a, *b, *S0;
    const int32_t *cu;
    int n_seqs, B, T, H, dk, dv, signed_gate;
    double *o, *S_T;
    int n_units;
    int next_unit; /* guarded by lock */
    pthread_mutex_t lock;
    int status;
} fwd_job;

static void run_unit(fwd_job *J, int unit, double *S, double *alpha, double *p) {
    const int H = J->H, dk = J->dk, dv = J->dv, T = J->T;
    const int n = unit / H, h = unit % H;
    long t0, t1, bofs;
    if (J->cu) {
        t0 = J->cu[n];
        t1 = J->cu[n + 1];
        bofs = 0;
    } else {
        t0 = 0;
        t1 = T;
        bofs = (long)n * T;
    }
    const size_t sofs = ((size_t)n * H + h) * (size_t)dk * dv;
    if (J->S0)
        memcpy(S, J->S0 + sofs, sizeof(double) * (size_t)dk * dv);
    else
        memset(S, 0, sizeof(double) * (size_t)dk * dv);
    for (long t = t0; t < t1; ++t) {
        const size_t row = (size_t)(bofs + t) * H + h; /* token-head row */
        double beta;
        gate_values(J->a + row * dk, J->b[row], dk, J->signed_gate, alpha, &beta);
        token_step(S, J->q + row * dk, J->k + row * dk, J->v + row * dv, alpha, beta,
                   dk, dv, J->o ? J->o + row * dv : NULL, p);
    }
    if (J->S_T) memcpy(J->S_T + sofs, S, sizeof(double) * (size_t)dk * dv);
}

static void *fwd_worker(void *arg) {
    fwd_job *J = (fwd_job *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)J->dk * J->dv);
    double *alpha = (double *)malloc(sizeof(double) * (size_t)J->dk);
    double *p = (double *)malloc(sizeof(double) * (size_t)J->dv);
    if (!S || !alpha || !p) {
        pthread_mutex_lock(&J->lock);
        J->status = ORACLE_ERR_NOMEM;
        pthread_mutex_unlock(&J->lock);
        free(S); free(alpha); free(p);
        return NULL;
    }
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->n_units) break;
        run_unit(J, u, S, alpha, p);
    }
    free(S); free(alpha); free(p);
    return NULL;
}

/*
 * Sequential forward over every (sequence, head) unit.  Units are spread over
 * n_threads POSIX threads (n_threads <= 0: one per online core).  Any of o,
 * S_T may be NULL (not written); S0 NULL means a zero initial state.
 * Returns 0, or a negative code for bad arguments / bad offsets.
 */
int oracle_ckda_fwd(const double *q, const double *k, const double *v, const double *a,
                    const double *b, const double *S0, const int32_t *cu_seqlens,
                    int n_seqs, int B, int T, int H, int dk, int dv, int signed_gate,
                    double *o, double *S_T, int n_threads) {
    if (!q || !k || !v || !a || !b) return ORACLE_ERR_ARG;
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return ORACLE_ERR_ARG;
    if (signed_gate < 0 || signed_gate > 4) return ORACLE_ERR_ARG;
    int N = B;
    if (cu_seqlens) {
        if (B != 1 || n_seqs < 0) return ORACLE_ERR_ARG;
        if (cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != T) return ORACLE_ERR_SEQLENS;
        for (int i = 0; i < n_seqs; ++i)
            if (cu_seqlens[i + 1] < cu_seqlens[i]) return ORACLE_ERR_SEQLENS;
        N = n_seqs;
    }
    fwd_job J;
    J.q = q; J.k = k; J.v = v; J.a = a; J.b = b; J.S0 = S0; J.cu = cu_seqlens;
    J.n_seqs = n_seqs; J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
    J.signed_gate = signed_gate; J.o = o; J.S_T = S_T;
    J.n_units = N * H; J.next_unit = 0; J.status = ORACLE_OK;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        n_threads = nc > 0 ? (int)nc : 1;
    }
    if (n_threads > J.n_units) n_threads = J.n_units > 0 ? J.n_units : 1;
    if (n_threads <= 1) {
        fwd_worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
        if (!th) { pthread_mutex_destroy(&J.lock); return ORACLE_ERR_NOMEM; }
        int started = 0;
        for (int i = 0; i < n_threads; ++i)
            if (pthread_create(&th[i], NULL, fwd_worker, &J) == 0) ++started;
        if (started == 0) fwd_worker(&J);
        for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return J.status;
}

/*
 * One recurrent decode step for B x H heads, S [B,H,dk,dv] updated in place.
 * q, k, a: [B,H,dk]; v, o: [B,H,dv]; b: [B,H].  Same body as one token of
 * oracle_ckda_fwd.
 */
int oracle_decode_step(const double *q, const double *k, const double *v, const double *a,
                       const double *b, double *S, int B, int H, int dk, int dv,
                       int signed_gate, double *o) {
    if (!q || !k || !v || !a || !b || !S) return ORACLE_ERR_ARG;
    if (B < 0 || H <= 0 || dk <= 0 || dv <= 0) return ORACLE_ERR_ARG;
    if (signed_gate < 0 || signed_gate > 4) return ORACLE_ERR_ARG;
    double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
    double *p = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!alpha || !p) { free(alpha); free(p); return ORACLE_ERR_NOMEM; }
    for (long u = 0; u < (long)B * H; ++u) {
        double beta;
        gate_values(a + (size_t)u * dk, b[u], dk, signed_gate, alpha, &beta);
        token_step(S + (size_t)u * dk * dv, q + (size_t)u * dk, k + (size_t)u * dk,
                   v + (size_t)u * dv, alpha, beta, dk, dv, o ? o + (size_t)u * dv : NULL, p);
    }
    free(alpha); free(p);
    return ORACLE_OK;
}

/*
 * Explicit transition matrix A = (I - beta k k^T) Diag(alpha), n x n row-major:
 * A_ij = (delta_ij - beta k_i k_j) alpha_j.  Section "Diagonal-plus-rank-one
 * (DPR1) transition" of the CKDA review.
 */
void oracle_transition(const double *k, const double *alpha, double beta, int n, double *A) {
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j)
            A[(size_t)i * n + j] = ((i == j ? 1.0 : 0.0) - beta * k[i] * k[j]) * alpha[j];
}

/*
 * Second, explicit-matrix statement of the same forward for one sequence and
 * one head (tiny inputs only, O(dk^3) per token):
 *   S <- A_t S + beta_t k_t v_t^T  with A_t built densely;  o_t = S^T q_t.
 * q, k, a: [T, dk]; v, o: [T, dv]; b: [T]; S0, S_T: [dk, dv] (S0 may be NULL).
 */
int oracle_ckda_fwd_explicit(const double *q, const double *k, const double *v,
                             const double *a, const double *b, const double *S0,
                             int T, int dk, int dv, int signed_gate, double *o, double *S_T) {
    if (!q || !k || !v || !a || !b || !S_T) return ORACLE_ERR_ARG;
    if (T < 0 || dk <= 0 || dv <= 0 || signed_gate < 0 || signed_gate > 4) return ORACLE_ERR_ARG;
    double *A = (double *)malloc(sizeof(double) * (size_t)dk * dk);
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *N = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
    if (!A || !S || !N || !alpha) { free(A); free(S); free(N); free(alpha); return ORACLE_ERR_NOMEM; }
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)dk * dv);
    else memset(S, 0, sizeof(double) * (size_t)dk * dv);
    for (int t = 0; t < T; ++t) {
        double beta;
        const double *kt = k + (size_t)t * dk;
        gate_values(a + (size_t)t * dk, b[t], dk, signed_gate, alpha, &beta);
        oracle_transition(kt, alpha, beta, dk, A);
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int m = 0; m < dk; ++m) acc += A[(size_t)i * dk + m] * S[(size_t)m * dv + j];
                N[(size_t)i * dv + j] = acc + beta * kt[i] * v[(size_t)t * dv + j];
            }
        memcpy(S, N, sizeof(double) * (size_t)dk * dv);
        if (o)
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += q[(size_t)t * dk + i] * S[(size_t)i * dv + j];
                o[(size_t)t * dv + j] = acc;
            }
    }
    memcpy(S_T, S, sizeof(double) * (size_t)dk * dv);
    free(A); free(S); free(N); free(alpha);
    return ORACLE_OK;
}
