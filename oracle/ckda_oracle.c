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
 * Backward (oracle_ckda_bwd): the gradients of L = sum dO . o + sum dS_T . S_T
 * with respect to q, k, v, a, b and S0, by the chain rule taken through the
 * same token steps in reverse order (states recomputed from checkpoints).  The
 * pages give no backward formulas; they measure the kernels forward plus
 * backward ("Complex KDA" review, Figure 5), and the reverse pass here is the
 * plain derivative of the forward above, pinned by finite differences and
 * closed forms in the tests.
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

/*
 * Derivatives of the activations, same forms as gate_values:
 * sigma'(x) = sigma(x) sigma(-x) (so 0 at +-inf), twice that for 2 sigma - 1 and
 * 2 sigma, and 1 for raw values.
 */
static double sigmoid_deriv(double x) { return sigmoid(x) * sigmoid(-x); }
static void gate_derivs(const double *a, double b, int n, int signed_gate,
                        double *dalpha_da, double *dbeta_db) {
    const int af = alpha_form(signed_gate), bf = beta_form(signed_gate);
    for (int i = 0; i < n; ++i)
        dalpha_da[i] = af == 0 ? sigmoid_deriv(a[i]) : (af == 1 ? 2.0 * sigmoid_deriv(a[i]) : 1.0);
    *dbeta_db = bf == 0 ? sigmoid_deriv(b) : (bf == 1 ? 2.0 * sigmoid_deriv(b) : 1.0);
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
 * Reverse of token_step for one token.  S_prev = S_{t-1}, S_cur = S_t.  On entry
 * dS holds dL/dS_t from the later tokens (and dS_T); on return dL/dS_{t-1}.
 * Forward quantities:  St = Diag(alpha) S_prev,  p = St^T k,  u = beta (v - p),
 * S_t = St + k u^T,  o = S_t^T q.  Their adjoints, in reverse:
 *   o:   dS += q dO^T,            dq = S_t dO
 *   S_t: dSt = dS,  dk = dS u,    du = dS^T k
 *   u:   dbeta = du . (v - p),    dv = beta du,   dp = -beta du
 *   p:   dSt += k dp^T,           dk += St dp
 *   St:  dalpha_i = sum_j dSt_ij S_prev_ij,       dS_{t-1} = Diag(alpha) dSt
 * and da = dalpha * alpha'(a), db = dbeta * beta'(b).  dO may be NULL (zero).
 */
static void token_step_bwd(const double *S_prev, const double *S_cur, const double *q,
                           const double *k, const double *v, const double *alpha, double beta,
                           const double *dalpha_da, double dbeta_db, const double *dO,
                           int dk, int dv, double *dS, double *dq, double *dk_out,
                           double *dv_out, double *da, double *db, double *St, double *p,
                           double *du) {
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        if (dO)
            for (int j = 0; j < dv; ++j) {
                dS[(size_t)i * dv + j] += q[i] * dO[j];
                acc += S_cur[(size_t)i * dv + j] * dO[j];
            }
        dq[i] = acc;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) St[(size_t)i * dv + j] = alpha[i] * S_prev[(size_t)i * dv + j];
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += k[i] * St[(size_t)i * dv + j];
        p[j] = acc;
    }
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) acc += dS[(size_t)i * dv + j] * beta * (v[j] - p[j]);
        dk_out[i] = acc;
    }
    double dbeta = 0.0;
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += dS[(size_t)i * dv + j] * k[i];
        du[j] = acc;
        dbeta += acc * (v[j] - p[j]);
        dv_out[j] = beta * acc;
    }
    /* dp = -beta du */
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) acc += St[(size_t)i * dv + j] * (-beta * du[j]);
        dk_out[i] += acc;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += k[i] * (-beta * du[j]);
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) acc += dS[(size_t)i * dv + j] * S_prev[(size_t)i * dv + j];
        da[i] = acc * dalpha_da[i];
        for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] *= alpha[i];
    }
    *db = dbeta * dbeta_db;
}

typedef struct {
    const double *q, *k, *v, *a, *b, *S0, *dO, *dS_T;
    const int32_t *cu;
    int B, T, H, dk, dv, signed_gate;
    double *gq, *gk, *gv, *ga, *gb, *gS0; /* outputs: dq, dk, dv, da, db, dS0 */
    int n_units;
    int next_unit; /* guarded by lock */
    pthread_mutex_t lock;
    int status;
} bwd_job;

#define BWD_SEG 64 /* tokens between state checkpoints */

static int run_unit_bwd(bwd_job *J, int unit) {
    const int H = J->H, dk = J->dk, dv = J->dv;
    const int n = unit / H, h = unit % H;
    const size_t dd = (size_t)dk * dv;
    long t0, t1, bofs;
    if (J->cu) {
        t0 = J->cu[n];
        t1 = J->cu[n + 1];
        bofs = 0;
    } else {
        t0 = 0;
        t1 = J->T;
        bofs = (long)n * J->T;
    }
    const long len = t1 - t0;
    const long n_seg = (len + BWD_SEG - 1) / BWD_SEG;
    const size_t sofs = ((size_t)n * H + h) * dd;
    /* checkpoints: the state before each segment; states: one segment's S_{t-1}, S_t chain */
    double *ckpt = (double *)malloc(sizeof(double) * dd * (size_t)(n_seg > 0 ? n_seg : 1));
    double *states = (double *)malloc(sizeof(double) * dd * (BWD_SEG + 1));
    double *dS = (double *)malloc(sizeof(double) * dd);
    double *St = (double *)malloc(sizeof(double) * dd);
    double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
    double *dalpha = (double *)malloc(sizeof(double) * (size_t)dk);
    double *p = (double *)malloc(sizeof(double) * (size_t)dv);
    double *du = (double *)malloc(sizeof(double) * (size_t)dv);
    int rc = ORACLE_OK;
    if (!ckpt || !states || !dS || !St || !alpha || !dalpha || !p || !du) {
        rc = ORACLE_ERR_NOMEM;
        goto done;
    }
    /* forward, keeping the state at every segment start */
    if (J->S0) memcpy(St, J->S0 + sofs, sizeof(double) * dd);
    else memset(St, 0, sizeof(double) * dd);
    for (long t = t0; t < t1; ++t) {
        if ((t - t0) % BWD_SEG == 0) memcpy(ckpt + (size_t)((t - t0) / BWD_SEG) * dd, St, sizeof(double) * dd);
        const size_t row = (size_t)(bofs + t) * H + h;
        double beta;
        gate_values(J->a + row * dk, J->b[row], dk, J->signed_gate, alpha, &beta);
        token_step(St, J->q + row * dk, J->k + row * dk, J->v + row * dv, alpha, beta, dk, dv,
                   NULL, p);
    }
    if (J->dS_T) memcpy(dS, J->dS_T + sofs, sizeof(double) * dd);
    else memset(dS, 0, sizeof(double) * dd);
    for (long sg = n_seg - 1; sg >= 0; --sg) {
        const long s0 = t0 + sg * BWD_SEG;
        const long s1 = s0 + BWD_SEG < t1 ? s0 + BWD_SEG : t1;
        memcpy(states, ckpt + (size_t)sg * dd, sizeof(double) * dd);
        for (long t = s0; t < s1; ++t) {
            const size_t row = (size_t)(bofs + t) * H + h;
            double beta;
            double *S = states + (size_t)(t - s0 + 1) * dd;
            memcpy(S, S - dd, sizeof(double) * dd);
            gate_values(J->a + row * dk, J->b[row], dk, J->signed_gate, alpha, &beta);
            token_step(S, J->q + row * dk, J->k + row * dk, J->v + row * dv, alpha, beta, dk, dv,
                       NULL, p);
        }
        for (long t = s1 - 1; t >= s0; --t) {
            const size_t row = (size_t)(bofs + t) * H + h;
            double beta, dbeta_db;
            gate_values(J->a + row * dk, J->b[row], dk, J->signed_gate, alpha, &beta);
            gate_derivs(J->a + row * dk, J->b[row], dk, J->signed_gate, dalpha, &dbeta_db);
            const double *S_cur = states + (size_t)(t - s0 + 1) * dd;
            token_step_bwd(S_cur - dd, S_cur, J->q + row * dk, J->k + row * dk, J->v + row * dv,
                           alpha, beta, dalpha, dbeta_db, J->dO ? J->dO + row * dv : NULL, dk, dv,
                           dS, J->gq + row * dk, J->gk + row * dk, J->gv + row * dv,
                           J->ga + row * dk, J->gb + row, St, p, du);
        }
    }
    if (J->gS0) memcpy(J->gS0 + sofs, dS, sizeof(double) * dd);
done:
    free(ckpt); free(states); free(dS); free(St); free(alpha); free(dalpha); free(p); free(du);
    return rc;
}

static void *bwd_worker(void *arg) {
    bwd_job *J = (bwd_job *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->n_units) break;
        if (run_unit_bwd(J, u) != ORACLE_OK) {
            pthread_mutex_lock(&J->lock);
            J->status = ORACLE_ERR_NOMEM;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

/*
 * Gradients of L = sum dO . o + sum dS_T . S_T for the forward of oracle_ckda_fwd
 * (same arguments, layouts and gate forms).  dO [B,T,H,dv] and dS_T [N,H,dk,dv]
 * may each be NULL (zero).  Outputs, all written: dq, dk, da [B,T,H,dk],
 * dv [B,T,H,dv], db [B,T,H], dS0 [N,H,dk,dv] (dS0 may be NULL: not written).
 * Every token belongs to exactly one sequence (cu_seqlens[N] == T is required),
 * so every element of dq, dk, dv, da, db is written.
 */
int oracle_ckda_bwd(const double *q, const double *k, const double *v, const double *a,
                    const double *b, const double *S0, const int32_t *cu_seqlens,
                    int n_seqs, int B, int T, int H, int dk, int dv, int signed_gate,
                    const double *dO, const double *dS_T, double *dq, double *dk_out,
                    double *dv_out, double *da, double *db, double *dS0, int n_threads) {
    if (!q || !k || !v || !a || !b || !dq || !dk_out || !dv_out || !da || !db)
        return ORACLE_ERR_ARG;
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
    bwd_job J;
    J.q = q; J.k = k; J.v = v; J.a = a; J.b = b; J.S0 = S0; J.dO = dO; J.dS_T = dS_T;
    J.cu = cu_seqlens; J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
    J.signed_gate = signed_gate;
    J.gq = dq; J.gk = dk_out; J.gv = dv_out; J.ga = da; J.gb = db; J.gS0 = dS0;
    J.n_units = N * H; J.next_unit = 0; J.status = ORACLE_OK;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        n_threads = nc > 0 ? (int)nc : 1;
    }
    if (n_threads > J.n_units) n_threads = J.n_units > 0 ? J.n_units : 1;
    if (n_threads <= 1) {
        bwd_worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
        if (!th) { pthread_mutex_destroy(&J.lock); return ORACLE_ERR_NOMEM; }
        int started = 0;
        for (int i = 0; i < n_threads; ++i)
            if (pthread_create(&th[i], NULL, bwd_worker, &J) == 0) ++started;
        if (started == 0) bwd_worker(&J);
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

/*
 * DeltaProduct form: nh rank-one delta-rule updates per token, the gate applied once.
 * The CKDA review names DeltaProduct2 (two rank-one updates per token, "one more value
 * path") as the other route to plane rotations, with throughput comparable to KDA's
 * (sections "Research motivation" and "Experimental results" (5)); per token t:
 *
 *   S <- Diag(alpha_t) S
 *   for j = 1 .. nh:  S <- S + beta_tj k_tj (v_tj - S^T k_tj)^T
 *   o_t = S^T q_t
 *
 * i.e. S_t = (I - b_t2 k_t2 k_t2^T)(I - b_t1 k_t1 k_t1^T) Diag(alpha_t) S_{t-1} + writes.
 * Gate and strength forms as oracle_ckda_fwd (signed_gate 0..4).
 * Layouts: q, a [B,T,H,dk]; k [B,T,nh,H,dk]; v [B,T,nh,H,dv]; b [B,T,nh,H];
 * o [B,T,H,dv] (or NULL); S0, S_T [N,H,dk,dv].  One thread, unit after unit.
 */
int oracle_ckda_fwd_product(const double *q, const double *k, const double *v, const double *a,
                            const double *b, const double *S0, const int32_t *cu_seqlens,
                            int n_seqs, int B, int T, int H, int dk, int dv, int nh,
                            int signed_gate, double *o, double *S_T) {
    if (!q || !k || !v || !a || !b || !S_T) return ORACLE_ERR_ARG;
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || nh < 1) return ORACLE_ERR_ARG;
    if (signed_gate < 0 || signed_gate > 4) return ORACLE_ERR_ARG;
    int N = B;
    if (cu_seqlens) {
        if (B != 1 || n_seqs < 0) return ORACLE_ERR_ARG;
        if (cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != T) return ORACLE_ERR_SEQLENS;
        for (int i = 0; i < n_seqs; ++i)
            if (cu_seqlens[i + 1] < cu_seqlens[i]) return ORACLE_ERR_SEQLENS;
        N = n_seqs;
    }
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
    double *pr = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!S || !alpha || !pr) { free(S); free(alpha); free(pr); return ORACLE_ERR_NOMEM; }
    for (int n = 0; n < N; ++n) {
        const long t0 = cu_seqlens ? cu_seqlens[n] : 0, t1 = cu_seqlens ? cu_seqlens[n + 1] : T;
        const long tok0 = cu_seqlens ? 0 : (long)n * T;  /* token row of t = 0 */
        for (int h = 0; h < H; ++h) {
            const size_t sofs = ((size_t)n * H + h) * (size_t)dk * dv;
            for (size_t e = 0; e < (size_t)dk * dv; ++e) S[e] = S0 ? S0[sofs + e] : 0.0;
            for (long t = t0; t < t1; ++t) {
                const size_t row = (size_t)(tok0 + t) * H + h;
                double unused;
                gate_values(a + row * dk, 0.0, dk, signed_gate, alpha, &unused);
                for (int i = 0; i < dk; ++i)
                    for (int c = 0; c < dv; ++c) S[(size_t)i * dv + c] *= alpha[i];
                for (int j = 0; j < nh; ++j) {
                    /* key, value and strength j of token t */
                    const size_t sub = ((size_t)(tok0 + t) * nh + j) * H + h;
                    const double *kj = k + sub * dk, *vj = v + sub * dv;
                    double bj;
                    gate_values(NULL, b[sub], 0, signed_gate, &unused, &bj);
                    for (int c = 0; c < dv; ++c) {
                        double acc = 0.0;
                        for (int i = 0; i < dk; ++i) acc += kj[i] * S[(size_t)i * dv + c];
                        pr[c] = acc;
                    }
                    for (int i = 0; i < dk; ++i)
                        for (int c = 0; c < dv; ++c)
                            S[(size_t)i * dv + c] += bj * kj[i] * (vj[c] - pr[c]);
                }
                if (o)
                    for (int c = 0; c < dv; ++c) {
                        double acc = 0.0;
                        for (int i = 0; i < dk; ++i) acc += q[row * dk + i] * S[(size_t)i * dv + c];
                        o[row * dv + c] = acc;
                    }
            }
            memcpy(S_T + sofs, S, sizeof(double) * (size_t)dk * dv);
        }
    }
    free(S); free(alpha); free(pr);
    return ORACLE_OK;
}
