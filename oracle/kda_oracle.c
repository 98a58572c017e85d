/*
 * KDA oracle: plain, slow, fp64 CPU implementation of the fine-grained gated
 * delta rule. TEST INFRASTRUCTURE ONLY. It is called by tests/, by
 * __graft_entry__.smoke() and by bench.py's CPU-baseline leg, never by the
 * product path. It shares no code, header or constant with the CUDA library.
 *
 * What it follows (pages of the subject, by title and section):
 *   "Decoding Hybrid Attention Architectures", section 3.4 (fine-grained
 *   gating) and the variant table of section 3.4: the state update
 *       S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T,
 *   read with S in R^{dk x dv} (rows = key channels), write term k v^T and
 *   readout o_t = S_t^T q_t; section 3.2 for the meaning of beta (update
 *   proportional to the difference between the new value and the stored one).
 *   "Technical Analysis ... Novel Hybrid Linear Attention", section 2 item 4
 *   (same update, Diag(a_t) per feature channel).
 *   Section 4 of the first page and section 3 of the second page for the
 *   chunkwise form (intra-chunk lower-triangular products, inter-chunk state
 *   passing, precomputed U and W); the exact decay placement used below is
 *   this oracle's own derivation from the recurrence (the printed chunk
 *   formulas are symbolic and garbled).
 *
 * Inputs are fp64. Layouts (row-major, contiguous):
 *   q, k, log_alpha : [B, T, H, dk]      v, o : [B, T, H, dv]
 *   beta            : [B, T, H]          S0, ST : [B, H, dk, dv]
 * alpha = exp(log_alpha); no activation, no q scaling.
 *
 * Variants (same pages, section 3.4 variant table and sections 3.1-3.3, plus
 * the per-dimension gated linear attention named beside it). Two switches:
 *   erase = 1: delta-rule family, S_t = (I - b k k^T) Diag(a_t) S_{t-1} + b k v^T
 *   erase = 0: linear-attention family, S_t = Diag(a_t) S_{t-1} + b k v^T
 *              (no erase term; b = 1 gives the pages' plain write k v^T)
 *   gate  = 0: a_t = exp(log_alpha) per key channel, log_alpha [B, T, H, dk]
 *   gate  = 1: one decay per token and head, log_alpha [B, T, H] (scalar gated
 *              delta rule: the scalar commutes with the erase term)
 *   gate  = 2: no decay (a_t = 1); log_alpha is not read (may be NULL)
 * So (erase, gate) = (1, 0) is KDA, (1, 1) the scalar gated delta rule, (1, 2)
 * the delta rule, (0, 0) per-dimension gated linear attention, (0, 2) with
 * beta = 1 pure linear attention.
 *
 * Pins: every function here is checked by tests/test_oracle.py against
 * closed forms (identity, linear attention with orthogonal keys, pure decay),
 * the exact-retrieval invariant, an independent scalar-gate recurrence,
 * brute-force agreement of the two formulations, state-passing and decode
 * chaining invariants, and ||(I+A)T - I||. The "mutation" argument exists only
 * so that a test can plant a mistake here and see a pin fail.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* Planted mistakes, used only by the mutation test. 0 = correct oracle. */
enum {
    MUT_NONE = 0,
    MUT_NO_DECAY = 1,        /* skip Diag(alpha)                              */
    MUT_DECAY_AFTER = 2,     /* decay applied after erase+write               */
    MUT_ERASE_SIGN = 3,      /* + instead of - on the erase term              */
    MUT_READ_BEFORE = 4,     /* o_t read from S_{t-1}                         */
    MUT_TRANSPOSED_READ = 5, /* o = S q instead of S^T q (needs dk == dv)     */
    MUT_BETA_WRITE_ONLY = 6, /* beta on the write only, not on the erase      */
    MUT_DECAY_COLUMNS = 7,   /* decay scales value channels (needs dk == dv)  */
    MUT_PREFIX_DECAY_K = 8,  /* chunkwise: prefix decay on K in state update  */
    MUT_STRICT_TRIL_O = 9,   /* chunkwise: strict instead of inclusive mask   */
    MUT_ERASE_ALWAYS = 10,   /* erase = 0 still applies the erase term        */
    MUT_SCALAR_GATE_TWICE = 11, /* gate = 1 applies the scalar decay twice    */
};

typedef struct {
    const double *q, *k, *v, *la, *beta, *S0;
    double *o, *ST;
    double *dbg_A, *dbg_T; /* chunkwise only: [B,H,NC,C,C] or NULL */
    int B, T, H, dk, dv, C, mutation;
    int erase, gate; /* variant switches, see the header */
    int next_head; /* shared work counter */
    pthread_mutex_t lock;
} job_t;

static int take_head(job_t *J) {
    pthread_mutex_lock(&J->lock);
    int h = J->next_head++;
    pthread_mutex_unlock(&J->lock);
    return h;
}

/* log a_t for key channel c of token t (see the gate switch). */
static double log_decay(const job_t *J, int b, int t, int h, int c) {
    if (J->gate == 2) return 0.0;
    if (J->gate == 1) {
        const double g = J->la[((long)b * J->T + t) * J->H + h];
        return (J->mutation == MUT_SCALAR_GATE_TWICE) ? 2.0 * g : g;
    }
    return J->la[(((long)b * J->T + t) * J->H + h) * J->dk + c];
}

/* Token-by-token recurrence for one (b, h). */
static void recurrent_head(job_t *J, int b, int h) {
    const int T = J->T, H = J->H, dk = J->dk, dv = J->dv, mut = J->mutation;
    double *S = (double *)malloc(sizeof(double) * dk * dv);
    double *u = (double *)malloc(sizeof(double) * dv);
    double *w = (double *)malloc(sizeof(double) * dv);
    double *lat = (double *)malloc(sizeof(double) * (dk > dv ? dk : dv));
    const long sbase = ((long)b * H + h) * dk * dv;
    if (J->S0) memcpy(S, J->S0 + sbase, sizeof(double) * dk * dv);
    else memset(S, 0, sizeof(double) * dk * dv);

    for (int t = 0; t < T; ++t) {
        const long tk = (((long)b * T + t) * H + h) * dk;
        const long tv = (((long)b * T + t) * H + h) * dv;
        const double *qt = J->q + tk, *kt = J->k + tk;
        for (int i = 0; i < dk; ++i) lat[i] = log_decay(J, b, t, h, i);
        const double *vt = J->v + tv;
        const double bt = J->beta[((long)b * T + t) * H + h];
        double *ot = J->o + tv;

        if (mut == MUT_READ_BEFORE) {
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * qt[i];
                ot[j] = acc;
            }
        }
        /* S <- Diag(alpha) S : row i (key channel i) scaled by alpha_i. */
        if (mut != MUT_NO_DECAY && mut != MUT_DECAY_AFTER) {
            for (int i = 0; i < dk; ++i) {
                const double a = (mut == MUT_DECAY_COLUMNS) ? 1.0 : exp(lat[i]);
                for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;
            }
            if (mut == MUT_DECAY_COLUMNS)
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) S[i * dv + j] *= exp(lat[j]);
        }
        /* u = S^T k : what the memory currently returns for key k. */
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * kt[i];
            u[j] = acc;
        }
        /* (I - b k k^T) S + b k v^T  ==  S + k (b (v - u))^T;  no erase: S + k (b v)^T */
        for (int j = 0; j < dv; ++j) {
            if (!J->erase && mut != MUT_ERASE_ALWAYS) w[j] = bt * vt[j];
            else if (mut == MUT_ERASE_SIGN) w[j] = bt * (vt[j] + u[j]);
            else if (mut == MUT_BETA_WRITE_ONLY) w[j] = bt * vt[j] - u[j];
            else w[j] = bt * (vt[j] - u[j]);
        }
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * w[j];
        if (mut == MUT_DECAY_AFTER) {
            for (int i = 0; i < dk; ++i) {
                const double a = exp(lat[i]);
                for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;
            }
        }
        /* o_t = S_t^T q_t */
        if (mut == MUT_TRANSPOSED_READ) {
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[j * dv + i] * qt[i];
                ot[j] = acc;
            }
        } else if (mut != MUT_READ_BEFORE) {
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * qt[i];
                ot[j] = acc;
            }
        }
    }
    if (J->ST) memcpy(J->ST + sbase, S, sizeof(double) * dk * dv);
    free(S);
    free(u);
    free(w);
    free(lat);
}

/*
 * Chunkwise reformulation for one (b, h), derived from the recurrence.
 * Within a chunk of n tokens with local cumulative log-decay
 * G_r = sum_{s<=r} log_alpha_s (per key channel) and chunk-start state S:
 *   A_rs = beta_r sum_c k_rc k_sc exp(G_rc - G_sc)        (s <  r), else 0
 *   P_rs = sum_c q_rc k_sc exp(G_rc - G_sc)                (s <= r), else 0
 *   T    = (I + A)^{-1}                 (unit lower triangular, substitution)
 *   W    = T (beta * K * exp(G)),   U = T (beta * V)
 *   D    = U - W S                  (per-token corrected write)
 *   O    = (Q * exp(G)) S + P D
 *   S'   = Diag(exp(G_last)) S + (K * exp(G_last - G))^T D
 * The tail chunk simply has fewer rows. exp arguments are all <= 0 here.
 */
static void chunkwise_head(job_t *J, int b, int h) {
    const int T = J->T, H = J->H, dk = J->dk, dv = J->dv, C = J->C, mut = J->mutation;
    const int erase = J->erase || mut == MUT_ERASE_ALWAYS;
    const int NC = (T + C - 1) / C;
    double *S = (double *)malloc(sizeof(double) * dk * dv);
    double *G = (double *)malloc(sizeof(double) * C * dk);
    double *A = (double *)malloc(sizeof(double) * C * C);
    double *P = (double *)malloc(sizeof(double) * C * C);
    double *Ti = (double *)malloc(sizeof(double) * C * C);
    double *W = (double *)malloc(sizeof(double) * C * dk);
    double *U = (double *)malloc(sizeof(double) * C * dv);
    double *D = (double *)malloc(sizeof(double) * C * dv);
    double *X = (double *)malloc(sizeof(double) * C * dk);
    double *Sn = (double *)malloc(sizeof(double) * dk * dv);
    const long sbase = ((long)b * H + h) * dk * dv;
    if (J->S0) memcpy(S, J->S0 + sbase, sizeof(double) * dk * dv);
    else memset(S, 0, sizeof(double) * dk * dv);

#define IDXK(t) ((((long)b * T + (t)) * H + h) * dk)
#define IDXV(t) ((((long)b * T + (t)) * H + h) * dv)
#define BETA(t) (J->beta[((long)b * T + (t)) * H + h])

    for (int ci = 0; ci < NC; ++ci) {
        const int t0 = ci * C;
        const int n = (T - t0 < C) ? (T - t0) : C;
        /* G: inclusive prefix sum of log-decay inside the chunk. */
        for (int c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int r = 0; r < n; ++r) {
                acc += log_decay(J, b, t0 + r, h, c);
                G[r * dk + c] = acc;
            }
        }
        /* A (strictly lower) and P (lower incl. diagonal). */
        for (int r = 0; r < n; ++r) {
            const double *kr = J->k + IDXK(t0 + r), *qr = J->q + IDXK(t0 + r);
            for (int s = 0; s < n; ++s) {
                double a = 0.0, p = 0.0;
                const int incl = (mut == MUT_STRICT_TRIL_O) ? (s < r) : (s <= r);
                if (s <= r) {
                    const double *ks = J->k + IDXK(t0 + s);
                    for (int c = 0; c < dk; ++c) {
                        const double e = exp(G[r * dk + c] - G[s * dk + c]);
                        a += kr[c] * ks[c] * e;
                        p += qr[c] * ks[c] * e;
                    }
                }
                /* no erase: the chunk's tokens do not correct one another */
                A[r * C + s] = (s < r && erase) ? BETA(t0 + r) * a : 0.0;
                P[r * C + s] = incl ? p : 0.0;
            }
        }
        /* T = (I + A)^{-1}: row r of T solves T_r + sum_{s<r} A_rs T_s = e_r. */
        for (int r = 0; r < n; ++r) {
            for (int j = 0; j < n; ++j) {
                double acc = (r == j) ? 1.0 : 0.0;
                for (int s = j; s < r; ++s) acc -= A[r * C + s] * Ti[s * C + j];
                Ti[r * C + j] = (j <= r) ? acc : 0.0;
            }
        }
        if (J->dbg_A || J->dbg_T) {
            const long off = (((long)b * H + h) * NC + ci) * C * C;
            for (int r = 0; r < C; ++r)
                for (int s = 0; s < C; ++s) {
                    const int in = (r < n && s < n);
                    if (J->dbg_A) J->dbg_A[off + r * C + s] = in ? A[r * C + s] : 0.0;
                    if (J->dbg_T) J->dbg_T[off + r * C + s] = in ? Ti[r * C + s] : (r == s);
                }
        }
        /* X = beta * K * exp(G);  W = T X;  U = T (beta * V). */
        for (int r = 0; r < n; ++r) {
            const double br = BETA(t0 + r);
            for (int c = 0; c < dk; ++c)
                X[r * dk + c] = br * J->k[IDXK(t0 + r) + c] * exp(G[r * dk + c]);
        }
        for (int r = 0; r < n; ++r) {
            for (int c = 0; c < dk; ++c) {
                double acc = 0.0;
                for (int s = 0; s <= r; ++s) acc += Ti[r * C + s] * X[s * dk + c];
                W[r * dk + c] = acc;
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int s = 0; s <= r; ++s) acc += Ti[r * C + s] * BETA(t0 + s) * J->v[IDXV(t0 + s) + j];
                U[r * dv + j] = acc;
            }
        }
        /* D = U - W S  (no erase: W S is not subtracted, D = beta V) */
        for (int r = 0; r < n; ++r)
            for (int j = 0; j < dv; ++j) {
                double acc = U[r * dv + j];
                if (erase)
                    for (int c = 0; c < dk; ++c) acc -= W[r * dk + c] * S[c * dv + j];
                D[r * dv + j] = acc;
            }
        /* O = (Q * exp(G)) S + P D */
        for (int r = 0; r < n; ++r) {
            const double *qr = J->q + IDXK(t0 + r);
            double *orow = J->o + IDXV(t0 + r);
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) acc += qr[c] * exp(G[r * dk + c]) * S[c * dv + j];
                for (int s = 0; s <= r; ++s) acc += P[r * C + s] * D[s * dv + j];
                orow[j] = acc;
            }
        }
        /* S' = Diag(exp(G_last)) S + (K * exp(G_last - G))^T D */
        for (int c = 0; c < dk; ++c) {
            const double gl = G[(n - 1) * dk + c];
            const double gam = exp(gl);
            for (int j = 0; j < dv; ++j) {
                double acc = gam * S[c * dv + j];
                for (int r = 0; r < n; ++r) {
                    const double kd = (mut == MUT_PREFIX_DECAY_K) ? exp(G[r * dk + c])
                                                                  : exp(gl - G[r * dk + c]);
                    acc += J->k[IDXK(t0 + r) + c] * kd * D[r * dv + j];
                }
                Sn[c * dv + j] = acc;
            }
        }
        memcpy(S, Sn, sizeof(double) * dk * dv);
    }
#undef IDXK
#undef IDXV
#undef BETA
    if (J->ST) memcpy(J->ST + sbase, S, sizeof(double) * dk * dv);
    free(S); free(G); free(A); free(P); free(Ti); free(W); free(U); free(D); free(X); free(Sn);
}

typedef struct { job_t *J; int chunkwise; } worker_arg_t;

static void *worker(void *p) {
    worker_arg_t *w = (worker_arg_t *)p;
    job_t *J = w->J;
    const int nh = J->B * J->H;
    for (;;) {
        const int id = take_head(J);
        if (id >= nh) break;
        if (w->chunkwise) chunkwise_head(J, id / J->H, id % J->H);
        else recurrent_head(J, id / J->H, id % J->H);
    }
    return NULL;
}

static int run(job_t *J, int chunkwise, int nthreads) {
    if (J->B < 0 || J->T < 0 || J->H < 0 || J->dk <= 0 || J->dv <= 0) return 1;
    if (chunkwise && J->C <= 0) return 1;
    if ((J->mutation == MUT_TRANSPOSED_READ || J->mutation == MUT_DECAY_COLUMNS) && J->dk != J->dv) return 1;
    const int nh = J->B * J->H;
    if (nh == 0) return 0;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads > nh) nthreads = nh;
    if (nthreads < 1) nthreads = 1;
    J->next_head = 0;
    pthread_mutex_init(&J->lock, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    worker_arg_t arg = {J, chunkwise};
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &arg);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return 0;
}

/* Token-by-token fp64 recurrence over all (b, h), variant (erase, gate). S0
 * may be NULL (zero state); ST may be NULL. nthreads <= 0 uses every online
 * core. Returns 0 on success, 1 on bad sizes or switches. */
int kda_oracle_recurrent_v(const double *q, const double *k, const double *v, const double *log_alpha,
                           const double *beta, const double *S0, double *o, double *ST,
                           int B, int T, int H, int dk, int dv, int erase, int gate, int nthreads,
                           int mutation) {
    job_t J;
    memset(&J, 0, sizeof(J));
    if ((erase != 0 && erase != 1) || gate < 0 || gate > 2 || (gate != 2 && !log_alpha)) return 1;
    J.q = q; J.k = k; J.v = v; J.la = log_alpha; J.beta = beta; J.S0 = S0; J.o = o; J.ST = ST;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.mutation = mutation;
    J.erase = erase; J.gate = gate;
    return run(&J, 0, nthreads);
}

/* The KDA recurrence (erase = 1, per-channel gate). */
int kda_oracle_recurrent(const double *q, const double *k, const double *v, const double *log_alpha,
                         const double *beta, const double *S0, double *o, double *ST,
                         int B, int T, int H, int dk, int dv, int nthreads, int mutation) {
    return kda_oracle_recurrent_v(q, k, v, log_alpha, beta, S0, o, ST, B, T, H, dk, dv, 1, 0, nthreads,
                                  mutation);
}

/* fp64 chunkwise reformulation with chunk size C (any C >= 1; the last chunk
 * may be shorter), variant (erase, gate). dbg_A / dbg_T, if non-NULL, receive
 * the per-chunk A and (I+A)^{-1} as [B, H, ceil(T/C), C, C] (padding
 * rows/cols: 0 for A, identity for T). */
int kda_oracle_chunkwise_v(const double *q, const double *k, const double *v, const double *log_alpha,
                           const double *beta, const double *S0, double *o, double *ST,
                           int B, int T, int H, int dk, int dv, int C, double *dbg_A, double *dbg_T,
                           int erase, int gate, int nthreads, int mutation) {
    job_t J;
    memset(&J, 0, sizeof(J));
    if ((erase != 0 && erase != 1) || gate < 0 || gate > 2 || (gate != 2 && !log_alpha)) return 1;
    J.q = q; J.k = k; J.v = v; J.la = log_alpha; J.beta = beta; J.S0 = S0; J.o = o; J.ST = ST;
    J.dbg_A = dbg_A; J.dbg_T = dbg_T;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.C = C; J.mutation = mutation;
    J.erase = erase; J.gate = gate;
    return run(&J, 1, nthreads);
}

/* The KDA chunkwise form (erase = 1, per-channel gate). */
int kda_oracle_chunkwise(const double *q, const double *k, const double *v, const double *log_alpha,
                         const double *beta, const double *S0, double *o, double *ST,
                         int B, int T, int H, int dk, int dv, int C, double *dbg_A, double *dbg_T,
                         int nthreads, int mutation) {
    return kda_oracle_chunkwise_v(q, k, v, log_alpha, beta, S0, o, ST, B, T, H, dk, dv, C, dbg_A, dbg_T, 1, 0,
                                  nthreads, mutation);
}

/* One recurrent decode step for N sequences x H heads: the recurrence with
 * T = 1, variant (erase, gate). Layouts: q, k [N, H, dk]; log_alpha [N, H, dk]
 * (gate 0), [N, H] (gate 1) or unused (gate 2); v, o [N, H, dv]; beta [N, H];
 * S_in, S_out [N, H, dk, dv] (S_out may equal S_in). */
int kda_oracle_decode_step_v(const double *q, const double *k, const double *v, const double *log_alpha,
                             const double *beta, const double *S_in, double *S_out, double *o,
                             int N, int H, int dk, int dv, int erase, int gate, int nthreads) {
    return kda_oracle_recurrent_v(q, k, v, log_alpha, beta, S_in, o, S_out, N, 1, H, dk, dv, erase, gate,
                                  nthreads, 0);
}

int kda_oracle_decode_step(const double *q, const double *k, const double *v, const double *log_alpha,
                           const double *beta, const double *S_in, double *S_out, double *o,
                           int N, int H, int dk, int dv, int nthreads) {
    return kda_oracle_decode_step_v(q, k, v, log_alpha, beta, S_in, S_out, o, N, H, dk, dv, 1, 0, nthreads);
}
