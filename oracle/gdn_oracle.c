/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle for the gated delta-rule recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check of the package entry file and
 * the CPU-baseline leg of the benchmark may load this library.  The product path (the CUDA
 * library and its Python binding) never calls it, and the two share no code.
 *
 * What it computes (the plain definition, one token at a time, no chunking):
 *
 *   per (sequence, head), state S in R^{dk x dv} (row-major, dv fastest):
 *     a_t = exp(log_alpha_t)                      forget gate in [0, 1]; log_alpha = -inf -> 0
 *     b_t = beta_t                                writing strength in [0, 2]
 *     S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T
 *     o_t = S_t^T q_t                             read-out uses the post-update state, no scale
 *
 * Sources:
 *   - Sykra README, "Architectural Highlights": Gated DeltaNet layer with a data-dependent forget
 *     gate alpha_t, O(d^2) per-token decode of a fixed d x d state.
 *   - DeltaPhase README, section 1 "Extended Householder Beta Range": beta in (0, 2); beta = 2 is
 *     an exact Householder reflection of the state.
 *   - DeltaPhase README, section 2 "Complex Phase Matrix Delta Memory": the delta rule as memory
 *     read-out -> error -> rank-one correction.  Written out for real vectors with the gate on
 *     the previous state, the update above is the same thing:
 *       S_t = a_t S_{t-1} + k_t u_t^T,  u_t = b_t (v_t - a_t S_{t-1}^T k_t).
 *     The loop below evaluates the first (product) form literally.
 *
 * Layouts (all contiguous, row-major):
 *   dense  : q,k [B,T,H,dk]  v,out [B,T,H,dv]  log_alpha,beta [B,T,H]  S0,S_final [B,H,dk,dv]
 *   varlen : cu_seqlens != NULL, int32 [B+1]; q,k [T,H,dk] etc. packed, sequence s owns tokens
 *            cu_seqlens[s] .. cu_seqlens[s+1]-1; states [B,H,dk,dv]
 *   decode : q,k [N,H,dk]  v,out [N,H,dv]  log_alpha,beta [N,H]  S_inout [N,H,dk,dv]
 * S0 == NULL means a zero initial state; S_final == NULL means the final state is not written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One token of the recurrence on one (sequence, head) state. kS is scratch of length dv. */
static void oracle_token(double *S, const double *q, const double *k, const double *v,
                         double log_alpha, double beta, double *o, double *kS, int dk, int dv)
{
    const double a = exp(log_alpha); /* exp(-inf) == 0: an exact reset */
    const double b = beta;
    /* kS = k^T S_{t-1}  (the memory read-out at key k) */
    for (int j = 0; j < dv; ++j) kS[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double ki = k[i];
        const double *Si = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) kS[j] += ki * Si[j];
    }
    /* S_t = a (S - b k (k^T S)) + b k v^T, entry by entry */
    for (int i = 0; i < dk; ++i) {
        const double ki = k[i];
        double *Si = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) Si[j] = a * (Si[j] - b * ki * kS[j]) + b * ki * v[j];
    }
    /* o_t = S_t^T q */
    if (o) {
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double qi = q[i];
            const double *Si = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) o[j] += qi * Si[j];
        }
    }
}

static int set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Number of threads the OpenMP runtime would use (1 without OpenMP). */
int gdn_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Whole-sequence forward by the sequential definition.
 *   units / n_units: optional list of (sequence * H + head) indices to compute; NULL = all.
 *   Outputs of units not listed are left untouched.
 * Returns 0, or -1 for invalid sizes.
 */
int gdn_oracle_forward(const double *q, const double *k, const double *v,
                       const double *log_alpha, const double *beta, const double *S0,
                       double *out, double *S_final, int B, int T, int H, int dk, int dv,
                       const int32_t *cu_seqlens, const int32_t *units, int n_units,
                       int nthreads)
{
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    set_threads(nthreads);
    const int total = units ? n_units : B * H;
    const size_t state = (size_t)dk * dv;
    int bad = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * state);
        double *kS = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!S || !kS) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int n = 0; n < total; ++n) {
            if (!S || !kS) continue;
            const int u = units ? units[n] : n;
            if (u < 0 || u >= B * H) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            const int s = u / H, h = u % H;
            long tok0, ntok;
            if (cu_seqlens) {
                tok0 = cu_seqlens[s];
                ntok = (long)cu_seqlens[s + 1] - cu_seqlens[s];
            } else {
                tok0 = (long)s * T;
                ntok = T;
            }
            if (S0) memcpy(S, S0 + (size_t)u * state, sizeof(double) * state);
            else memset(S, 0, sizeof(double) * state);
            for (long t = tok0; t < tok0 + ntok; ++t) {
                const size_t th = (size_t)t * H + h;
                oracle_token(S, q + th * dk, k + th * dk, v + th * dv, log_alpha[th], beta[th],
                             out ? out + th * dv : NULL, kS, dk, dv);
            }
            if (S_final) memcpy(S_final + (size_t)u * state, S, sizeof(double) * state);
        }
        free(S);
        free(kS);
    }
    return bad ? -1 : 0;
}

/*
 * Gradients of the whole-sequence forward by reverse mode over the same sequential definition.
 *   dout: dL/dout (layout of out); dS_final: dL/dS_final or NULL (zero).
 *   Writes dq, dk, dv_ (layouts of q, k, v), dlog_alpha, dbeta (layouts of the gates) and dS0
 *   (layout of S0; may be NULL).  Each unit keeps all of its states S_0 .. S_T (meant for the
 *   short sequences of the tests).
 * Per token, with G = dL/dS_t (after adding the read-out's q_t do_t^T), u = S_{t-1}^T k and
 * r = G^T k, the chain rule through S_t = a (S - b k (k^T S)) + b k v^T gives
 *     dq_t = S_t do_t,  dv_t = b r,  dbeta_t = r . (v - a u),
 *     dlog_alpha_t = a <G, S_{t-1} - b k u^T>   (0 at an exact reset, a = 0),
 *     dk_t = G b (v - a u) - a b S_{t-1} r,      dL/dS_{t-1} = a (G - b k r^T).
 * Returns 0, or -1 for invalid sizes or a failed allocation.
 */
int gdn_oracle_backward(const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *beta, const double *S0,
                        const double *dout, const double *dS_final, double *dq, double *dk,
                        double *dv_, double *dlog_alpha, double *dbeta, double *dS0, int B, int T,
                        int H, int dk_, int dv, const int32_t *cu_seqlens, int nthreads)
{
    const int DK = dk_;
    if (B < 0 || T < 0 || H <= 0 || DK <= 0 || dv <= 0) return -1;
    set_threads(nthreads);
    const size_t state = (size_t)DK * dv;
    int bad = 0;
#pragma omp parallel
    {
        double *kS = (double *)malloc(sizeof(double) * (size_t)dv);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        double *r = (double *)malloc(sizeof(double) * (size_t)dv);
        double *G = (double *)malloc(sizeof(double) * state);
        if (!kS || !u || !r || !G) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int un = 0; un < B * H; ++un) {
            if (!kS || !u || !r || !G) continue;
            const int s = un / H, h = un % H;
            long tok0, ntok;
            if (cu_seqlens) {
                tok0 = cu_seqlens[s];
                ntok = (long)cu_seqlens[s + 1] - cu_seqlens[s];
            } else {
                tok0 = (long)s * T;
                ntok = T;
            }
            double *St = (double *)malloc(sizeof(double) * state * (size_t)(ntok + 1));
            if (!St) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            /* forward, keeping S_0 .. S_ntok */
            if (S0) memcpy(St, S0 + (size_t)un * state, sizeof(double) * state);
            else memset(St, 0, sizeof(double) * state);
            for (long t = 0; t < ntok; ++t) {
                const size_t th = (size_t)(tok0 + t) * H + h;
                memcpy(St + (size_t)(t + 1) * state, St + (size_t)t * state, sizeof(double) * state);
                oracle_token(St + (size_t)(t + 1) * state, q + th * DK, k + th * DK, v + th * dv,
                             log_alpha[th], beta[th], NULL, kS, DK, dv);
            }
            /* reverse */
            if (dS_final) memcpy(G, dS_final + (size_t)un * state, sizeof(double) * state);
            else memset(G, 0, sizeof(double) * state);
            for (long t = ntok - 1; t >= 0; --t) {
                const size_t th = (size_t)(tok0 + t) * H + h;
                const double *S_t = St + (size_t)(t + 1) * state, *Sp = St + (size_t)t * state;
                const double *qt = q + th * DK, *kt = k + th * DK, *vt = v + th * dv, *dot = dout + th * dv;
                const double a = exp(log_alpha[th]), b = beta[th];
                /* read-out o_t = S_t^T q_t */
                for (int i = 0; i < DK; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        acc += S_t[(size_t)i * dv + j] * dot[j];
                        G[(size_t)i * dv + j] += qt[i] * dot[j];
                    }
                    dq[th * DK + i] = acc;
                }
                /* the update */
                for (int j = 0; j < dv; ++j) {
                    double uj = 0.0, rj = 0.0;
                    for (int i = 0; i < DK; ++i) {
                        uj += kt[i] * Sp[(size_t)i * dv + j];
                        rj += kt[i] * G[(size_t)i * dv + j];
                    }
                    u[j] = uj;
                    r[j] = rj;
                }
                double db = 0.0, da = 0.0;
                for (int j = 0; j < dv; ++j) {
                    dv_[th * dv + j] = b * r[j];
                    db += r[j] * (vt[j] - a * u[j]);
                }
                for (int i = 0; i < DK; ++i) {
                    double dki = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        const double g = G[(size_t)i * dv + j];
                        da += g * (Sp[(size_t)i * dv + j] - b * kt[i] * u[j]);
                        dki += g * b * (vt[j] - a * u[j]) - a * b * Sp[(size_t)i * dv + j] * r[j];
                    }
                    dk[th * DK + i] = dki;
                }
                dbeta[th] = db;
                dlog_alpha[th] = (a == 0.0) ? 0.0 : a * da;
                for (int i = 0; i < DK; ++i)
                    for (int j = 0; j < dv; ++j)
                        G[(size_t)i * dv + j] = a * (G[(size_t)i * dv + j] - b * kt[i] * r[j]);
            }
            if (dS0) memcpy(dS0 + (size_t)un * state, G, sizeof(double) * state);
            free(St);
        }
        free(kS);
        free(u);
        free(r);
        free(G);
    }
    return bad ? -1 : 0;
}

/*
 * One decode step: every (n, h) state takes exactly one token, in place.
 * Returns 0, or -1 for invalid sizes.
 */
int gdn_oracle_decode_step(const double *q, const double *k, const double *v,
                           const double *log_alpha, const double *beta, double *S_inout,
                           double *out, int N, int H, int dk, int dv, int nthreads)
{
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    set_threads(nthreads);
    const size_t state = (size_t)dk * dv;
    int bad = 0;
#pragma omp parallel
    {
        double *kS = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!kS) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(static)
        for (int u = 0; u < N * H; ++u) {
            if (!kS) continue;
            oracle_token(S_inout + (size_t)u * state, q + (size_t)u * dk, k + (size_t)u * dk,
                         v + (size_t)u * dv, log_alpha[u], beta[u], out + (size_t)u * dv, kS, dk,
                         dv);
        }
        free(kS);
    }
    return bad ? -1 : 0;
}
