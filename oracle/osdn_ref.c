/*
 * osdn_ref.c -- fp64 CPU oracle for the Online Scaled DeltaNet (OSDN) forward pass and, by
 * reverse-mode differentiation of the same token loop, its gradient (osdn_ref_bwd).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct statement of what
 * the GPU library computes.  Only the tests, the smoke check and the benchmark's CPU
 * baseline may load it; the product path never does.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * Source: the technical summary pages of "OSDN: Improving Delta Rule with Provable Online
 * Preconditioning in Linear Attention" (Italian and German editions, same sections):
 *   - section 1 (problem statement): per-token loss f_t(S) = 1/2 ||S k_t - v_t||^2 and
 *     the delta rule S_t = S_{t-1} + beta_t (v_t - S_{t-1} k_t) k_t^T;
 *   - section 2.1 (algebraic equivalence): the right-preconditioned gradient step
 *     S_t = S_{t-1} - beta_t grad f_t(S_{t-1}) D_t equals the delta rule with the write
 *     key replaced by k~_t = d_t (.) k_t;
 *   - section 2.2 (decoupled hypergradient feedback): d_t is updated by online gradient
 *     descent on the surrogate h_t, whose closed form is
 *     h_t(d) = ((1 - beta_t <d, k_t^2>)^2 - 1) / (2 ||k_t||^2); its gradient is
 *     grad_d h_t = -beta_t (1 - beta_t <d, k_t^2>) k_t^2 / ||k_t||^2;
 *   - section 2.3 (APF): a per-token, per-head retention gate r_{t,h} multiplies d only.
 *
 * Readings taken where the pages are silent or garbled (each is pinned by a test):
 *   - The APF equation is printed with "+ eta grad h"; section 2.2 calls the update
 *     gradient DESCENT on h, and only descent lowers h, so the step here is
 *     d_{t+1} = r_t d_t - eta grad_d h_t(d_t).  No projection or clipping is applied.
 *   - Token t writes with d_t, the preconditioner before its own update; d_0 defaults
 *     to the all-ones vector, S_0 to zero.  The output is o_t = scale * S_t q_t, read
 *     from the state after token t's write (DeltaNet convention).
 *   - When ||k_t||^2 == 0 the gradient is taken to be zero.
 *   - With packed variable-length input (cu_seqlens) every sequence starts from its
 *     own d_0 / S_0 and returns its own final state.
 *
 * Layouts (row-major, fp64):
 *   q, k, k_tilde : [B, T, H, Dk]        v, o : [B, T, H, Dv]
 *   beta, r       : [B, T, H]            S0, ST : [N, H, Dv, Dk]   d0, dT : [N, H, Dk]
 *   Fixed length: N = B and sequence n is rows n*T .. n*T+T-1.
 *   Packed: B == 1, T = total tokens, N = num_seqs and sequence n is rows
 *   cu_seqlens[n] .. cu_seqlens[n+1]-1 (cu_seqlens is a HOST array of N+1 entries).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static void seq_bounds(int32_t n, const int32_t* cu_seqlens, int32_t T, int64_t* first,
                       int64_t* count) {
    if (cu_seqlens) {
        *first = cu_seqlens[n];
        *count = (int64_t)cu_seqlens[n + 1] - (int64_t)cu_seqlens[n];
    } else {
        *first = (int64_t)n * T;
        *count = T;
    }
}

int osdn_ref_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ---------------------------------------------------------------------------------
 * Residual contraction (section 3, Theorem 5.2; the experiments' q_geo): the geometric mean
 * of the token-local residual ratios rho_t = f_t(S_t) / f_t(S_{t-1}) of one (sequence, head),
 *   q_geo = (prod_t rho_t)^(1 / T_n) = exp(mean_t log rho_t),
 * given rho [B, T, H]; q_geo [N, H].  A ratio of 0 makes q_geo 0; a sequence with no tokens
 * gets 1 (the empty product).
 * ------------------------------------------------------------------------------- */
void osdn_ref_rho_geomean(const double* rho, double* q_geo, const int32_t* cu_seqlens,
                          int32_t num_seqs, int32_t B, int32_t T, int32_t H) {
    const int32_t N = cu_seqlens ? num_seqs : B;
    for (int32_t n = 0; n < N; ++n) {
        int64_t first, count;
        seq_bounds(n, cu_seqlens, T, &first, &count);
        for (int32_t h = 0; h < H; ++h) {
            double sum_log = 0.0;
            for (int64_t t = 0; t < count; ++t) sum_log += log(rho[(first + t) * H + h]);
            q_geo[(int64_t)n * H + h] = count > 0 ? exp(sum_log / (double)count) : 1.0;
        }
    }
}

/* ---------------------------------------------------------------------------------
 * Phase 1: the preconditioner scan over the key stream (section 2.2, two-phase split,
 * step 1).  Emits k~_t = d_t (.) k_t for every token and the final d.
 * ------------------------------------------------------------------------------- */
void osdn_ref_precond_scan(const double* k, const double* beta, const double* r, double eta,
                           const double* d0, double* k_tilde, double* dT, double* rho,
                           const int32_t* cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                           int32_t H, int32_t Dk) {
    const int32_t N = cu_seqlens ? num_seqs : B;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int32_t n = 0; n < N; ++n) {
        for (int32_t h = 0; h < H; ++h) {
            double* d = (double*)malloc(sizeof(double) * Dk);
            for (int32_t i = 0; i < Dk; ++i) d[i] = d0 ? d0[((int64_t)n * H + h) * Dk + i] : 1.0;
            int64_t first, count;
            seq_bounds(n, cu_seqlens, T, &first, &count);
            for (int64_t t = first; t < first + count; ++t) {
                const int64_t th = t * H + h;
                const double* kt = k + th * Dk;
                const double bt = beta[th];
                const double rt = r ? r[th] : 1.0;
                double knorm2 = 0.0, s = 0.0; /* ||k_t||^2 and <d_t, k_t^2> */
                for (int32_t i = 0; i < Dk; ++i) {
                    knorm2 += kt[i] * kt[i];
                    s += d[i] * kt[i] * kt[i];
                }
                for (int32_t i = 0; i < Dk; ++i) k_tilde[th * Dk + i] = d[i] * kt[i];
                /* residual-contraction ratio of the write (section 3): (1 - beta_t s_t)^2 */
                if (rho) rho[th] = (1.0 - bt * s) * (1.0 - bt * s);
                for (int32_t i = 0; i < Dk; ++i) {
                    const double grad =
                        knorm2 > 0.0 ? -bt * (1.0 - bt * s) * kt[i] * kt[i] / knorm2 : 0.0;
                    d[i] = rt * d[i] - eta * grad;
                }
            }
            if (dT)
                for (int32_t i = 0; i < Dk; ++i) dT[((int64_t)n * H + h) * Dk + i] = d[i];
            free(d);
        }
    }
}

/* ---------------------------------------------------------------------------------
 * Phase 2: the delta rule with a separate write key (section 2.1), token by token:
 *   u_t = v_t - S_{t-1} k_t,   S_t = S_{t-1} + beta_t u_t k~_t^T,   o_t = scale S_t q_t.
 * ------------------------------------------------------------------------------- */
void osdn_ref_delta_fwd(const double* q, const double* k, const double* k_tilde, const double* v,
                        const double* beta, double scale, const double* S0, double* o,
                        double* ST, const int32_t* cu_seqlens, int32_t num_seqs, int32_t B,
                        int32_t T, int32_t H, int32_t Dk, int32_t Dv) {
    const int32_t N = cu_seqlens ? num_seqs : B;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int32_t n = 0; n < N; ++n) {
        for (int32_t h = 0; h < H; ++h) {
            double* S = (double*)malloc(sizeof(double) * Dv * Dk);
            double* u = (double*)malloc(sizeof(double) * Dv);
            const int64_t sbase = ((int64_t)n * H + h) * Dv * Dk;
            for (int64_t e = 0; e < (int64_t)Dv * Dk; ++e) S[e] = S0 ? S0[sbase + e] : 0.0;
            int64_t first, count;
            seq_bounds(n, cu_seqlens, T, &first, &count);
            for (int64_t t = first; t < first + count; ++t) {
                const int64_t th = t * H + h;
                const double* kt = k + th * Dk;
                const double* kw = k_tilde + th * Dk;
                const double* qt = q + th * Dk;
                const double* vt = v + th * Dv;
                const double bt = beta[th];
                for (int32_t j = 0; j < Dv; ++j) {
                    double sk = 0.0;
                    for (int32_t i = 0; i < Dk; ++i) sk += S[(int64_t)j * Dk + i] * kt[i];
                    u[j] = vt[j] - sk;
                }
                for (int32_t j = 0; j < Dv; ++j)
                    for (int32_t i = 0; i < Dk; ++i) S[(int64_t)j * Dk + i] += bt * u[j] * kw[i];
                for (int32_t j = 0; j < Dv; ++j) {
                    double sq = 0.0;
                    for (int32_t i = 0; i < Dk; ++i) sq += S[(int64_t)j * Dk + i] * qt[i];
                    o[th * Dv + j] = scale * sq;
                }
            }
            if (ST)
                for (int64_t e = 0; e < (int64_t)Dv * Dk; ++e) ST[sbase + e] = S[e];
            free(u);
            free(S);
        }
    }
}

/* The token loop of both phases; alpha (NULL: no decay) as in osdn_ref_fwd_gated below. */
static void fwd_impl(const double* q, const double* k, const double* v, const double* beta,
                     const double* r, double eta, const double* d0, const double* S0, double scale,
                     const double* alpha, int32_t alpha_per_channel, double* o, double* k_tilde,
                     double* ST, double* dT, const int32_t* cu_seqlens, int32_t num_seqs, int32_t B,
                     int32_t T, int32_t H, int32_t Dk, int32_t Dv) {
    const int32_t N = cu_seqlens ? num_seqs : B;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int32_t n = 0; n < N; ++n) {
        for (int32_t h = 0; h < H; ++h) {
            double* S = (double*)malloc(sizeof(double) * Dv * Dk);
            double* d = (double*)malloc(sizeof(double) * Dk);
            double* kw = (double*)malloc(sizeof(double) * Dk);
            double* u = (double*)malloc(sizeof(double) * Dv);
            const int64_t sbase = ((int64_t)n * H + h) * Dv * Dk;
            const int64_t dbase = ((int64_t)n * H + h) * Dk;
            for (int64_t e = 0; e < (int64_t)Dv * Dk; ++e) S[e] = S0 ? S0[sbase + e] : 0.0;
            for (int32_t i = 0; i < Dk; ++i) d[i] = d0 ? d0[dbase + i] : 1.0;
            int64_t first, count;
            seq_bounds(n, cu_seqlens, T, &first, &count);
            for (int64_t t = first; t < first + count; ++t) {
                const int64_t th = t * H + h;
                const double* kt = k + th * Dk;
                const double* qt = q + th * Dk;
                const double* vt = v + th * Dv;
                const double bt = beta[th];
                const double rt = r ? r[th] : 1.0;
                if (alpha)  /* the backbone's decay of the key channels, before the write */
                    for (int32_t j = 0; j < Dv; ++j)
                        for (int32_t i = 0; i < Dk; ++i)
                            S[(int64_t)j * Dk + i] *= alpha_per_channel ? alpha[th * Dk + i] : alpha[th];
                double knorm2 = 0.0, s = 0.0;
                for (int32_t i = 0; i < Dk; ++i) {
                    knorm2 += kt[i] * kt[i];
                    s += d[i] * kt[i] * kt[i];
                    kw[i] = d[i] * kt[i];
                }
                if (k_tilde)
                    for (int32_t i = 0; i < Dk; ++i) k_tilde[th * Dk + i] = kw[i];
                for (int32_t j = 0; j < Dv; ++j) {
                    double sk = 0.0;
                    for (int32_t i = 0; i < Dk; ++i) sk += S[(int64_t)j * Dk + i] * kt[i];
                    u[j] = vt[j] - sk;
                }
                for (int32_t j = 0; j < Dv; ++j)
                    for (int32_t i = 0; i < Dk; ++i) S[(int64_t)j * Dk + i] += bt * u[j] * kw[i];
                for (int32_t j = 0; j < Dv; ++j) {
                    double sq = 0.0;
                    for (int32_t i = 0; i < Dk; ++i) sq += S[(int64_t)j * Dk + i] * qt[i];
                    o[th * Dv + j] = scale * sq;
                }
                for (int32_t i = 0; i < Dk; ++i) {
                    const double grad =
                        knorm2 > 0.0 ? -bt * (1.0 - bt * s) * kt[i] * kt[i] / knorm2 : 0.0;
                    d[i] = rt * d[i] - eta * grad;
                }
            }
            if (ST)
                for (int64_t e = 0; e < (int64_t)Dv * Dk; ++e) ST[sbase + e] = S[e];
            if (dT)
                for (int32_t i = 0; i < Dk; ++i) dT[dbase + i] = d[i];
            free(u);
            free(kw);
            free(d);
            free(S);
        }
    }
}

/* ---------------------------------------------------------------------------------
 * Both phases in one token loop: the method exactly as stated, with no split.
 * Per token: k~ = d (.) k;  u = v - S k;  S += beta u k~^T;  o = scale S q;
 *            d <- r d - eta grad_d h(d).
 * k_tilde and dT may be NULL.
 * ------------------------------------------------------------------------------- */
void osdn_ref_fwd(const double* q, const double* k, const double* v, const double* beta,
                  const double* r, double eta, const double* d0, const double* S0, double scale,
                  double* o, double* k_tilde, double* ST, double* dT, const int32_t* cu_seqlens,
                  int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv) {
    fwd_impl(q, k, v, beta, r, eta, d0, S0, scale, NULL, 0, o, k_tilde, ST, dT, cu_seqlens, num_seqs,
             B, T, H, Dk, Dv);
}

/* ---------------------------------------------------------------------------------
 * Both phases on a gated backbone (OSDN on Gated DeltaNet or Kimi Delta Attention).
 * The pages train OSDN on GDN and KDA backbones without printing the combined update; the
 * Gated DeltaNet-2 page (section 1) gives the gated delta rule, key-major,
 * S_t = (I - beta k k^T) D_t S_{t-1} + beta k v^T with D_t = Diag(alpha_t) for KDA and
 * alpha_t I for GDN.  Reading taken here: the state decays first, then OSDN's write key
 * replaces the written key,
 *   Sbar = S_{t-1} Diag(alpha_t)  (value-major S: the key channels decay),
 *   S_t = Sbar + beta (v - Sbar k) k~^T,   k~ = d (.) k,
 * and the preconditioner recurrence is unchanged (its surrogate is f_t around Sbar, the same
 * function of k, beta and d).  alpha is [B,T,H] (GDN) when alpha_per_channel == 0, or
 * [B,T,H,Dk] (KDA) when it is 1; all other arguments as osdn_ref_fwd.
 * ------------------------------------------------------------------------------- */
void osdn_ref_fwd_gated(const double* q, const double* k, const double* v, const double* beta,
                        const double* r, double eta, const double* d0, const double* S0,
                        double scale, const double* alpha, int32_t alpha_per_channel, double* o,
                        double* k_tilde, double* ST, double* dT, const int32_t* cu_seqlens,
                        int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t Dk,
                        int32_t Dv) {
    fwd_impl(q, k, v, beta, r, eta, d0, S0, scale, alpha, alpha_per_channel, o, k_tilde, ST, dT,
             cu_seqlens, num_seqs, B, T, H, Dk, Dv);
}

/* ---------------------------------------------------------------------------------
 * Gradient of the forward pass: reverse-mode differentiation of the token loop of
 * osdn_ref_fwd, step by step in reverse order (the pages give no backward pass; this is
 * the chain rule applied to the forward steps above, nothing else).  For
 *   L = <dO, o> + <dST, S_T> + <ddT, d_T>
 * it returns dL/dq, dL/dk, dL/dv, dL/dbeta, dL/dr (when r is non-NULL), dL/deta (one
 * scalar over the whole batch), dL/dS0 and dL/dd0.  dST and ddT may be NULL (zero).
 * Every token's state is kept for the reverse sweep, so this is for small problems.
 * Per token, with S, d the state before the token and a = k (.) k, n = ||k||^2:
 *   s = <d, a>, w = d (.) k, u = v - S k, S' = S + beta u w^T, o = scale S' q,
 *   g = eta beta (1 - beta s) / n (0 when n == 0), d' = r d + g a.
 * ------------------------------------------------------------------------------- */
/* The reverse sweep of osdn_ref_bwd; with alpha (NULL: no decay) it differentiates the gated
 * loop of osdn_ref_fwd_gated and writes dL/dalpha into dalpha. */
static void bwd_impl(const double* q, const double* k, const double* v, const double* beta,
                     const double* r, double eta, const double* d0, const double* S0, double scale,
                     const double* alpha, int32_t apc, const double* dO, const double* dST,
                     const double* ddT, double* dq, double* dk, double* dv, double* dbeta,
                     double* dr, double* deta, double* dalpha, double* dS0, double* dd0,
                     const int32_t* cu_seqlens, int32_t num_seqs, int32_t B, int32_t T, int32_t H,
                     int32_t Dk, int32_t Dv) {
    const int32_t N = cu_seqlens ? num_seqs : B;
    const int64_t SZ = (int64_t)Dv * Dk;
    double eta_total = 0.0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(+ : eta_total)
    for (int32_t n = 0; n < N; ++n) {
        for (int32_t h = 0; h < H; ++h) {
            int64_t first, count;
            seq_bounds(n, cu_seqlens, T, &first, &count);
            const int64_t sbase = ((int64_t)n * H + h) * SZ;
            const int64_t dbase = ((int64_t)n * H + h) * Dk;
            /* states before each token: Sall[c], dall[c]; after the last token: index count */
            double* Sall = (double*)malloc(sizeof(double) * (count + 1) * SZ);
            double* dall = (double*)malloc(sizeof(double) * (count + 1) * Dk);
            double* w = (double*)malloc(sizeof(double) * Dk);
            double* u = (double*)malloc(sizeof(double) * Dv);
            double* gS = (double*)malloc(sizeof(double) * SZ);
            double* gd = (double*)malloc(sizeof(double) * Dk);
            double* gdp = (double*)malloc(sizeof(double) * Dk);
            double* ga = (double*)malloc(sizeof(double) * Dk);
            double* gk = (double*)malloc(sizeof(double) * Dk);
            double* gw = (double*)malloc(sizeof(double) * Dk);
            double* gu = (double*)malloc(sizeof(double) * Dv);
            double* Sb = (double*)malloc(sizeof(double) * SZ);  /* the decayed state S Diag(alpha) */
            for (int64_t e = 0; e < SZ; ++e) Sall[e] = S0 ? S0[sbase + e] : 0.0;
            for (int32_t i = 0; i < Dk; ++i) dall[i] = d0 ? d0[dbase + i] : 1.0;
            /* forward sweep (the same steps as osdn_ref_fwd) */
            for (int64_t c = 0; c < count; ++c) {
                const int64_t th = (first + c) * H + h;
                const double* kt = k + th * Dk;
                const double* vt = v + th * Dv;
                const double bt = beta[th], rt = r ? r[th] : 1.0;
                const double* Sp = Sall + c * SZ;  /* before the token */
                const double* S = Sp;                /* after the decay: the state the write sees */
                if (alpha) {
                    for (int32_t j = 0; j < Dv; ++j)
                        for (int32_t i = 0; i < Dk; ++i)
                            Sb[(int64_t)j * Dk + i] =
                                Sp[(int64_t)j * Dk + i] * (apc ? alpha[th * Dk + i] : alpha[th]);
                    S = Sb;
                }
                const double* d = dall + c * Dk;
                double* Sn = Sall + (c + 1) * SZ;
                double* dn = dall + (c + 1) * Dk;
                double knorm2 = 0.0, s = 0.0;
                for (int32_t i = 0; i < Dk; ++i) {
                    knorm2 += kt[i] * kt[i];
                    s += d[i] * kt[i] * kt[i];
                    w[i] = d[i] * kt[i];
                }
                for (int32_t j = 0; j < Dv; ++j) {
                    double sk = 0.0;
                    for (int32_t i = 0; i < Dk; ++i) sk += S[(int64_t)j * Dk + i] * kt[i];
                    u[j] = vt[j] - sk;
                }
                for (int32_t j = 0; j < Dv; ++j)
                    for (int32_t i = 0; i < Dk; ++i)
                        Sn[(int64_t)j * Dk + i] = S[(int64_t)j * Dk + i] + bt * u[j] * w[i];
                const double g = knorm2 > 0.0 ? eta * bt * (1.0 - bt * s) / knorm2 : 0.0;
                for (int32_t i = 0; i < Dk; ++i) dn[i] = rt * d[i] + g * kt[i] * kt[i];
            }
            /* reverse sweep: gS, gd are the adjoints of the state after token c */
            for (int64_t e = 0; e < SZ; ++e) gS[e] = dST ? dST[sbase + e] : 0.0;
            for (int32_t i = 0; i < Dk; ++i) gd[i] = ddT ? ddT[dbase + i] : 0.0;
            for (int64_t c = count - 1; c >= 0; --c) {
                const int64_t th = (first + c) * H + h;
                const double* kt = k + th * Dk;
                const double* qt = q + th * Dk;
                const double* vt = v + th * Dv;
                const double* gOt = dO + th * Dv;
                const double bt = beta[th], rt = r ? r[th] : 1.0;
                const double* Sp = Sall + c * SZ;  /* before the token */
                const double* S = Sp;                /* after the decay: the state the write sees */
                if (alpha) {
                    for (int32_t j = 0; j < Dv; ++j)
                        for (int32_t i = 0; i < Dk; ++i)
                            Sb[(int64_t)j * Dk + i] =
                                Sp[(int64_t)j * Dk + i] * (apc ? alpha[th * Dk + i] : alpha[th]);
                    S = Sb;
                }
                const double* d = dall + c * Dk;
                const double* Sn = Sall + (c + 1) * SZ;
                double knorm2 = 0.0, s = 0.0;
                for (int32_t i = 0; i < Dk; ++i) {
                    knorm2 += kt[i] * kt[i];
                    s += d[i] * kt[i] * kt[i];
                    w[i] = d[i] * kt[i];
                }
                for (int32_t j = 0; j < Dv; ++j) {
                    double sk = 0.0;
                    for (int32_t i = 0; i < Dk; ++i) sk += S[(int64_t)j * Dk + i] * kt[i];
                    u[j] = vt[j] - sk;
                }
                const double g = knorm2 > 0.0 ? eta * bt * (1.0 - bt * s) / knorm2 : 0.0;
                double gbeta = 0.0;
                /* o = scale S' q */
                for (int32_t i = 0; i < Dk; ++i) {
                    double acc = 0.0;
                    for (int32_t j = 0; j < Dv; ++j) acc += Sn[(int64_t)j * Dk + i] * gOt[j];
                    dq[th * Dk + i] = scale * acc;
                }
                for (int32_t j = 0; j < Dv; ++j)
                    for (int32_t i = 0; i < Dk; ++i) gS[(int64_t)j * Dk + i] += scale * gOt[j] * qt[i];
                /* d' = r d + g a */
                double gr = 0.0, gg = 0.0;
                for (int32_t i = 0; i < Dk; ++i) {
                    gr += gd[i] * d[i];
                    gg += gd[i] * kt[i] * kt[i];
                    ga[i] = g * gd[i];
                    gdp[i] = rt * gd[i];
                }
                if (dr) dr[th] = gr;
                if (knorm2 > 0.0) {  /* g = eta beta (1 - beta s) / n */
                    eta_total += gg * bt * (1.0 - bt * s) / knorm2;
                    gbeta += gg * eta * (1.0 - 2.0 * bt * s) / knorm2;
                    const double gs = gg * (-eta * bt * bt / knorm2);
                    const double gn = gg * (-g / knorm2);
                    for (int32_t i = 0; i < Dk; ++i) {
                        gdp[i] += gs * kt[i] * kt[i];  /* s = <d, a> */
                        ga[i] += gs * d[i] + gn;       /* s and n = sum of a */
                    }
                }
                /* S' = S + beta u w^T */
                for (int32_t j = 0; j < Dv; ++j) {
                    double acc = 0.0;
                    for (int32_t i = 0; i < Dk; ++i) {
                        gbeta += gS[(int64_t)j * Dk + i] * u[j] * w[i];
                        acc += gS[(int64_t)j * Dk + i] * w[i];
                    }
                    gu[j] = bt * acc;
                }
                for (int32_t i = 0; i < Dk; ++i) {
                    double acc = 0.0;
                    for (int32_t j = 0; j < Dv; ++j) acc += gS[(int64_t)j * Dk + i] * u[j];
                    gw[i] = bt * acc;
                }
                /* u = v - S k */
                for (int32_t j = 0; j < Dv; ++j) dv[th * Dv + j] = gu[j];
                for (int32_t i = 0; i < Dk; ++i) {
                    double acc = 0.0;
                    for (int32_t j = 0; j < Dv; ++j) acc += gu[j] * S[(int64_t)j * Dk + i];
                    gk[i] = -acc;
                }
                for (int32_t j = 0; j < Dv; ++j)
                    for (int32_t i = 0; i < Dk; ++i) gS[(int64_t)j * Dk + i] -= gu[j] * kt[i];
                /* w = d (.) k and a = k (.) k */
                for (int32_t i = 0; i < Dk; ++i) {
                    gdp[i] += gw[i] * kt[i];
                    gk[i] += gw[i] * d[i] + 2.0 * kt[i] * ga[i];
                    dk[th * Dk + i] = gk[i];
                    gd[i] = gdp[i];
                }
                dbeta[th] = gbeta;
                if (alpha) {  /* S = Sp Diag(alpha): dalpha from Sp, then the adjoint of Sp */
                    if (apc) {
                        for (int32_t i = 0; i < Dk; ++i) {
                            double acc = 0.0;
                            for (int32_t j = 0; j < Dv; ++j)
                                acc += gS[(int64_t)j * Dk + i] * Sp[(int64_t)j * Dk + i];
                            dalpha[th * Dk + i] = acc;
                        }
                        for (int32_t j = 0; j < Dv; ++j)
                            for (int32_t i = 0; i < Dk; ++i) gS[(int64_t)j * Dk + i] *= alpha[th * Dk + i];
                    } else {
                        double acc = 0.0;
                        for (int64_t e = 0; e < SZ; ++e) acc += gS[e] * Sp[e];
                        dalpha[th] = acc;
                        for (int64_t e = 0; e < SZ; ++e) gS[e] *= alpha[th];
                    }
                }
            }
            for (int64_t e = 0; e < SZ; ++e) dS0[sbase + e] = gS[e];
            for (int32_t i = 0; i < Dk; ++i) dd0[dbase + i] = gd[i];
            free(Sb);
            free(gu);
            free(gw);
            free(gk);
            free(ga);
            free(gdp);
            free(gd);
            free(gS);
            free(u);
            free(w);
            free(dall);
            free(Sall);
        }
    }
    if (deta) *deta = eta_total;
}

void osdn_ref_bwd(const double* q, const double* k, const double* v, const double* beta,
                  const double* r, double eta, const double* d0, const double* S0, double scale,
                  const double* dO, const double* dST, const double* ddT, double* dq, double* dk,
                  double* dv, double* dbeta, double* dr, double* deta, double* dS0, double* dd0,
                  const int32_t* cu_seqlens, int32_t num_seqs, int32_t B, int32_t T, int32_t H,
                  int32_t Dk, int32_t Dv) {
    bwd_impl(q, k, v, beta, r, eta, d0, S0, scale, NULL, 0, dO, dST, ddT, dq, dk, dv, dbeta, dr,
             deta, NULL, dS0, dd0, cu_seqlens, num_seqs, B, T, H, Dk, Dv);
}

/* The gradient of osdn_ref_fwd_gated (same arguments as osdn_ref_bwd plus alpha as in
 * osdn_ref_fwd_gated); dalpha has alpha's shape. */
void osdn_ref_bwd_gated(const double* q, const double* k, const double* v, const double* beta,
                        const double* r, double eta, const double* d0, const double* S0,
                        double scale, const double* alpha, int32_t alpha_per_channel,
                        const double* dO, const double* dST, const double* ddT, double* dq,
                        double* dk, double* dv, double* dbeta, double* dr, double* deta,
                        double* dalpha, double* dS0, double* dd0, const int32_t* cu_seqlens,
                        int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t Dk,
                        int32_t Dv) {
    bwd_impl(q, k, v, beta, r, eta, d0, S0, scale, alpha, alpha_per_channel, dO, dST, ddT, dq, dk,
             dv, dbeta, dr, deta, dalpha, dS0, dd0, cu_seqlens, num_seqs, B, T, H, Dk, Dv);
}
