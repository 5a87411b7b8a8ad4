/*
 * Float64 CPU oracle for the selective diagonal state-space scan and its exact gradient.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the package's smoke check and the bench's CPU-baseline
 * leg may load this file's library.  It shares no code, header, table or helper with the CUDA
 * path: it is the plain definition, written as a sequential loop over time per independent
 * channel, plus the hand-derived reverse-time adjoint.  No blocking, fusion or reordering of the
 * arithmetic beyond "channels are independent" (OpenMP runs whole channels on separate threads;
 * the cross-channel sums dB, dC, dr, dphi are added per thread, then thread by thread in index
 * order, so a fixed thread count gives a bitwise-fixed result).  Build without -ffast-math.
 *
 * Real mode.  The selective SSM of "选择性状态空间模型(S3M)原理与工程实践" §1.1 (step size
 * delta = softplus(projection), decay A = -exp(log_A), transition exp(A·delta)), with the Euler
 * input term delta·B_t·x_t:
 *     delta_t = softplus(delta_raw_t),  A_n = -exp(A_log_n),  a_{t,n} = exp(delta_t A_n)
 *     h_{t,n} = a_{t,n} h_{t-1,n} + delta_t Bm_{t,n} x_t,   h_{-1} = 0
 *     y_t     = sum_n Cm_{t,n} h_{t,n} + Dskip x_t
 * The gradient is the exact reverse-time adjoint of "Breaking the Memory Wall: Exact Analytical
 * Differentiation via Tiled Operator-Space Evolution" (abstract: exact analytical derivatives in
 * the state space, no stored graph), derived by hand for the loss L = sum dy·y:
 *     g_t    = Cm_t dy_t + a_{t+1} g_{t+1},  g_{L-1} = Cm_{L-1} dy_{L-1}     (g_t = dL/dh_t)
 *     q_t    = g_t a_t h_{t-1}                                               (dL/d log a_t)
 *     dx_t   = Dskip dy_t + delta_t sum_n g_t Bm_t
 *     ddelta = sum_n A_n q_t + x_t sum_n g_t Bm_t;   ddelta_raw = ddelta · sigmoid(delta_raw)
 *     dBm_t  = sum_d g_t delta_t x_t;   dCm_t = sum_d dy_t h_t
 *     dA_log = A_n sum_{b,t} delta_t q_t;   dDskip = sum_{b,t} dy_t x_t
 *
 * Options of the real mode (ssm_oracle_real_ex):
 *   - initial state h_{-1} = h0 [B,D,N] instead of zero, and the final state hL = h_{L-1} out;
 *     with an upstream gradient dhL of the final state the loss becomes L = sum dy·y + sum dhL·hL,
 *     so g_{L-1} = Cm dy + dhL, and dh0 = dL/dh0 = a_0 g_0 is returned (h_{-1} = h0 enters q_0);
 *   - zero-order-hold input term, the blog's §1.1 discretisation B̄ = (delta A)^{-1}(exp(delta A) - 1)
 *     delta B, which for a diagonal A is phi_{t,n} Bm_{t,n} x_t with phi = expm1(delta A) / A.
 *     Then dphi/ddelta = a and dphi/dA = (delta a - phi) / A, so
 *       dx_t = Dskip dy_t + sum_n g phi Bm;   ddelta = sum_n A q + x_t sum_n g a Bm;
 *       dBm_t = sum_d g phi x;   dA_n gets, beside delta q, g Bm x (delta a - phi) / A.
 *
 * Complex mode.  "SPARC: Shared Phase and Retention Control for Efficient Adaptive Spectral
 * Recurrence" (abstract: two input-dependent scalars, retention r_t and phase phi_t, drive all
 * complex modes, each with its own timescale lambda_k and frequency omega_k; diagonal affine
 * recurrence):
 *     s_t = softplus(r_t),  a_{t,k} = exp(-lambda_k s_t + i omega_k phi_t),  h_t = a_t h_{t-1} + u_t
 * Loss L = Re sum conj(g) h; complex gradients use d/dRe + i d/dIm (PyTorch's .grad convention):
 *     mu_t = g_t + conj(a_{t+1}) mu_{t+1};  du_t = mu_t;  q_t = mu_t conj(a_t h_{t-1})
 *     dlambda_k = -sum s_t Re q;  dr_t = sigmoid(r_t) (-sum_k lambda_k Re q)
 *     domega_k  =  sum phi_t Im q;  dphi_t = sum_k omega_k Im q
 */
#include <complex.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double softplus(double z) { return z > 0.0 ? z + log1p(exp(-z)) : log1p(exp(z)); }

static double sigmoid(double z) {
    if (z >= 0.0) return 1.0 / (1.0 + exp(-z));
    double e = exp(z);
    return e / (1.0 + e);
}

int ssm_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int pick_threads(int nthreads) {
    int m = ssm_oracle_max_threads();
    if (nthreads <= 0 || nthreads > m) nthreads = m;
    return nthreads;
}

/*
 * Real mode, channels d in [d_lo, d_hi).  Inputs (row-major, float64):
 *   x, draw, dy [B,L,D]; Bm, Cm [B,L,N]; A_log [D,N]; Dskip [D].  dy may be NULL (forward only).
 * Outputs (NULL to skip): y [B,L,D] and, when dy is given, dx, ddraw [B,L,D] — only entries with
 * d in range are written; ckpt [B, ceil(L/T), D, N] holds h at the last step of every chunk of T
 * steps; dA_log [D,N] and dD [D] rows in range (summed over all b); dB, dC [B,L,N] are fully
 * overwritten with the sums over the channels in range.
 * Returns 0, or -1 on a bad argument / allocation failure.
 */
/*
 * As above, with the options: zoh != 0 selects the zero-order-hold input term; h0 [B,D,N] (NULL:
 * zero) is the initial state; hL [B,D,N] (NULL: skip) receives the final state; dhL [B,D,N] (NULL:
 * zero) is the upstream gradient of the final state; dh0 [B,D,N] (NULL: skip) receives the gradient
 * with respect to h0 (both only for d in range).
 */
int ssm_oracle_real_ex(int64_t B, int64_t L, int64_t D, int64_t N, int64_t T,
                       const double* x, const double* draw, const double* A_log, const double* Bm,
                       const double* Cm, const double* Dskip, const double* dy,
                       int64_t d_lo, int64_t d_hi, int nthreads, int zoh,
                       const double* h0, const double* dhL,
                       double* y, double* ckpt, double* dx, double* ddraw,
                       double* dA_log, double* dB, double* dC, double* dD,
                       double* hL, double* dh0) {
    if (B < 0 || L < 0 || D <= 0 || N <= 0 || T <= 0 || d_lo < 0 || d_hi > D || d_lo > d_hi)
        return -1;
    const int64_t nC = (L + T - 1) / T;
    const int bwd = dy != NULL;
    nthreads = pick_threads(nthreads);
    const size_t bln = (size_t)B * (size_t)L * (size_t)N;
    double** part_dB = NULL;
    double** part_dC = NULL;
    int fail = 0;
    if (bwd) {
        part_dB = (double**)calloc((size_t)nthreads, sizeof(double*));
        part_dC = (double**)calloc((size_t)nthreads, sizeof(double*));
        if (!part_dB || !part_dC) { free(part_dB); free(part_dC); return -1; }
    }

#pragma omp parallel num_threads(nthreads)
    {
        int tid = 0;
#ifdef _OPENMP
        tid = omp_get_thread_num();
#endif
        double* hh = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * (size_t)N);
        double* aa = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * (size_t)N);
        double* A = (double*)malloc(sizeof(double) * (size_t)N);
        double* h = (double*)malloc(sizeof(double) * (size_t)N);
        double* v = (double*)malloc(sizeof(double) * (size_t)N);
        double* dAsum = (double*)malloc(sizeof(double) * (size_t)N);
        double* myB = NULL;
        double* myC = NULL;
        if (bwd) {
            myB = (double*)calloc(bln > 0 ? bln : 1, sizeof(double));
            myC = (double*)calloc(bln > 0 ? bln : 1, sizeof(double));
            part_dB[tid] = myB;
            part_dC[tid] = myC;
        }
        if (!hh || !aa || !A || !h || !v || !dAsum || (bwd && (!myB || !myC))) {
#pragma omp atomic write
            fail = 1;
        }
#pragma omp barrier
        if (!fail) {
#pragma omp for schedule(static)
            for (int64_t d = d_lo; d < d_hi; ++d) {
                for (int64_t n = 0; n < N; ++n) {
                    A[n] = -exp(A_log[d * N + n]);
                    dAsum[n] = 0.0;
                }
                double dDsum = 0.0;
                for (int64_t b = 0; b < B; ++b) {
                    /* forward: sequential recurrence, full history of a and h kept */
                    const int64_t s0 = (b * D + d) * N;  /* offset of this row in h0/hL/dhL/dh0 */
                    for (int64_t n = 0; n < N; ++n) h[n] = h0 ? h0[s0 + n] : 0.0;
                    for (int64_t t = 0; t < L; ++t) {
                        const int64_t i = (b * L + t) * D + d;
                        const double* Bt = Bm + (b * L + t) * N;
                        const double* Ct = Cm + (b * L + t) * N;
                        const double delta = softplus(draw[i]);
                        double acc = 0.0;
                        for (int64_t n = 0; n < N; ++n) {
                            const double a = exp(delta * A[n]);
                            const double w = zoh ? expm1(delta * A[n]) / A[n] : delta;
                            h[n] = a * h[n] + w * Bt[n] * x[i];
                            aa[t * N + n] = a;
                            hh[t * N + n] = h[n];
                            acc += Ct[n] * h[n];
                        }
                        if (y) y[i] = acc + Dskip[d] * x[i];
                        if (ckpt && (t == L - 1 || (t + 1) % T == 0)) {
                            double* ck = ckpt + ((b * nC + t / T) * D + d) * N;
                            for (int64_t n = 0; n < N; ++n) ck[n] = h[n];
                        }
                    }
                    if (hL)
                        for (int64_t n = 0; n < N; ++n) hL[s0 + n] = h[n];
                    if (!bwd) continue;
                    /* backward: reverse-time adjoint; v = a_{t+1} g_{t+1}, dhL beyond the end */
                    for (int64_t n = 0; n < N; ++n) v[n] = dhL ? dhL[s0 + n] : 0.0;
                    for (int64_t t = L - 1; t >= 0; --t) {
                        const int64_t i = (b * L + t) * D + d;
                        const double* Bt = Bm + (b * L + t) * N;
                        const double* Ct = Cm + (b * L + t) * N;
                        const double delta = softplus(draw[i]);
                        /* sum_gwB: sum_n g w Bm (w = delta, or phi for zoh); sum_gdB: sum_n g
                         * (dw/ddelta) Bm (dw/ddelta = 1, or a for zoh) */
                        double sum_gwB = 0.0, sum_gdB = 0.0, sum_Aq = 0.0;
                        for (int64_t n = 0; n < N; ++n) {
                            const double a = aa[t * N + n];
                            const double hprev =
                                t > 0 ? hh[(t - 1) * N + n] : (h0 ? h0[s0 + n] : 0.0);
                            const double g = Ct[n] * dy[i] + v[n];
                            const double q = g * a * hprev;
                            const double w = zoh ? expm1(delta * A[n]) / A[n] : delta;
                            const double dw_ddelta = zoh ? a : 1.0;
                            sum_Aq += A[n] * q;
                            sum_gwB += g * w * Bt[n];
                            sum_gdB += g * dw_ddelta * Bt[n];
                            dAsum[n] += delta * q;
                            if (zoh) dAsum[n] += g * Bt[n] * x[i] * (delta * a - w) / A[n];
                            myB[(b * L + t) * N + n] += g * w * x[i];
                            myC[(b * L + t) * N + n] += dy[i] * hh[t * N + n];
                            v[n] = a * g;
                        }
                        if (dx) dx[i] = Dskip[d] * dy[i] + sum_gwB;
                        if (ddraw) ddraw[i] = (sum_Aq + x[i] * sum_gdB) * sigmoid(draw[i]);
                        dDsum += dy[i] * x[i];
                    }
                    if (dh0)
                        for (int64_t n = 0; n < N; ++n) dh0[s0 + n] = v[n];
                }
                if (bwd) {
                    if (dA_log)
                        for (int64_t n = 0; n < N; ++n) dA_log[d * N + n] = A[n] * dAsum[n];
                    if (dD) dD[d] = dDsum;
                }
            }
        }
        free(hh); free(aa); free(A); free(h); free(v); free(dAsum);
    }

    if (bwd) {
        if (!fail) {
            if (dB) memset(dB, 0, sizeof(double) * bln);
            if (dC) memset(dC, 0, sizeof(double) * bln);
            for (int tt = 0; tt < nthreads; ++tt) {
                for (size_t j = 0; j < bln; ++j) {
                    if (dB) dB[j] += part_dB[tt][j];
                    if (dC) dC[j] += part_dC[tt][j];
                }
            }
        }
        for (int tt = 0; tt < nthreads; ++tt) { free(part_dB[tt]); free(part_dC[tt]); }
        free(part_dB);
        free(part_dC);
    }
    return fail ? -1 : 0;
}

int ssm_oracle_real(int64_t B, int64_t L, int64_t D, int64_t N, int64_t T,
                    const double* x, const double* draw, const double* A_log, const double* Bm,
                    const double* Cm, const double* Dskip, const double* dy,
                    int64_t d_lo, int64_t d_hi, int nthreads,
                    double* y, double* ckpt, double* dx, double* ddraw,
                    double* dA_log, double* dB, double* dC, double* dD) {
    return ssm_oracle_real_ex(B, L, D, N, T, x, draw, A_log, Bm, Cm, Dskip, dy, d_lo, d_hi,
                              nthreads, 0, NULL, NULL, y, ckpt, dx, ddraw, dA_log, dB, dC, dD,
                              NULL, NULL);
}

/*
 * Complex mode, modes k in [k_lo, k_hi).  u, g, h, du are [B,L,K] complex (interleaved re, im
 * doubles); r, phi [B,L]; lambda, omega [K].  g may be NULL (forward only).  h, du entries with k
 * in range are written; dlambda, domega entries in range; dr, dphi [B,L] are fully overwritten
 * with the sums over the modes in range.  Returns 0 or -1.
 */
int ssm_oracle_complex(int64_t B, int64_t L, int64_t K,
                       const double* u_, const double* r, const double* phi,
                       const double* lambda, const double* omega, const double* g_,
                       int64_t k_lo, int64_t k_hi, int nthreads,
                       double* h_, double* du_, double* dr, double* dphi,
                       double* dlambda, double* domega) {
    if (B < 0 || L < 0 || K <= 0 || k_lo < 0 || k_hi > K || k_lo > k_hi) return -1;
    const double complex* u = (const double complex*)u_;
    const double complex* g = (const double complex*)g_;
    double complex* hout = (double complex*)h_;
    double complex* du = (double complex*)du_;
    const int bwd = g != NULL;
    nthreads = pick_threads(nthreads);
    const size_t bl = (size_t)B * (size_t)L;
    double** part_r = NULL;
    double** part_p = NULL;
    int fail = 0;
    if (bwd) {
        part_r = (double**)calloc((size_t)nthreads, sizeof(double*));
        part_p = (double**)calloc((size_t)nthreads, sizeof(double*));
        if (!part_r || !part_p) { free(part_r); free(part_p); return -1; }
    }

#pragma omp parallel num_threads(nthreads)
    {
        int tid = 0;
#ifdef _OPENMP
        tid = omp_get_thread_num();
#endif
        const size_t Lp = (size_t)(L > 0 ? L : 1);
        double complex* hh = (double complex*)malloc(sizeof(double complex) * Lp);
        double complex* aa = (double complex*)malloc(sizeof(double complex) * Lp);
        double* myr = NULL;
        double* myp = NULL;
        if (bwd) {
            myr = (double*)calloc(bl > 0 ? bl : 1, sizeof(double));
            myp = (double*)calloc(bl > 0 ? bl : 1, sizeof(double));
            part_r[tid] = myr;
            part_p[tid] = myp;
        }
        if (!hh || !aa || (bwd && (!myr || !myp))) {
#pragma omp atomic write
            fail = 1;
        }
#pragma omp barrier
        if (!fail) {
#pragma omp for schedule(static)
            for (int64_t k = k_lo; k < k_hi; ++k) {
                const double lam = lambda[k], om = omega[k];
                double dlam = 0.0, dom = 0.0;
                for (int64_t b = 0; b < B; ++b) {
                    double complex h = 0.0;
                    for (int64_t t = 0; t < L; ++t) {
                        const int64_t j = b * L + t;
                        const double s = softplus(r[j]);
                        const double complex a = cexp(-lam * s + I * (om * phi[j]));
                        h = a * h + u[j * K + k];
                        aa[t] = a;
                        hh[t] = h;
                        if (hout) hout[j * K + k] = h;
                    }
                    if (!bwd) continue;
                    double complex mu_next = 0.0; /* conj(a_{t+1}) mu_{t+1} */
                    for (int64_t t = L - 1; t >= 0; --t) {
                        const int64_t j = b * L + t;
                        const double s = softplus(r[j]);
                        const double complex mu = g[j * K + k] + mu_next;
                        const double complex hprev = t > 0 ? hh[t - 1] : 0.0;
                        const double complex q = mu * conj(aa[t] * hprev);
                        if (du) du[j * K + k] = mu;
                        dlam += -s * creal(q);
                        dom += phi[j] * cimag(q);
                        myr[j] += -lam * creal(q);
                        myp[j] += om * cimag(q);
                        mu_next = conj(aa[t]) * mu;
                    }
                }
                if (bwd) {
                    if (dlambda) dlambda[k] = dlam;
                    if (domega) domega[k] = dom;
                }
            }
        }
        free(hh); free(aa);
    }

    if (bwd) {
        if (!fail) {
            if (dr) memset(dr, 0, sizeof(double) * bl);
            if (dphi) memset(dphi, 0, sizeof(double) * bl);
            for (int tt = 0; tt < nthreads; ++tt) {
                for (size_t j = 0; j < bl; ++j) {
                    if (dr) dr[j] += part_r[tt][j];
                    if (dphi) dphi[j] += part_p[tt][j];
                }
            }
            if (dr)
                for (size_t j = 0; j < bl; ++j) dr[j] *= sigmoid(r[j]);
        }
        for (int tt = 0; tt < nthreads; ++tt) { free(part_r[tt]); free(part_p[tt]); }
        free(part_r);
        free(part_p);
    }
    return fail ? -1 : 0;
}

/*
 * Complex mode, exact structured real-time recurrent learning (SPARC abstract: the diagonal
 * recurrence admits exact structured RTRL for online credit assignment).  Forward-mode
 * sensitivities of the state to each mode's own parameters are carried with the state:
 *     S^lambda_t = dh_t/dlambda = a_t S^lambda_{t-1} + (da_t/dlambda) h_{t-1},  da/dlambda = -s_t a_t
 *     S^omega_t  = dh_t/domega  = a_t S^omega_{t-1}  + (da_t/domega)  h_{t-1},  da/domega  = i phi_t a_t
 * and the gradient of the online loss L = Re sum_t conj(g_t) h_t accumulates as the steps arrive:
 *     dL/dlambda += Re(conj(g_t) S^lambda_t),   dL/domega += Re(conj(g_t) S^omega_t).
 * No reverse pass and nothing of the trajectory is kept: the result equals the reverse-time
 * adjoint's dlambda, domega (the same numbers by a different method).
 * state [B,3,K] complex (h, S^lambda, S^omega) may be NULL (start from zero, final values not
 * returned); when given it is read as the state before t = 0 and overwritten with the state after
 * t = L-1, so consecutive calls continue one sequence.  h (optional) receives the trajectory.
 * dlambda, domega [K] receive this call's sums over b and t.  Returns 0 or -1.
 */
int ssm_oracle_complex_rtrl(int64_t B, int64_t L, int64_t K,
                            const double* u_, const double* r, const double* phi,
                            const double* lambda, const double* omega, const double* g_,
                            int nthreads, double* h_, double* state_,
                            double* dlambda, double* domega) {
    if (B < 0 || L < 0 || K <= 0 || !g_ || !dlambda || !domega) return -1;
    const double complex* u = (const double complex*)u_;
    const double complex* g = (const double complex*)g_;
    double complex* hout = (double complex*)h_;
    double complex* state = (double complex*)state_;
    nthreads = pick_threads(nthreads);
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t k = 0; k < K; ++k) {
        const double lam = lambda[k], om = omega[k];
        double dlam = 0.0, dom = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            double complex h = 0.0, Sl = 0.0, So = 0.0;
            if (state) {
                h = state[(b * 3 + 0) * K + k];
                Sl = state[(b * 3 + 1) * K + k];
                So = state[(b * 3 + 2) * K + k];
            }
            for (int64_t t = 0; t < L; ++t) {
                const int64_t j = b * L + t;
                const double s = softplus(r[j]);
                const double complex a = cexp(-lam * s + I * (om * phi[j]));
                Sl = a * Sl + (-s * a) * h;          /* uses h_{t-1} */
                So = a * So + (I * phi[j] * a) * h;
                h = a * h + u[j * K + k];
                if (hout) hout[j * K + k] = h;
                const double complex gt = g[j * K + k];
                dlam += creal(conj(gt) * Sl);
                dom += creal(conj(gt) * So);
            }
            if (state) {
                state[(b * 3 + 0) * K + k] = h;
                state[(b * 3 + 1) * K + k] = Sl;
                state[(b * 3 + 2) * K + k] = So;
            }
        }
        dlambda[k] = dlam;
        domega[k] = dom;
    }
    return 0;
}

/*
 * Flash PD-SSM scan ("Flash PD-SSM: Memory-Optimized Structured Sparse State-Space Models",
 * technical summary: hard selection and gradient propagation).  Per batch b and head e, a real
 * state h in R^N; at every step the transition is A_t = P_{k_t} D_t, where
 *   k_t = argmax_k scores[b,t,e,k]   (ties: the lowest k),
 *   P_k is dictionary matrix k, a one-hot column selector: column j holds a single 1, in row
 *       dict[k*N + j]  (so (P_k v)_i = sum over j with dict[k*N+j] == i of v_j),
 *   D_t = diag(d[b,t,e,:]),
 * and h_t = A_t h_{t-1} + bt[b,t,e,:], h_{-1} = h0 (NULL: zero).  Outputs h [B,L,H,N] and the
 * selection sel [B,L,H] (k_t).
 * Backward (g = dL/dh_t given for every t, so L = sum_t <g_t, h_t>): with the hard forward
 * matrices the adjoint is mu_t = g_t + A_{t+1}^T mu_{t+1}, (A^T mu)_j = d_j mu_{dict[k*N+j]};
 *   dbt_t = mu_t,   dd_t[j] = mu_t[dict[k_t*N+j]] h_{t-1}[j],   dh0 = A_0^T mu_0.
 * The selection is discrete, so its gradient is the straight-through surrogate of the summary
 * (the hard choice in the forward pass, a temperature-tau softmax p = softmax(scores_t / tau) in
 * the backward pass):  c_k = <mu_t, P_k D_t h_{t-1}>,  dscores_t[k] = p_k (c_k - sum_k' p_k' c_k') / tau.
 * g NULL: forward only.  Returns 0 or -1.
 */
int ssm_oracle_pdssm(int64_t B, int64_t L, int64_t H, int64_t N, int64_t K,
                     const double* scores, const int32_t* dict, const double* d, const double* bt,
                     const double* h0, const double* g, double tau, int nthreads,
                     double* h_out, int32_t* sel_out, double* dd, double* dbt, double* dscores,
                     double* dh0) {
    if (B < 0 || L < 0 || H <= 0 || N <= 0 || K <= 0 || !scores || !dict || !d || !bt || !h_out)
        return -1;
    if (g && !(tau > 0.0)) return -1;
    for (int64_t i = 0; i < K * N; ++i)
        if (dict[i] < 0 || dict[i] >= N) return -1;
    nthreads = pick_threads(nthreads);
    int fail = 0;
#pragma omp parallel num_threads(nthreads)
    {
        double* hprev = (double*)malloc(sizeof(double) * (size_t)N);
        double* hnew = (double*)malloc(sizeof(double) * (size_t)N);
        double* mu = (double*)malloc(sizeof(double) * (size_t)N);
        double* w = (double*)malloc(sizeof(double) * (size_t)N);
        double* c = (double*)malloc(sizeof(double) * (size_t)K);
        double* p = (double*)malloc(sizeof(double) * (size_t)K);
        if (!hprev || !hnew || !mu || !w || !c || !p) {
#pragma omp atomic write
            fail = 1;
        }
#pragma omp barrier
        if (!fail) {
#pragma omp for schedule(static)
            for (int64_t be = 0; be < B * H; ++be) {
                const int64_t b = be / H, e = be % H;
                /* forward */
                for (int64_t n = 0; n < N; ++n) hprev[n] = h0 ? h0[be * N + n] : 0.0;
                for (int64_t t = 0; t < L; ++t) {
                    const int64_t row = (b * L + t) * H + e;   /* (b, t, e) */
                    const double* sc = scores + row * K;
                    int64_t kb = 0;
                    for (int64_t k = 1; k < K; ++k)
                        if (sc[k] > sc[kb]) kb = k;
                    if (sel_out) sel_out[row] = (int32_t)kb;
                    for (int64_t n = 0; n < N; ++n) hnew[n] = bt[row * N + n];
                    for (int64_t j = 0; j < N; ++j) hnew[dict[kb * N + j]] += d[row * N + j] * hprev[j];
                    for (int64_t n = 0; n < N; ++n) {
                        h_out[row * N + n] = hnew[n];
                        hprev[n] = hnew[n];
                    }
                }
                if (!g) continue;
                /* backward: w = A_{t+1}^T mu_{t+1} */
                for (int64_t n = 0; n < N; ++n) w[n] = 0.0;
                for (int64_t t = L - 1; t >= 0; --t) {
                    const int64_t row = (b * L + t) * H + e;
                    const double* sc = scores + row * K;
                    int64_t kb = 0;
                    for (int64_t k = 1; k < K; ++k)
                        if (sc[k] > sc[kb]) kb = k;
                    for (int64_t n = 0; n < N; ++n) mu[n] = g[row * N + n] + w[n];
                    const double* hp = t > 0 ? h_out + (row - H) * N : NULL;  /* (b, t-1, e) */
                    for (int64_t n = 0; n < N; ++n) {
                        const double hpn = t > 0 ? hp[n] : (h0 ? h0[be * N + n] : 0.0);
                        if (dbt) dbt[row * N + n] = mu[n];
                        if (dd) dd[row * N + n] = mu[dict[kb * N + n]] * hpn;
                        w[n] = d[row * N + n] * mu[dict[kb * N + n]];
                    }
                    if (dscores) {
                        double mx = sc[0];
                        for (int64_t k = 1; k < K; ++k) mx = sc[k] > mx ? sc[k] : mx;
                        double zs = 0.0;
                        for (int64_t k = 0; k < K; ++k) {
                            p[k] = exp((sc[k] - mx) / tau);
                            zs += p[k];
                        }
                        double pc = 0.0;
                        for (int64_t k = 0; k < K; ++k) {
                            double ck = 0.0;
                            for (int64_t j = 0; j < N; ++j) {
                                const double hpj = t > 0 ? hp[j] : (h0 ? h0[be * N + j] : 0.0);
                                ck += mu[dict[k * N + j]] * d[row * N + j] * hpj;
                            }
                            p[k] /= zs;
                            c[k] = ck;
                            pc += p[k] * ck;
                        }
                        for (int64_t k = 0; k < K; ++k) dscores[row * K + k] = p[k] * (c[k] - pc) / tau;
                    }
                }
                if (dh0)
                    for (int64_t n = 0; n < N; ++n) dh0[be * N + n] = w[n];
            }
        }
        free(hprev); free(hnew); free(mu); free(w); free(c); free(p);
    }
    return fail ? -1 : 0;
}

/*
 * Step-size projection in front of the real scan ("选择性状态空间模型(S3M)原理与工程实践" §1.1:
 * delta = softplus(projection(x)); §4.1 merges the discretisation with this matrix product).  Per
 * row m (one (batch, step) pair) the pre-activation of every channel d is a rank-R linear map of
 * the row's low-rank input u:
 *     delta_raw[m, d] = sum_r u[m, r] w[d, r] + bias[d]
 * and for an upstream gradient g = dL/d delta_raw:
 *     du[m, r] = sum_d g[m, d] w[d, r],   dw[d, r] = sum_m g[m, d] u[m, r],   dbias[d] = sum_m g[m, d].
 * Plain loops in float64, rows split across threads (forward, du) or channels split across threads
 * (dw, dbias); every sum runs in index order.  bias and dbias may be NULL.
 */
int ssm_oracle_dtproj(int64_t M, int64_t D, int64_t R, const double* u, const double* w,
                      const double* bias, double* out) {
    if (M < 0 || D < 1 || R < 1 || !u || !w || !out) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int64_t r = 0; r < R; ++r) acc += u[m * R + r] * w[d * R + r];
            out[m * D + d] = acc + (bias ? bias[d] : 0.0);
        }
    return 0;
}

int ssm_oracle_dtproj_bwd(int64_t M, int64_t D, int64_t R, const double* u, const double* w,
                          const double* g, double* du, double* dw, double* dbias) {
    if (M < 0 || D < 1 || R < 1 || !u || !w || !g || !du || !dw) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t r = 0; r < R; ++r) {
            double acc = 0.0;
            for (int64_t d = 0; d < D; ++d) acc += g[m * D + d] * w[d * R + r];
            du[m * R + r] = acc;
        }
#pragma omp parallel for schedule(static)
    for (int64_t d = 0; d < D; ++d) {
        for (int64_t r = 0; r < R; ++r) {
            double acc = 0.0;
            for (int64_t m = 0; m < M; ++m) acc += g[m * D + d] * u[m * R + r];
            dw[d * R + r] = acc;
        }
        if (dbias) {
            double acc = 0.0;
            for (int64_t m = 0; m < M; ++m) acc += g[m * D + d];
            dbias[d] = acc;
        }
    }
    return 0;
}
