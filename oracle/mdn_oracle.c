/*
 * mdn_oracle.c -- fp64 CPU oracle for the Momentum DeltaNet (MDN) forward
 * pass and decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline / reference arm may call this code.  It shares no
 * code, header, table or helper with the CUDA library, and the library never
 * calls it.
 *
 * What it follows ("MDN: Parallelizing Stepwise Momentum for Delta Linear
 * Attention"; paper.rainbus.top summary, step 1; ijyty.com article, sections
 * 3 and 6): per head, with S (fast weight) and M (momentum), both d_k x d_v,
 *
 *     p_t       = alpha_t k_t
 *     vtilde_t  = v_t - S_{t-1}^T p_t
 *     M_t       = mu_t M_{t-1} - eta_t k_t vtilde_t^T
 *     S_t       = alpha_t S_{t-1} - beta_t M_t
 *     o_t       = S_t^T qhat_t,   qhat_t = q_t - d k_t   (output correction,
 *                                                        summary step 7)
 *
 * with alpha_t = exp(alpha_log_t) and mu_t = exp(mu_log_t).  The chunkwise
 * method reaches this result exactly (up to rounding order), so the oracle is
 * this definition, stepped one token at a time in fp64, with no chunking and
 * no log domain.  Heads are independent; OpenMP runs them in parallel.
 *
 * mdn_oracle_chunk_coeffs writes the per-chunk coefficients of the unrolled
 * form (summary steps 2 and 5) by their plain definitions, for checking a
 * coefficient kernel.  Every cumulative quantity restarts at each chunk.
 *
 * Layouts (all row-major, contiguous):
 *   q, k, v, o, vtilde : [B, T, H, d]     (decode step: [B, H, d])
 *   gates              : [B, T, H]        (decode step: [B, H])
 *   S0, M0, S_T, M_T   : [B, H, d_k, d_v], row index over d_k
 *
 * mdn_oracle_gates maps raw per-token pre-activations to the four gates by the
 * stable parameterisation (summary, step 6; article, sections 5 and 8):
 *     eta   = tanh(x) + 1            (or 2 sigmoid(x), the ablated variant)
 *     theta = arctan(eta * s)
 *     alpha = cos^2(theta) sigmoid(a),  beta = sin^2(theta) sigmoid(b)
 *     log mu = max(log sigmoid(c), mu_log_min)
 *
 * Parity pins: every function here is checked against results the pages or
 * the mathematics fix (closed form, special cases, spectrum, hand-worked
 * values) by the CPU tests; none is unpinned.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int mdn_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* One head, T tokens.  Token t of this head sits at q + t*tok_stride (and
 * likewise k, v, o, vt); its gates at alpha_log + t*gate_stride.  S and M are
 * the d_k x d_v states, updated in place.  work holds 2*d_k doubles. */
static void run_head(const double *q, const double *k, const double *v,
                     ptrdiff_t tok_stride,
                     const double *alpha_log, const double *mu_log,
                     const double *beta, const double *eta, ptrdiff_t gate_stride,
                     double d, int T, int dk, int dv,
                     double *S, double *M, double *o, double *vt, double *work)
{
    double *p = work;          /* p_t = alpha_t k_t          */
    double *qhat = work + dk;  /* qhat_t = q_t - d k_t       */
    for (int t = 0; t < T; ++t) {
        const double *qt = q + (ptrdiff_t)t * tok_stride;
        const double *kt = k + (ptrdiff_t)t * tok_stride;
        const double *vv = v + (ptrdiff_t)t * tok_stride;
        double *ot = o + (ptrdiff_t)t * tok_stride;
        double *vtt = vt + (ptrdiff_t)t * tok_stride;
        const double alpha = exp(alpha_log[(ptrdiff_t)t * gate_stride]);
        const double mu = exp(mu_log[(ptrdiff_t)t * gate_stride]);
        const double b = beta[(ptrdiff_t)t * gate_stride];
        const double e = eta[(ptrdiff_t)t * gate_stride];

        for (int i = 0; i < dk; ++i) p[i] = alpha * kt[i];

        /* vtilde_t = v_t - S_{t-1}^T p_t */
        for (int j = 0; j < dv; ++j) vtt[j] = vv[j];
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) vtt[j] -= S[(ptrdiff_t)i * dv + j] * p[i];

        /* M_t = mu_t M_{t-1} - eta_t k_t vtilde_t^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                double *m = &M[(ptrdiff_t)i * dv + j];
                *m = mu * (*m) - e * kt[i] * vtt[j];
            }

        /* S_t = alpha_t S_{t-1} - beta_t M_t */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                ptrdiff_t ij = (ptrdiff_t)i * dv + j;
                S[ij] = alpha * S[ij] - b * M[ij];
            }

        /* o_t = S_t^T qhat_t */
        for (int i = 0; i < dk; ++i) qhat[i] = qt[i] - d * kt[i];
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) ot[j] += S[(ptrdiff_t)i * dv + j] * qhat[i];
    }
}

/* Whole-sequence forward pass.  S0/M0 may be NULL (zero states).  Returns 0,
 * or -1 on a bad argument or an allocation failure. */
int mdn_oracle_chunk_fwd(const double *q, const double *k, const double *v,
                         const double *alpha_log, const double *mu_log,
                         const double *beta, const double *eta, double d,
                         const double *S0, const double *M0,
                         int B, int T, int H, int dk, int dv,
                         double *o, double *vtilde, double *S_T, double *M_T)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (dk != dv) return -1; /* q, k, v share one token layout */
    const ptrdiff_t state = (ptrdiff_t)dk * dv;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H, h = bh % H;
        double *work = (double *)malloc(sizeof(double) * 2 * (size_t)dk);
        if (!work) { failed |= 1; continue; }
        double *S = S_T + (ptrdiff_t)bh * state;
        double *M = M_T + (ptrdiff_t)bh * state;
        if (S0) memcpy(S, S0 + (ptrdiff_t)bh * state, sizeof(double) * state);
        else memset(S, 0, sizeof(double) * state);
        if (M0) memcpy(M, M0 + (ptrdiff_t)bh * state, sizeof(double) * state);
        else memset(M, 0, sizeof(double) * state);
        const ptrdiff_t tok0 = ((ptrdiff_t)b * T * H + h) * dk;
        const ptrdiff_t gate0 = (ptrdiff_t)b * T * H + h;
        run_head(q + tok0, k + tok0, v + tok0, (ptrdiff_t)H * dk,
                 alpha_log + gate0, mu_log + gate0, beta + gate0, eta + gate0, H,
                 d, T, dk, dv, S, M, o + tok0, vtilde + tok0, work);
        free(work);
    }
    return failed ? -1 : 0;
}

/* One decode token for every head: S, M updated in place; o and vtilde
 * ([B,H,d]) written; vtilde may be NULL. */
int mdn_oracle_step(const double *q, const double *k, const double *v,
                    const double *alpha_log, const double *mu_log,
                    const double *beta, const double *eta, double d,
                    double *S, double *M, int B, int H, int dk, int dv,
                    double *o, double *vtilde)
{
    if (B < 0 || H < 0 || dk <= 0 || dv <= 0 || dk != dv) return -1;
    const ptrdiff_t state = (ptrdiff_t)dk * dv;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int bh = 0; bh < B * H; ++bh) {
        double *work = (double *)malloc(sizeof(double) * (2 * (size_t)dk + (size_t)dv));
        if (!work) { failed |= 1; continue; }
        double *vt = vtilde ? vtilde + (ptrdiff_t)bh * dv : work + 2 * dk;
        const ptrdiff_t tok = (ptrdiff_t)bh * dk;
        run_head(q + tok, k + tok, v + tok, 0, alpha_log + bh, mu_log + bh,
                 beta + bh, eta + bh, 0, d, 1, dk, dv, S + (ptrdiff_t)bh * state,
                 M + (ptrdiff_t)bh * state, o + (ptrdiff_t)bh * dv, vt, work);
        free(work);
    }
    return failed ? -1 : 0;
}

/* Per-chunk coefficients of the unrolled form, each cumulative quantity
 * restarting at the first token of its chunk (positions r = 1..L of a chunk
 * of L <= C tokens; the last chunk may be short):
 *
 *   la_r = sum_{j<=r} alpha_log_j                 (log of alphabar_r)
 *   lm_r = sum_{j<=r} mu_log_j                    (log of mubar_r)
 *   lc_r = log c_r,  c_r = sum_{j<=r} beta_j mubar_j / alphabar_j
 *   gamma_{r,i} = eta_i * (alphabar_r / mubar_i) * (c_r - c_{i-1}),  i <= r
 *              = eta_i * sum_{j=i}^{r} (alphabar_r/alphabar_j) beta_j (mubar_j/mubar_i)
 *
 * (the second form of Gamma writes c_r - c_{i-1} as the sum of its terms; the
 * eta_i factor is the write scale of token i, see the reading of the unrolled
 * form in the design notes).  la, lm, lc: [B, H, T];  gamma: [B, H, NT, C, C]
 * with NT = ceil(T / C), zero above the diagonal and in rows/columns past the
 * end of a short last chunk.  gamma may be NULL. */
int mdn_oracle_chunk_coeffs(const double *alpha_log, const double *mu_log,
                            const double *beta, const double *eta,
                            int B, int T, int H, int C,
                            double *la, double *lm, double *lc, double *gamma)
{
    if (B < 0 || T < 0 || H < 0 || C <= 0) return -1;
    const int NT = (T + C - 1) / C;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H, h = bh % H;
        for (int n = 0; n < NT; ++n) {
            const int t0 = n * C;
            const int L = (T - t0) < C ? (T - t0) : C;
            double *la_c = la + (ptrdiff_t)bh * T + t0;
            double *lm_c = lm + (ptrdiff_t)bh * T + t0;
            double *lc_c = lc + (ptrdiff_t)bh * T + t0;
            double sa = 0.0, sm = 0.0;
            for (int r = 0; r < L; ++r) {
                const ptrdiff_t g = ((ptrdiff_t)b * T + t0 + r) * H + h;
                sa += alpha_log[g];
                sm += mu_log[g];
                la_c[r] = sa;
                lm_c[r] = sm;
            }
            /* lc_r = log sum_{j<=r} exp(log beta_j + lm_j - la_j), evaluated
             * as a shifted log-sum-exp so that fp64 does not overflow. */
            for (int r = 0; r < L; ++r) {
                double mx = -INFINITY;
                for (int j = 0; j <= r; ++j) {
                    const ptrdiff_t g = ((ptrdiff_t)b * T + t0 + j) * H + h;
                    const double x = log(beta[g]) + lm_c[j] - la_c[j];
                    if (x > mx) mx = x;
                }
                double s = 0.0;
                if (mx > -INFINITY) {
                    for (int j = 0; j <= r; ++j) {
                        const ptrdiff_t g = ((ptrdiff_t)b * T + t0 + j) * H + h;
                        s += exp(log(beta[g]) + lm_c[j] - la_c[j] - mx);
                    }
                    lc_c[r] = mx + log(s);
                } else {
                    lc_c[r] = -INFINITY;
                }
            }
            if (!gamma) continue;
            double *G = gamma + ((ptrdiff_t)bh * NT + n) * C * C;
            for (int r = 0; r < C; ++r)
                for (int i = 0; i < C; ++i) {
                    double acc = 0.0;
                    if (r < L && i <= r) {
                        const ptrdiff_t gi = ((ptrdiff_t)b * T + t0 + i) * H + h;
                        for (int j = i; j <= r; ++j) {
                            const ptrdiff_t gj = ((ptrdiff_t)b * T + t0 + j) * H + h;
                            acc += exp(la_c[r] - la_c[j]) * beta[gj] * exp(lm_c[j] - lm_c[i]);
                        }
                        acc *= eta[gi];
                    }
                    G[(ptrdiff_t)r * C + i] = acc;
                }
        }
    }
    return 0;
}

/* log(sigmoid(x)) without overflow for either sign of x. */
static double log_sigmoid(double x)
{
    return x >= 0.0 ? -log1p(exp(-x)) : x - log1p(exp(x));
}

/* The four gates of n tokens from their pre-activations (see the header).
 * eta_act: 0 = tanh(x) + 1, 1 = 2 sigmoid(x).  Outputs: alpha_log = log alpha,
 * mu_log, beta, eta, each [n]. */
int mdn_oracle_gates(const double *x_eta, const double *a, const double *b,
                     const double *c, ptrdiff_t n, double s, double mu_log_min,
                     int eta_act, double *alpha_log, double *mu_log, double *beta,
                     double *eta)
{
    if (n < 0 || (eta_act != 0 && eta_act != 1)) return -1;
    for (ptrdiff_t i = 0; i < n; ++i) {
        const double e = eta_act == 0 ? tanh(x_eta[i]) + 1.0 : 2.0 / (1.0 + exp(-x_eta[i]));
        const double theta = atan(e * s);
        const double ct = cos(theta), st = sin(theta);
        eta[i] = e;
        alpha_log[i] = log(ct * ct) + log_sigmoid(a[i]);
        beta[i] = st * st * exp(log_sigmoid(b[i]));
        const double lm = log_sigmoid(c[i]);
        mu_log[i] = lm > mu_log_min ? lm : mu_log_min;
    }
    return 0;
}
