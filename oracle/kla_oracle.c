/*
 * kla_oracle.c -- plain sequential CPU oracle of the Kalman linear-attention
 * forward pass, in fp64.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file; only the tests, the small smoke check and the benchmark's CPU
 * baseline leg do. It shares no code, header or constant with the CUDA path.
 *
 * What it computes (Kalman Linear Attention, technical summary section 1
 * "probabilistic formulation", and the Kalman Delta Networks abstract for the
 * isotropic variant): per sequence n and head h, an information-form Kalman
 * filter whose state is a precision lambda and an information vector eta.
 *
 *   diagonal mode, per key i (one precision per key dimension):
 *     predict (exactly discretised OU prior, decay a, process noise qn):
 *         den      = a[t,i]^2 + qn[t,i] * lambda[i]
 *         g        = a[t,i] / den              (forget gate, precision ratio)
 *         lambda[i]= lambda[i] / den           (Moebius map of lambda)
 *         eta[i,:] = g * eta[i,:]
 *     update (token = noisy observation through k with value precision beta):
 *         lambda[i]+= beta[t] * k[t,i]^2
 *         eta[i,:] += beta[t] * k[t,i] * v[t,:]
 *     readout (posterior mean through the query):
 *         o[t,:]   = sum_i q[t,i] * eta[i,:] / lambda[i]
 *
 *   isotropic mode (one precision per head): a, qn per (t,h);
 *         den = a^2 + qn*lambda ; g = a/den ; lambda = lambda/den + beta*|k|^2/dk
 *         eta[i,:] = g*eta[i,:] + beta*k[i]*v ; o = sum_i q[i]*eta[i,:]/lambda
 *
 * Every step predicts and then updates, the first one included: lambda0/eta0
 * are the posterior before the first token, so a sequence split in two calls
 * (final state of the first handed to the second) equals one call.
 * Varlen: each packed sequence restarts from its own lambda0/eta0.
 *
 * The Moebius helpers expose the 2x2 matrix form of one predict+update step,
 *     lambda' = ((1 + b*qn) lambda + b*a^2) / (qn lambda + a^2),  b = beta*k^2,
 * (Kalman Linear Attention, technical summary section 2, the Moebius
 * precision recursion) for the associativity checks.
 *
 * Inputs are float (bf16 and fp32 values are exact in float); all arithmetic is
 * double. Layouts are row-major with tokens flattened over the batch:
 *   q,k [Ntok,H,dk]  v [Ntok,H,dv]  a,qn [Ntok,H,dk] (iso [Ntok,H])  beta [Ntok,H]
 *   lambda0 [N,H,dk] (iso [N,H])  eta0 [N,H,dk,dv]   out [Ntok,H,dv]
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One (sequence, head) unit, tokens [t0, t1). Returns 0 on success. */
static int run_unit(int n, int h, long t0, long t1, int H, int dk, int dv, int iso,
                    const float *q, const float *k, const float *v,
                    const float *a, const float *qn, const float *beta,
                    const float *lambda0, const float *eta0,
                    double *out, double *final_lambda, double *final_eta,
                    double *lambda_traj)
{
    int nl = iso ? 1 : dk;
    double *lam = (double *)malloc(sizeof(double) * nl);
    double *eta = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    if (!lam || !eta) { free(lam); free(eta); return 1; }

    for (int i = 0; i < nl; ++i)
        lam[i] = lambda0 ? (double)lambda0[((size_t)n * H + h) * nl + i] : 1.0;
    for (size_t e = 0; e < (size_t)dk * dv; ++e)
        eta[e] = eta0 ? (double)eta0[((size_t)n * H + h) * dk * dv + e] : 0.0;

    for (long t = t0; t < t1; ++t) {
        size_t th = (size_t)t * H + h;           /* token-head index */
        const float *qt = q + th * dk, *kt = k + th * dk, *vt = v + th * dv;
        double bt = (double)beta[th];
        if (iso) {
            double at = a[th], qnt = qn[th];
            double ksq = 0.0;
            for (int i = 0; i < dk; ++i) ksq += (double)kt[i] * (double)kt[i];
            double den = at * at + qnt * lam[0];
            double g = at / den;
            lam[0] = lam[0] / den + bt * ksq / (double)dk;
            for (int i = 0; i < dk; ++i) {
                double w = bt * (double)kt[i];
                double *row = eta + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) row[j] = g * row[j] + w * (double)vt[j];
            }
            if (lambda_traj) lambda_traj[th] = lam[0];
        } else {
            const float *at = a + th * dk, *qnt = qn + th * dk;
            for (int i = 0; i < dk; ++i) {
                double ai = at[i], ki = kt[i];
                double den = ai * ai + (double)qnt[i] * lam[i];
                double g = ai / den;
                lam[i] = lam[i] / den + bt * ki * ki;
                double w = bt * ki;
                double *row = eta + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) row[j] = g * row[j] + w * (double)vt[j];
                if (lambda_traj) lambda_traj[th * dk + i] = lam[i];
            }
        }
        if (out) {
            double *ot = out + th * dv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                double c = (double)qt[i] / lam[iso ? 0 : i];
                const double *row = eta + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) ot[j] += c * row[j];
            }
        }
    }
    if (final_lambda)
        for (int i = 0; i < nl; ++i) final_lambda[((size_t)n * H + h) * nl + i] = lam[i];
    if (final_eta)
        memcpy(final_eta + ((size_t)n * H + h) * dk * dv, eta, sizeof(double) * (size_t)dk * dv);
    free(lam);
    free(eta);
    return 0;
}

/*
 * Full forward. cu_seqlens (host int32 [num_seqs+1]) or NULL for B rows of T
 * tokens. Any of out / final_lambda / final_eta / lambda_traj may be NULL.
 * lambda_traj receives the posterior precision after every token
 * ([Ntok,H,dk], iso [Ntok,H]). units_begin/units_end select a sub-range of the
 * (sequence, head) units, unit = n*H + h (pass 0 and -1 for all); the
 * benchmark's CPU baseline times a bounded sample this way.
 * num_threads <= 0 uses the OpenMP default. Returns 0 on success.
 */
int kla_oracle_forward(int B, int T, int H, int dk, int dv, int iso,
                       const int *cu_seqlens, int num_seqs,
                       const float *q, const float *k, const float *v,
                       const float *a, const float *qn, const float *beta,
                       const float *lambda0, const float *eta0,
                       double *out, double *final_lambda, double *final_eta,
                       double *lambda_traj, long units_begin, long units_end,
                       int num_threads)
{
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    int N = cu_seqlens ? num_seqs : B;
    long units = (long)N * H;
    if (units_end < 0 || units_end > units) units_end = units;
    if (units_begin < 0) units_begin = 0;
    int err = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
#endif
    for (long u = units_begin; u < units_end; ++u) {
        int n = (int)(u / H), h = (int)(u % H);
        long t0 = cu_seqlens ? cu_seqlens[n] : (long)n * T;
        long t1 = cu_seqlens ? cu_seqlens[n + 1] : (long)(n + 1) * T;
        err |= run_unit(n, h, t0, t1, H, dk, dv, iso, q, k, v, a, qn, beta,
                        lambda0, eta0, out, final_lambda, final_eta, lambda_traj);
    }
    return err;
}

/* Threads the OpenMP runtime would use (1 without OpenMP). */
int kla_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- Moebius form of one predict+update step ---------------------------- */

/* M = [[1 + b*qn, b*a^2], [qn, a^2]] with b = beta*k^2 (or beta*|k|^2/dk in
 * isotropic mode). lambda' = (M00 lambda + M01) / (M10 lambda + M11). */
void kla_oracle_mobius_element(double a, double qn, double b, double *M)
{
    M[0] = 1.0 + b * qn;
    M[1] = b * a * a;
    M[2] = qn;
    M[3] = a * a;
}

/* out = L * R (apply R first, then L). out may alias neither input. */
void kla_oracle_mobius_compose(const double *L, const double *R, double *out)
{
    out[0] = L[0] * R[0] + L[1] * R[2];
    out[1] = L[0] * R[1] + L[1] * R[3];
    out[2] = L[2] * R[0] + L[3] * R[2];
    out[3] = L[2] * R[1] + L[3] * R[3];
}

double kla_oracle_mobius_apply(const double *M, double lam)
{
    return (M[0] * lam + M[1]) / (M[2] * lam + M[3]);
}

/* ---- Kalman Delta Network: the Kalman-gain residual (delta-style) write ---
 *
 * Kalman Delta Networks abstract: the memory is the state of a linear-Gaussian
 * state-space model; the transition propagates its mean and its uncertainty,
 * and the Kalman gain weights each residual write; diagonal KDN projects each
 * one-step posterior onto diagonal Gaussians (online mean-field variational
 * inference), isotropic KDN keeps one uncertainty scalar per head. The pages
 * give no equations; this is the plainest reading of that statement:
 *
 *   state: mean M[dk][dv] (one column per value dimension, all columns with the
 *   same key covariance), diagonal covariance diag(1/lambda) (iso: I/lambda).
 *   predict (the same OU prior as the KLA filter):
 *       M~[i,:]   = a[t,i] * M[i,:]
 *       lambda~[i]= lambda[i] / (a[t,i]^2 + qn[t,i] * lambda[i])
 *   observe v = M^T k + noise of precision beta (per value dimension):
 *       innovation  r[j] = v[j] - sum_i k[i] M~[i,j]
 *       gain        G[i] = (k[i]/lambda~[i]) * beta / (1 + beta * sum_i k[i]^2/lambda~[i])
 *       mean write  M[i,j] = M~[i,j] + G[i] * r[j]      (the exact posterior mean
 *                   given the diagonal prior: the textbook Kalman update)
 *       precision   lambda[i] = lambda~[i] + beta * k[i]^2   (the diagonal of the
 *                   posterior precision lambda~ + beta k k^T: the mean-field
 *                   projection; iso: + beta * |k|^2 / dk as for the KLA filter)
 *   readout (posterior mean through the query): o[j] = sum_i q[i] M[i,j]
 *
 * So the precision path is the KLA filter's Moebius recursion, and only the mean
 * write differs: it is coupled across keys through the shared innovation. With
 * one-hot keys both coincide (per key: M = (lambda~ M~ + beta v)/(lambda~ + beta)).
 * M0 is the prior mean before the first token (default 0), lambda0 its
 * precision (default 1); layouts as for kla_oracle_forward, M0 / final_M
 * [N,H,dk,dv].
 */
static int run_kdn_unit(int n, int h, long t0, long t1, int H, int dk, int dv, int iso,
                        const float *q, const float *k, const float *v,
                        const float *a, const float *qn, const float *beta,
                        const float *lambda0, const float *M0,
                        double *out, double *final_lambda, double *final_M)
{
    int nl = iso ? 1 : dk;
    double *lam = (double *)malloc(sizeof(double) * nl);
    double *M = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *w = (double *)malloc(sizeof(double) * dk);      /* k / lambda~ */
    double *r = (double *)malloc(sizeof(double) * dv);      /* innovation */
    if (!lam || !M || !w || !r) { free(lam); free(M); free(w); free(r); return 1; }

    for (int i = 0; i < nl; ++i)
        lam[i] = lambda0 ? (double)lambda0[((size_t)n * H + h) * nl + i] : 1.0;
    for (size_t e = 0; e < (size_t)dk * dv; ++e)
        M[e] = M0 ? (double)M0[((size_t)n * H + h) * dk * dv + e] : 0.0;

    for (long t = t0; t < t1; ++t) {
        size_t th = (size_t)t * H + h;
        const float *qt = q + th * dk, *kt = k + th * dk, *vt = v + th * dv;
        double bt = (double)beta[th];
        /* predict: mean decays by a, precision through the OU prior */
        for (int i = 0; i < dk; ++i) {
            double ai = iso ? (double)a[th] : (double)a[th * dk + i];
            double *row = M + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) row[j] *= ai;
        }
        if (iso) {
            double den = (double)a[th] * (double)a[th] + (double)qn[th] * lam[0];
            lam[0] = lam[0] / den;
        } else {
            for (int i = 0; i < dk; ++i) {
                double ai = a[th * dk + i];
                lam[i] = lam[i] / (ai * ai + (double)qn[th * dk + i] * lam[i]);
            }
        }
        /* innovation and gain */
        double s = 0.0, ksq = 0.0;
        for (int i = 0; i < dk; ++i) {
            double ki = kt[i];
            w[i] = ki / lam[iso ? 0 : i];
            s += ki * w[i];
            ksq += ki * ki;
        }
        for (int j = 0; j < dv; ++j) {
            double pred = 0.0;
            for (int i = 0; i < dk; ++i) pred += (double)kt[i] * M[(size_t)i * dv + j];
            r[j] = (double)vt[j] - pred;
        }
        double gam = bt / (1.0 + bt * s);
        /* residual write */
        for (int i = 0; i < dk; ++i) {
            double gi = gam * w[i];
            double *row = M + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) row[j] += gi * r[j];
        }
        /* precision: diagonal of the posterior precision */
        if (iso) lam[0] += bt * ksq / (double)dk;
        else
            for (int i = 0; i < dk; ++i) lam[i] += bt * (double)kt[i] * (double)kt[i];
        if (out) {
            double *ot = out + th * dv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                double c = qt[i];
                const double *row = M + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) ot[j] += c * row[j];
            }
        }
    }
    if (final_lambda)
        for (int i = 0; i < nl; ++i) final_lambda[((size_t)n * H + h) * nl + i] = lam[i];
    if (final_M)
        memcpy(final_M + ((size_t)n * H + h) * dk * dv, M, sizeof(double) * (size_t)dk * dv);
    free(lam); free(M); free(w); free(r);
    return 0;
}

/* KDN forward; arguments as kla_oracle_forward, M0 / final_M in place of eta. */
int kdn_oracle_forward(int B, int T, int H, int dk, int dv, int iso,
                       const int *cu_seqlens, int num_seqs,
                       const float *q, const float *k, const float *v,
                       const float *a, const float *qn, const float *beta,
                       const float *lambda0, const float *M0,
                       double *out, double *final_lambda, double *final_M,
                       long units_begin, long units_end, int num_threads)
{
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    int N = cu_seqlens ? num_seqs : B;
    long units = (long)N * H;
    if (units_end < 0 || units_end > units) units_end = units;
    if (units_begin < 0) units_begin = 0;
    int err = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
#endif
    for (long u = units_begin; u < units_end; ++u) {
        int n = (int)(u / H), h = (int)(u % H);
        long t0 = cu_seqlens ? cu_seqlens[n] : (long)n * T;
        long t1 = cu_seqlens ? cu_seqlens[n + 1] : (long)(n + 1) * T;
        err |= run_kdn_unit(n, h, t0, t1, H, dk, dv, iso, q, k, v, a, qn, beta,
                            lambda0, M0, out, final_lambda, final_M);
    }
    return err;
}

/* ---- Gradients of the KLA filter (reverse mode) --------------------------
 *
 * Kalman Linear Attention abstract: the layer is meant for efficient parallel
 * training, so its forward pass has a backward pass. This is the plain reverse
 * sweep of the recursion above, step by step in reverse order, with every
 * state kept from the forward sweep (lambda and eta before each token's
 * predict). Given the loss gradients dout [Ntok,H,dv] and, optionally,
 * dfinal_lambda / dfinal_eta of the final state, per token (diag, per key i):
 *   readout  o = sum_i q_i eta'_i / lam'_i:
 *       dq_i     = sum_j do_j eta'_ij / lam'_i
 *       deta'_ij+= q_i do_j / lam'_i
 *       dlam'_i += -q_i (sum_j eta'_ij do_j) / lam'_i^2
 *   update   eta' = g eta + beta k v^T, lam' = lam~ + beta k^2:
 *       dg_i     = sum_j deta'_ij eta_ij       (eta: before the predict)
 *       dv_j    += sum_i deta'_ij beta k_i
 *       dk_i    += beta sum_j deta'_ij v_j + 2 beta k_i dlam'_i
 *       dbeta   += sum_i k_i sum_j deta'_ij v_j + sum_i k_i^2 dlam'_i
 *       dlam~_i  = dlam'_i
 *   predict  den = a^2 + qn lam, lam~ = lam / den, g = a / den:
 *       dden     = -(dlam~ lam + dg a) / den^2
 *       da       = dg / den + 2 a dden,  dqn = lam dden
 *       dlam_i   = dlam~ / den + qn dden,  deta_ij = g_i deta'_ij
 * (isotropic: a, qn, g, lam per head; the precision term beta |k|^2 / dk).
 * The adjoints left after the first token are dlambda0, deta0.
 */
static int run_unit_backward(int n, int h, long t0, long t1, int H, int dk, int dv, int iso,
                             const float *q, const float *k, const float *v,
                             const float *a, const float *qn, const float *beta,
                             const float *lambda0, const float *eta0, const float *dout,
                             const float *dfinal_lambda, const float *dfinal_eta,
                             double *dq, double *dk_, double *dv_, double *da, double *dqn,
                             double *dbeta, double *dlambda0, double *deta0)
{
    int nl = iso ? 1 : dk;
    long L = t1 - t0;
    size_t S = (size_t)dk * dv;
    /* states before each token's predict: lam_s[t][nl], eta_s[t][dk*dv]; and the final one */
    double *lam_s = (double *)malloc(sizeof(double) * nl * (size_t)(L + 1));
    double *eta_s = (double *)malloc(sizeof(double) * S * (size_t)(L + 1));
    double *dlam = (double *)malloc(sizeof(double) * nl);
    double *deta = (double *)malloc(sizeof(double) * S);
    double *dlt = (double *)malloc(sizeof(double) * nl);   /* adjoint of lam~ */
    double *dg = (double *)malloc(sizeof(double) * nl);
    double *pk = (double *)malloc(sizeof(double) * dk);    /* sum_j deta'_ij v_j */
    if (!lam_s || !eta_s || !dlam || !deta || !dlt || !dg || !pk) {
        free(lam_s); free(eta_s); free(dlam); free(deta); free(dlt); free(dg); free(pk);
        return 1;
    }
    size_t u = (size_t)n * H + h;
    for (int i = 0; i < nl; ++i) lam_s[i] = lambda0 ? (double)lambda0[u * nl + i] : 1.0;
    for (size_t e = 0; e < S; ++e) eta_s[e] = eta0 ? (double)eta0[u * S + e] : 0.0;

    /* forward sweep, keeping every state */
    for (long s = 0; s < L; ++s) {
        size_t th = (size_t)(t0 + s) * H + h;
        const float *kt = k + th * dk, *vt = v + th * dv;
        const double *lp = lam_s + (size_t)s * nl, *ep = eta_s + (size_t)s * S;
        double *ln = lam_s + (size_t)(s + 1) * nl, *en = eta_s + (size_t)(s + 1) * S;
        double bt = beta[th], ksq = 0.0;
        for (int i = 0; i < dk; ++i) ksq += (double)kt[i] * (double)kt[i];
        for (int i = 0; i < nl; ++i) {
            double ai = iso ? a[th] : a[th * dk + i], qi = iso ? qn[th] : qn[th * dk + i];
            double den = ai * ai + qi * lp[i];
            ln[i] = lp[i] / den + (iso ? bt * ksq / (double)dk : bt * (double)kt[i] * (double)kt[i]);
        }
        for (int i = 0; i < dk; ++i) {
            int c = iso ? 0 : i;
            double ai = iso ? a[th] : a[th * dk + i], qi = iso ? qn[th] : qn[th * dk + i];
            double g = ai / (ai * ai + qi * lp[c]);
            for (int j = 0; j < dv; ++j)
                en[(size_t)i * dv + j] = g * ep[(size_t)i * dv + j] + bt * (double)kt[i] * (double)vt[j];
        }
    }

    /* reverse sweep */
    for (int i = 0; i < nl; ++i) dlam[i] = dfinal_lambda ? (double)dfinal_lambda[u * nl + i] : 0.0;
    for (size_t e = 0; e < S; ++e) deta[e] = dfinal_eta ? (double)dfinal_eta[u * S + e] : 0.0;
    for (long s = L - 1; s >= 0; --s) {
        size_t th = (size_t)(t0 + s) * H + h;
        const float *qt = q + th * dk, *kt = k + th * dk, *vt = v + th * dv, *dot = dout + th * dv;
        const double *lp = lam_s + (size_t)s * nl, *ep = eta_s + (size_t)s * S;
        const double *ln = lam_s + (size_t)(s + 1) * nl, *en = eta_s + (size_t)(s + 1) * S;
        double bt = beta[th], db = 0.0;
        /* readout */
        for (int i = 0; i < dk; ++i) {
            int c = iso ? 0 : i;
            double eo = 0.0;
            for (int j = 0; j < dv; ++j) eo += en[(size_t)i * dv + j] * (double)dot[j];
            dq[th * dk + i] = eo / ln[c];
            dlam[c] += -(double)qt[i] * eo / (ln[c] * ln[c]);
            for (int j = 0; j < dv; ++j) deta[(size_t)i * dv + j] += (double)qt[i] * (double)dot[j] / ln[c];
        }
        /* update */
        for (int c = 0; c < nl; ++c) dg[c] = 0.0;
        for (int j = 0; j < dv; ++j) dv_[th * dv + j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            int c = iso ? 0 : i;
            double gi = 0.0, p = 0.0;
            for (int j = 0; j < dv; ++j) {
                double d = deta[(size_t)i * dv + j];
                gi += d * ep[(size_t)i * dv + j];
                p += d * (double)vt[j];
                dv_[th * dv + j] += d * bt * (double)kt[i];
            }
            dg[c] += gi;
            pk[i] = p;
        }
        for (int i = 0; i < dk; ++i) {
            int c = iso ? 0 : i;
            double ki = kt[i];
            double lamterm = iso ? 2.0 * bt * ki * dlam[0] / (double)dk : 2.0 * bt * ki * dlam[i];
            dk_[th * dk + i] = bt * pk[i] + lamterm;
            db += ki * pk[i] + (iso ? ki * ki * dlam[0] / (double)dk : ki * ki * dlam[c]);
        }
        dbeta[th] = db;
        for (int c = 0; c < nl; ++c) dlt[c] = dlam[c];
        /* predict */
        for (int c = 0; c < nl; ++c) {
            double ai = iso ? a[th] : a[th * dk + c], qi = iso ? qn[th] : qn[th * dk + c];
            double den = ai * ai + qi * lp[c];
            double dden = -(dlt[c] * lp[c] + dg[c] * ai) / (den * den);
            double dai = dg[c] / den + 2.0 * ai * dden;
            double dqi = lp[c] * dden;
            if (iso) { da[th] = dai; dqn[th] = dqi; }
            else { da[th * dk + c] = dai; dqn[th * dk + c] = dqi; }
            dlam[c] = dlt[c] / den + qi * dden;
        }
        for (int i = 0; i < dk; ++i) {
            int c = iso ? 0 : i;
            double ai = iso ? a[th] : a[th * dk + i], qi = iso ? qn[th] : qn[th * dk + i];
            double g = ai / (ai * ai + qi * lp[c]);
            for (int j = 0; j < dv; ++j) deta[(size_t)i * dv + j] *= g;
        }
    }
    if (dlambda0)
        for (int c = 0; c < nl; ++c) dlambda0[u * nl + c] = dlam[c];
    if (deta0) memcpy(deta0 + u * S, deta, sizeof(double) * S);
    free(lam_s); free(eta_s); free(dlam); free(deta); free(dlt); free(dg); free(pk);
    return 0;
}

/* Backward of kla_oracle_forward: layouts as there; every gradient output is
 * [shape of its input] in double; dfinal_lambda / dfinal_eta / dlambda0 /
 * deta0 may be NULL. Returns 0 on success. */
int kla_oracle_backward(int B, int T, int H, int dk, int dv, int iso,
                        const int *cu_seqlens, int num_seqs,
                        const float *q, const float *k, const float *v,
                        const float *a, const float *qn, const float *beta,
                        const float *lambda0, const float *eta0, const float *dout,
                        const float *dfinal_lambda, const float *dfinal_eta,
                        double *dq, double *dk_, double *dv_, double *da, double *dqn,
                        double *dbeta, double *dlambda0, double *deta0,
                        long units_begin, long units_end, int num_threads)
{
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || !dout) return 1;
    int N = cu_seqlens ? num_seqs : B;
    long units = (long)N * H;
    if (units_end < 0 || units_end > units) units_end = units;
    if (units_begin < 0) units_begin = 0;
    int err = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
#endif
    for (long u = units_begin; u < units_end; ++u) {
        int n = (int)(u / H), h = (int)(u % H);
        long t0 = cu_seqlens ? cu_seqlens[n] : (long)n * T;
        long t1 = cu_seqlens ? cu_seqlens[n + 1] : (long)(n + 1) * T;
        err |= run_unit_backward(n, h, t0, t1, H, dk, dv, iso, q, k, v, a, qn, beta, lambda0, eta0,
                                 dout, dfinal_lambda, dfinal_eta, dq, dk_, dv_, da, dqn, dbeta,
                                 dlambda0, deta0);
    }
    return err;
}
