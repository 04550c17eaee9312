/*
 * m3_oracle.c -- plain fp64 CPU oracle for the Mamba-3 mixer recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct reference
 * that the CUDA path is checked against.  It shares no code, header, table or
 * constant with the CUDA library, and nothing on the product path may call it:
 * only tests, the smoke check and the bench's CPU-baseline leg load it.
 *
 * What it computes (Mamba-3 paper summary, "Technical Approach" section):
 *
 *   Exponential-trapezoidal recurrence, Proposition 1:
 *       h_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1}^T + gamma_t B_t x_t^T
 *       alpha_t = exp(dt_t A_t), beta_t = (1 - lam_t) dt_t alpha_t, gamma_t = lam_t dt_t
 *
 *   Complex transition realised as a real block-diagonal rotation, Proposition 2:
 *       the transition exp(dt (A + i theta)) = alpha_t R_t, where R_t rotates each
 *       state pair [h_{2i}, h_{2i+1}] by the angle dt_t theta_t[i], with
 *       R(phi) = [[cos phi, -sin phi], [sin phi, cos phi]].
 *
 *   Complex + exponential-trapezoidal, Proposition 4, moved back from the RoPE
 *   frame to the original frame (Propositions 2 and 3): the left-endpoint
 *   trapezoid term carries the full transition, so it is rotated as well:
 *       h_t = R_t (alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1}^T) + gamma_t B_t x_t^T
 *
 *   MIMO ("Multi-Input, Multi-Output Formulation"): B_t is N x R, x_t is P x R and
 *   the input term is the rank-R sum  sum_r B_t[:,r] x_t[:,r]^T.  The readout is
 *   Y_t = H_t^T C_t (P x R), plus the per-head skip D * x_t.
 *
 *   Output gate ("Technical Approach", output gating): the readout, skip included,
 *   is multiplied element-wise by SiLU(z) = z / (1 + exp(-z)); m3o_gate applies it.
 *
 *   BC normalisation and BC biases ("Technical Approach", BCNorm and BC biases), in
 *   m3o_scan_ex: each token's B and C column (one per rank r, length N) is scaled to
 *   unit RMS, B / sqrt(mean_n B^2 + eps), then the head's bias vector (one value per
 *   state channel n, shared by the rank columns) is added.  The carried previous
 *   token's B is kept raw in the state and goes through the same map when used.
 *
 *   MIMO lightweight expansion ("Multi-Input, Multi-Output (MIMO) Formulation", MIMO
 *   Parameterization Choices), in m3o_expand: the per-head input x (and gate z) has P
 *   values per token; a learned data-independent vector w [H][R][P] scales it element-wise
 *   to the rank-R input, X[r][p] = x[p] * w[h][r][p], which then enters the recurrence
 *   (and the skip) like any MIMO input.
 *
 *   Sequence start ("Parallel representation under SSD"): the unrolling starts
 *   from h_0 = gamma_0 B_0 x_0, i.e. a fresh state has h = 0 and no previous
 *   token (x_{-1} = 0, B_{-1} = 0).  Across calls the previous token (x, B) is
 *   carried with the state so that beta_0 of the next call sees it.
 *
 * Layouts (row-major, last index contiguous), all fp64:
 *   x, y      [b][T][H][R][P]          B, C   [b][T][G][R][N]
 *   dt, A, lam[b][T][H]                theta  [b][T][G][N/2]     D [H] (may be NULL)
 *   h         [b][H][N][P]   (in: initial state, out: final state, original frame)
 *   x_prev    [b][H][R][P]   (in/out)  B_prev [b][G][R][N] (in/out)
 * Head h reads group g = h / (H / G).
 *
 * Parallelised over independent (batch, head) pairs with OpenMP only; the time
 * loop is the plain sequential recurrence.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define M3O_THETA_IS_ANGLE 1u

typedef struct {
    int32_t batch, nheads, ngroups, headdim, dstate, rank;
} m3o_dims;

/* One token of the recurrence for one head, in place on h / xp / bp. */
static void m3o_step(int N, int P, int R, double dt, double a, double lam,
                     const double* th, const double* X, const double* Bt,
                     const double* Ct, double Dh, double* h, double* xp, double* bp,
                     double* Y, unsigned flags)
{
    const double alpha = exp(dt * a);
    const double beta = (1.0 - lam) * dt * alpha;
    const double gamma = lam * dt;

    /* M = alpha h + beta * sum_r Bp[:,r] Xp[:,r]^T */
    for (int n = 0; n < N; ++n)
        for (int p = 0; p < P; ++p) {
            double v = 0.0;
            for (int r = 0; r < R; ++r) v += bp[r * N + n] * xp[r * P + p];
            h[n * P + p] = alpha * h[n * P + p] + beta * v;
        }

    /* rotate each state pair (2i, 2i+1) by phi_i = dt * theta_i */
    for (int i = 0; i < N / 2; ++i) {
        const double phi = (flags & M3O_THETA_IS_ANGLE) ? th[i] : dt * th[i];
        const double c = cos(phi), s = sin(phi);
        double* r0 = h + (2 * i) * P;
        double* r1 = h + (2 * i + 1) * P;
        for (int p = 0; p < P; ++p) {
            const double m0 = r0[p], m1 = r1[p];
            r0[p] = c * m0 - s * m1;
            r1[p] = s * m0 + c * m1;
        }
    }

    /* + gamma * sum_r B_t[:,r] X_t[:,r]^T */
    for (int n = 0; n < N; ++n)
        for (int p = 0; p < P; ++p) {
            double v = 0.0;
            for (int r = 0; r < R; ++r) v += Bt[r * N + n] * X[r * P + p];
            h[n * P + p] += gamma * v;
        }

    /* Y[r][p] = sum_n h[n][p] C_t[n][r] + D x_t[r][p] */
    for (int r = 0; r < R; ++r)
        for (int p = 0; p < P; ++p) {
            double v = 0.0;
            for (int n = 0; n < N; ++n) v += h[n * P + p] * Ct[r * N + n];
            Y[r * P + p] = v + Dh * X[r * P + p];
        }

    memcpy(xp, X, sizeof(double) * (size_t)R * P);
    memcpy(bp, Bt, sizeof(double) * (size_t)R * N);
}

/* Effective B or C column set of one head: out[r][n] = norm(in[r][:])[n] + bias[n], where
 * norm scales the column to unit RMS (eps > 0) or leaves it (eps <= 0); bias may be NULL. */
static void m3o_bc_map(int N, int R, const double* in, const double* bias, double eps,
                       double* out)
{
    for (int r = 0; r < R; ++r) {
        double scale = 1.0;
        if (eps > 0.0) {
            double ss = 0.0;
            for (int n = 0; n < N; ++n) ss += in[r * N + n] * in[r * N + n];
            scale = 1.0 / sqrt(ss / N + eps);
        }
        for (int n = 0; n < N; ++n)
            out[r * N + n] = in[r * N + n] * scale + (bias ? bias[n] : 0.0);
    }
}

static int m3o_check(const m3o_dims* d, int64_t T)
{
    if (!d) return 1;
    if (d->batch < 0 || d->nheads <= 0 || d->ngroups <= 0 || d->headdim <= 0 ||
        d->dstate <= 0 || d->rank <= 0 || T < 0)
        return 2;
    if (d->nheads % d->ngroups) return 2;
    if (d->dstate % 2) return 2;
    return 0;
}

/*
 * Run T tokens of the recurrence for every (batch, head).  The state (h, x_prev,
 * B_prev) is updated in place.  Returns 0 on success, non-zero on bad arguments.
 * nthreads <= 0 uses the OpenMP default.  B_bias / C_bias [H][N] may be NULL; bc_eps > 0
 * turns on the BC normalisation (see the header).
 */
int m3o_scan_ex(const m3o_dims* d, int64_t T, uint32_t flags, const double* x,
                const double* B, const double* C, const double* dt, const double* A,
                const double* lam, const double* theta, const double* D, const double* B_bias,
                const double* C_bias, double bc_eps, double* h, double* x_prev,
                double* B_prev, double* y, int nthreads)
{
    int rc = m3o_check(d, T);
    if (rc) return rc;
    const int Bn = d->batch, H = d->nheads, G = d->ngroups, P = d->headdim,
              N = d->dstate, R = d->rank;
    const int hpg = H / G;
    if (T == 0 || Bn == 0) return 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t bh = 0; bh < (int64_t)Bn * H; ++bh) {
        const int b = (int)(bh / H), hh = (int)(bh % H), g = hh / hpg;
        const double* bb = B_bias ? B_bias + (size_t)hh * N : NULL;
        const double* cb = C_bias ? C_bias + (size_t)hh * N : NULL;
        double* bp = (double*)malloc(sizeof(double) * (size_t)R * N);
        double* Bh = (double*)malloc(sizeof(double) * (size_t)R * N);
        double* Ch = (double*)malloc(sizeof(double) * (size_t)R * N);
        m3o_bc_map(N, R, B_prev + ((size_t)b * G + g) * R * N, bb, bc_eps, bp);
        double* xp = x_prev + ((size_t)b * H + hh) * R * P;
        double* hs = h + ((size_t)b * H + hh) * N * P;
        const double Dh = D ? D[hh] : 0.0;
        for (int64_t t = 0; t < T; ++t) {
            const size_t bt = (size_t)b * T + t;
            m3o_bc_map(N, R, B + (bt * G + g) * R * N, bb, bc_eps, Bh);
            m3o_bc_map(N, R, C + (bt * G + g) * R * N, cb, bc_eps, Ch);
            m3o_step(N, P, R, dt[bt * H + hh], A[bt * H + hh], lam[bt * H + hh],
                     theta + (bt * G + g) * (N / 2), x + (bt * H + hh) * R * P, Bh, Ch, Dh, hs,
                     xp, bp, y + (bt * H + hh) * R * P, flags);
        }
        free(bp);
        free(Bh);
        free(Ch);
    }
    /* B_prev <- B_{T-1}, once per group (every head of the group read the old value) */
    for (int b = 0; b < Bn; ++b)
        memcpy(B_prev + (size_t)b * G * R * N, B + ((size_t)b * T + (T - 1)) * G * R * N,
               sizeof(double) * (size_t)G * R * N);
    return 0;
}

int m3o_scan(const m3o_dims* d, int64_t T, uint32_t flags, const double* x,
             const double* B, const double* C, const double* dt, const double* A,
             const double* lam, const double* theta, const double* D, double* h,
             double* x_prev, double* B_prev, double* y, int nthreads)
{
    return m3o_scan_ex(d, T, flags, x, B, C, dt, A, lam, theta, D, NULL, NULL, 0.0, h, x_prev,
                       B_prev, y, nthreads);
}

/* A single decode step is the same recurrence for one token (T = 1). */
int m3o_decode(const m3o_dims* d, uint32_t flags, const double* x, const double* B,
               const double* C, const double* dt, const double* A, const double* lam,
               const double* theta, const double* D, double* h, double* x_prev,
               double* B_prev, double* y, int nthreads)
{
    return m3o_scan(d, 1, flags, x, B, C, dt, A, lam, theta, D, h, x_prev, B_prev, y,
                    nthreads);
}

/*
 * Backward pass (reverse-mode derivative) of m3o_scan for a scalar loss L whose gradients
 * with respect to the outputs are dy [b][T][H][R][P] (dL/dy) and dhT [b][H][N][P] (dL/dh_T,
 * may be NULL: zero).  The derivative is taken through the recurrence exactly as m3o_step
 * evaluates it (Proposition 1 with the rotation of Propositions 2 and 4), one token at a
 * time in reverse, with the states h_t recomputed by m3o_step itself:
 *
 *   forward, per token:  M = alpha h_{t-1} + beta Bp Xp^T;  U = R(phi) M;
 *                        h_t = U + gamma B_t X_t^T;  Y_t = h_t^T C_t + D X_t
 *   reverse, per token (Lam = dL/dh_t, starting from dhT):
 *     Lam += C_t dY_t^T;  dC_t = h_t dY_t^T;  dX_t += D dY_t;  dD += <dY_t, X_t>
 *     dgamma = <Lam, B_t X_t^T>;  dB_t += gamma Lam X_t;  dX_t += gamma B_t^T Lam
 *     dM = R(phi)^T Lam;  dphi_i = sum_p (Lam_{2i+1} U_{2i} - Lam_{2i} U_{2i+1})
 *     dalpha = <dM, h_{t-1}>;  dbeta = <dM, Bp Xp^T>;  dBp += beta dM Xp;  dXp += beta Bp^T dM
 *     Lam <- alpha dM
 *   and through alpha = exp(dt A), beta = (1 - lam) dt alpha, gamma = lam dt, phi = dt theta:
 *     ddt = dalpha alpha A + dbeta (1 - lam)(alpha + dt alpha A) + dgamma lam + sum_i dphi_i theta_i
 *     dA = dalpha alpha dt + dbeta (1 - lam) dt alpha dt,  dlam = -dbeta dt alpha + dgamma dt
 *     dtheta_i = dphi_i dt  (dphi_i with M3O_THETA_IS_ANGLE)
 *   Bp, Xp of token t are B_{t-1}, X_{t-1} (B_prev, x_prev at t = 0), so dBp / dXp add to the
 *   previous token's dB / dX, or form dB_prev / dx_prev; dh0 is the final Lam.
 *
 * B, C, theta and B_prev are shared by the heads of a group, so their gradients are sums over
 * those heads; dD sums over batch and tokens.  The gradients of the carried x_prev / B_prev
 * outputs (copies of the last token) are not inputs here: a caller chaining calls adds them
 * to dx / dB of the last token.  Outputs are overwritten.  h0, x_prev, B_prev may be NULL
 * (zeros); with D NULL there is no skip and dD is left untouched (may be NULL).
 * Parallel over batch rows (the heads of a row share its group gradients).
 */
int m3o_scan_bwd(const m3o_dims* d, int64_t T, uint32_t flags, const double* x,
                 const double* B, const double* C, const double* dt, const double* A,
                 const double* lam, const double* theta, const double* D, const double* h0,
                 const double* x_prev, const double* B_prev, const double* dy, const double* dhT,
                 double* dx, double* dB, double* dC, double* ddt, double* dA, double* dlam,
                 double* dtheta, double* dD, double* dh0, double* dx_prev, double* dB_prev,
                 int nthreads)
{
    int rc = m3o_check(d, T);
    if (rc) return rc;
    const int Bn = d->batch, H = d->nheads, G = d->ngroups, P = d->headdim, N = d->dstate,
              R = d->rank;
    const int hpg = H / G;
    memset(dx, 0, sizeof(double) * (size_t)Bn * T * H * R * P);
    memset(dB, 0, sizeof(double) * (size_t)Bn * T * G * R * N);
    memset(dC, 0, sizeof(double) * (size_t)Bn * T * G * R * N);
    memset(ddt, 0, sizeof(double) * (size_t)Bn * T * H);
    memset(dA, 0, sizeof(double) * (size_t)Bn * T * H);
    memset(dlam, 0, sizeof(double) * (size_t)Bn * T * H);
    memset(dtheta, 0, sizeof(double) * (size_t)Bn * T * G * (N / 2));
    memset(dh0, 0, sizeof(double) * (size_t)Bn * H * N * P);
    memset(dx_prev, 0, sizeof(double) * (size_t)Bn * H * R * P);
    memset(dB_prev, 0, sizeof(double) * (size_t)Bn * G * R * N);
    double* dDb = (double*)calloc((size_t)(Bn > 0 ? Bn : 1) * H, sizeof(double));
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int b = 0; b < Bn; ++b) {
        const size_t NP = (size_t)N * P;
        double* hs = (double*)malloc(sizeof(double) * (size_t)(T + 1) * NP);  /* h_{t-1}, t=0..T */
        double* xp = (double*)malloc(sizeof(double) * (size_t)R * P);
        double* bp = (double*)malloc(sizeof(double) * (size_t)R * N);
        double* Y = (double*)malloc(sizeof(double) * (size_t)R * P);
        double* Lam = (double*)malloc(sizeof(double) * NP);
        double* dM = (double*)malloc(sizeof(double) * NP);
        for (int hh = 0; hh < H; ++hh) {
            const int g = hh / hpg;
            const double Dh = D ? D[hh] : 0.0;
            /* forward, keeping every state: hs[t + 1] = h_t, hs[0] = h0 */
            if (h0) memcpy(hs, h0 + ((size_t)b * H + hh) * NP, sizeof(double) * NP);
            else memset(hs, 0, sizeof(double) * NP);
            if (x_prev) memcpy(xp, x_prev + ((size_t)b * H + hh) * R * P, sizeof(double) * R * P);
            else memset(xp, 0, sizeof(double) * R * P);
            if (B_prev) memcpy(bp, B_prev + ((size_t)b * G + g) * R * N, sizeof(double) * R * N);
            else memset(bp, 0, sizeof(double) * R * N);
            for (int64_t t = 0; t < T; ++t) {
                const size_t bt = (size_t)b * T + t;
                memcpy(hs + (t + 1) * NP, hs + t * NP, sizeof(double) * NP);
                m3o_step(N, P, R, dt[bt * H + hh], A[bt * H + hh], lam[bt * H + hh],
                         theta + (bt * G + g) * (N / 2), x + (bt * H + hh) * R * P,
                         B + (bt * G + g) * R * N, C + (bt * G + g) * R * N, Dh,
                         hs + (t + 1) * NP, xp, bp, Y, flags);
            }
            /* reverse */
            if (dhT) memcpy(Lam, dhT + ((size_t)b * H + hh) * NP, sizeof(double) * NP);
            else memset(Lam, 0, sizeof(double) * NP);
            for (int64_t t = T - 1; t >= 0; --t) {
                const size_t bt = (size_t)b * T + t;
                const double dtv = dt[bt * H + hh], av = A[bt * H + hh], lv = lam[bt * H + hh];
                const double alpha = exp(dtv * av);
                const double beta = (1.0 - lv) * dtv * alpha;
                const double gamma = lv * dtv;
                const double* X = x + (bt * H + hh) * R * P;
                const double* Bt = B + (bt * G + g) * R * N;
                const double* Ct = C + (bt * G + g) * R * N;
                const double* th = theta + (bt * G + g) * (N / 2);
                const double* dY = dy + (bt * H + hh) * R * P;
                const double* ht = hs + (t + 1) * NP;
                const double* hprev = hs + t * NP;
                const double* Xp = t > 0 ? x + ((bt - 1) * H + hh) * R * P
                                         : (x_prev ? x_prev + ((size_t)b * H + hh) * R * P : NULL);
                const double* Bp = t > 0 ? B + ((bt - 1) * G + g) * R * N
                                         : (B_prev ? B_prev + ((size_t)b * G + g) * R * N : NULL);
                double* dXt = dx + (bt * H + hh) * R * P;
                double* dBt = dB + (bt * G + g) * R * N;
                double* dCt = dC + (bt * G + g) * R * N;
                double* dBp = t > 0 ? dB + ((bt - 1) * G + g) * R * N : dB_prev + ((size_t)b * G + g) * R * N;
                double* dXpo = t > 0 ? dx + ((bt - 1) * H + hh) * R * P : dx_prev + ((size_t)b * H + hh) * R * P;

                /* readout Y = h^T C + D X */
                for (int n = 0; n < N; ++n)
                    for (int p = 0; p < P; ++p) {
                        double v = 0.0;
                        for (int r = 0; r < R; ++r) v += Ct[r * N + n] * dY[r * P + p];
                        Lam[n * P + p] += v;
                    }
                for (int r = 0; r < R; ++r)
                    for (int n = 0; n < N; ++n) {
                        double v = 0.0;
                        for (int p = 0; p < P; ++p) v += ht[n * P + p] * dY[r * P + p];
                        dCt[r * N + n] += v;
                    }
                for (int e = 0; e < R * P; ++e) {
                    dXt[e] += Dh * dY[e];
                    if (D) dDb[(size_t)b * H + hh] += dY[e] * X[e];
                }
                /* h_t = U + gamma B X^T */
                double dgamma = 0.0;
                for (int r = 0; r < R; ++r)
                    for (int n = 0; n < N; ++n) {
                        double v = 0.0;
                        for (int p = 0; p < P; ++p) v += Lam[n * P + p] * X[r * P + p];
                        dgamma += Bt[r * N + n] * v;
                        dBt[r * N + n] += gamma * v;
                    }
                for (int r = 0; r < R; ++r)
                    for (int p = 0; p < P; ++p) {
                        double v = 0.0;
                        for (int n = 0; n < N; ++n) v += Bt[r * N + n] * Lam[n * P + p];
                        dXt[r * P + p] += gamma * v;
                    }
                /* U = R(phi) M, U = h_t - gamma B X^T */
                double dphi_theta = 0.0;
                for (int i = 0; i < N / 2; ++i) {
                    const double phi = (flags & M3O_THETA_IS_ANGLE) ? th[i] : dtv * th[i];
                    const double c = cos(phi), s = sin(phi);
                    double dphi = 0.0;
                    for (int p = 0; p < P; ++p) {
                        double bx0 = 0.0, bx1 = 0.0;
                        for (int r = 0; r < R; ++r) {
                            bx0 += Bt[r * N + 2 * i] * X[r * P + p];
                            bx1 += Bt[r * N + 2 * i + 1] * X[r * P + p];
                        }
                        const double u0 = ht[(2 * i) * P + p] - gamma * bx0;
                        const double u1 = ht[(2 * i + 1) * P + p] - gamma * bx1;
                        const double l0 = Lam[(2 * i) * P + p], l1 = Lam[(2 * i + 1) * P + p];
                        dphi += l1 * u0 - l0 * u1;
                        dM[(2 * i) * P + p] = c * l0 + s * l1;
                        dM[(2 * i + 1) * P + p] = -s * l0 + c * l1;
                    }
                    if (flags & M3O_THETA_IS_ANGLE) {
                        dtheta[(bt * G + g) * (N / 2) + i] += dphi;
                    } else {
                        dtheta[(bt * G + g) * (N / 2) + i] += dphi * dtv;
                        dphi_theta += dphi * th[i];
                    }
                }
                /* M = alpha h_{t-1} + beta Bp Xp^T */
                double dalpha = 0.0, dbeta = 0.0;
                for (size_t e = 0; e < NP; ++e) dalpha += dM[e] * hprev[e];
                for (int r = 0; r < R; ++r)
                    for (int n = 0; n < N; ++n) {
                        double v = 0.0;
                        for (int p = 0; p < P; ++p) v += dM[n * P + p] * (Xp ? Xp[r * P + p] : 0.0);
                        if (Bp) dbeta += Bp[r * N + n] * v;
                        dBp[r * N + n] += beta * v;
                    }
                for (int r = 0; r < R; ++r)
                    for (int p = 0; p < P; ++p) {
                        double v = 0.0;
                        for (int n = 0; n < N; ++n) v += (Bp ? Bp[r * N + n] : 0.0) * dM[n * P + p];
                        dXpo[r * P + p] += beta * v;
                    }
                for (size_t e = 0; e < NP; ++e) Lam[e] = alpha * dM[e];
                /* coefficients */
                ddt[bt * H + hh] = dalpha * alpha * av + dbeta * (1.0 - lv) * (alpha + dtv * alpha * av) +
                                   dgamma * lv + dphi_theta;
                dA[bt * H + hh] = dalpha * alpha * dtv + dbeta * (1.0 - lv) * dtv * alpha * dtv;
                dlam[bt * H + hh] = -dbeta * dtv * alpha + dgamma * dtv;
            }
            memcpy(dh0 + ((size_t)b * H + hh) * NP, Lam, sizeof(double) * NP);
        }
        free(hs); free(xp); free(bp); free(Y); free(Lam); free(dM);
    }
    if (D && dD) {
        for (int hh = 0; hh < H; ++hh) {
            double v = 0.0;
            for (int b = 0; b < Bn; ++b) v += dDb[(size_t)b * H + hh];
            dD[hh] = v;
        }
    }
    free(dDb);
    return 0;
}

/* out[row][h][r][p] = in[row][h][p] * w[h][r][p] for rows of H heads: the lightweight
 * expansion of a per-head P-vector to the P x R MIMO input (or gate). */
void m3o_expand(int64_t rows, int H, int R, int P, const double* in, const double* w,
                double* out)
{
    for (int64_t i = 0; i < rows; ++i)
        for (int h = 0; h < H; ++h)
            for (int r = 0; r < R; ++r)
                for (int p = 0; p < P; ++p)
                    out[((i * H + h) * R + r) * P + p] =
                        in[(i * H + h) * P + p] * w[((size_t)h * R + r) * P + p];
}

/* y[i] <- y[i] * SiLU(z[i]) for n elements: the output gate on the readout (skip included). */
void m3o_gate(int64_t n, const double* z, double* y)
{
    for (int64_t i = 0; i < n; ++i) y[i] *= z[i] / (1.0 + exp(-z[i]));
}

int m3o_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
