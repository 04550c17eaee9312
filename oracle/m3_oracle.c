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
