// scan_bwd.cu -- backward pass (reverse-mode gradients) of the Mamba-3 recurrence.
//
// The forward is the exponential-trapezoidal recurrence with the data-dependent rotation
// (Mamba-3 paper summary, "Technical Approach": Proposition 1, Propositions 2 and 4) and the
// rank-R MIMO input and readout, per token:
//     M = alpha h_{t-1} + beta Bp Xp^T,  U = R(phi) M,  h_t = U + gamma B X^T,
//     Y = h_t^T C + D X.
// Its derivative, token by token in reverse with the adjoint Lam = dL/dh_t:
//     Lam += C dY^T;  dC = h_t dY^T;  dX = D dY + gamma B^T Lam (+ beta_{t+1} B^T dM_{t+1});
//     dB = gamma Lam X^T (+ beta_{t+1} dM_{t+1} X^T);  dM = R(phi)^T Lam;
//     dphi_i = sum_p (Lam_{2i+1} U_{2i} - Lam_{2i} U_{2i+1});  dalpha = <dM, h_{t-1}>;
//     dbeta = <dM, Bp Xp^T>;  dgamma = <Lam, B X^T>;  Lam <- alpha dM
// and through alpha = e^{dt A}, beta = (1 - lam) dt alpha, gamma = lam dt, phi = dt theta.
//
// One CTA per (batch, head), sequential in time, fp32.  Thread (pair i, column block cb) holds
// h_t and Lam for state rows 2i, 2i+1 and up to CPM columns in registers.  Tokens are taken in
// segments of `seg` (<= 16, by the shared-memory budget): a segment's inputs are staged in
// shared memory at once (X and B from the token before the segment, so the previous token's
// X and B need no copy; the coefficients and the rotation's cos / sin precomputed), so that
// forward steps need no barrier.  A first pass stores h before every segment (checkpoints);
// then, from the last segment, its states are recomputed into a per-head buffer (seg N P
// floats, L2-resident) and the segment is swept in reverse.  Sums over columns (dC, dB, the
// angle and the scalar terms) are shuffles across a pair's CB lanes; sums over state pairs
// (dX, and the scalars of dt, A, lam) are folded per warp and added into per-segment shared
// accumulators (shared-memory atomics: the order of the adds, and so the last bits of dX,
// ddt, dA and dlam, may vary from run to run).  B, C, theta, B_prev and D are shared across
// heads or batch rows: each head writes its own partial sums to the workspace and a second
// kernel adds them up in a fixed order.
#include "m3_internal.h"

namespace m3 {

namespace {

// ranks of 3 and more keep R-fold partial sums per pair in registers: at most 512 threads
__host__ __device__ constexpr int bwd_max_threads(int R) { return R >= 3 ? 512 : 1024; }

struct BwdShape {
    int CB, CP, NT;        // column blocks, columns per block, threads
};

// At most 8 columns per thread; down to 4 while the threads fit (more, lighter threads hide
// the per-token latency chain better).
__host__ __device__ inline BwdShape bwd_shape(int N, int P, int R) {
    BwdShape s;
    s.CB = 1;
    while ((P + s.CB - 1) / s.CB > 8) s.CB *= 2;
    while (s.CB < 16 && (P + 2 * s.CB - 1) / (2 * s.CB) >= 4 &&
           (N / 2) * 2 * s.CB <= bwd_max_threads(R))
        s.CB *= 2;
    s.CP = (P + s.CB - 1) / s.CB;
    s.NT = (N / 2) * s.CB;
    return s;
}

// shared memory floats with segments of `seg` tokens: X, B of seg + 1 tokens; dY, C,
// coefficients [8], cos, sin of seg tokens; the carried dX [R][P]; the segment's sums over
// the state pairs (B^T Lam and Bp^T dM [seg][R][P], the four scalars [seg][4]); one scratch
__host__ __device__ inline size_t bwd_smem_floats(int N, int P, int R, int seg) {
    const size_t RP = (size_t)R * P, RN = (size_t)R * N;
    return (seg + 1) * (RP + RN) + seg * (RP + RN + 8 + N) + RP + 2 * seg * RP + 4 * seg + 4;
}

// longest segment (<= 16 tokens) whose staging keeps two CTAs on an SM, else one
inline int bwd_seg(int N, int P, int R) {
    for (int budget : {100 * 1024, 227 * 1024})
        for (int seg = 16; seg >= 1; seg /= 2)
            if (sizeof(float) * bwd_smem_floats(N, P, R, seg) <= (size_t)budget) return seg;
    return 0;
}

// CPM: columns per thread the registers are sized for (4 or 8; the shape's CP <= CPM)
template <typename IO, int R, int CPM>
__global__ void __launch_bounds__(bwd_max_threads(R)) scan_bwd_kernel(BwdArgs a) {
    extern __shared__ float sm[];
    const int N = a.N, P = a.P, H = a.H, G = a.G, SEG = a.seg;
    const int RP = R * P, RN = R * N, NH = N / 2;
    const long long T = a.T;
    const BwdShape sh = bwd_shape(N, P, R);
    const int CB = sh.CB, NT = sh.NT;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - b * H, g = h / (H / G);
    const int tid = threadIdx.x;
    const int i = tid / CB, cb = tid - i * CB;          // state pair, column block
    const int n0 = 2 * i, n1 = 2 * i + 1;
    // this thread's columns: cb, cb + CB, cb + 2 CB, ... (adjacent lanes, adjacent columns)
    // lanes of this warp that exist (a pair's CB lanes never straddle a warp: CB divides 32)
    const int wlanes = min(32, NT - (tid & ~31));
    const unsigned full = wlanes == 32 ? 0xffffffffu : ((1u << wlanes) - 1u);
    const int lane = tid & 31;

    float* sX = sm;                                  // [SEG+1][R][P] tokens t0-1 .. t1-1
    float* sB = sX + (size_t)(SEG + 1) * RP;         // [SEG+1][R][N]
    float* sG = sB + (size_t)(SEG + 1) * RN;         // [SEG][R][P] dY
    float* sC = sG + (size_t)SEG * RP;               // [SEG][R][N]
    float* sK = sC + (size_t)SEG * RN;               // [SEG][8] alpha beta gamma dt A lam
    float* sCs = sK + (size_t)SEG * 8;               // [SEG][N/2] cos
    float* sSn = sCs + (size_t)SEG * NH;             // [SEG][N/2] sin
    float* cxp = sSn + (size_t)SEG * NH;             // [R][P] dX of the previous token
    float* accU = cxp + RP;                          // [SEG][R][P] sum over pairs of B^T Lam
    float* accP = accU + (size_t)SEG * RP;           // [SEG][R][P] sum over pairs of Bp^T dM
    float* accK = accP + (size_t)SEG * RP;           // [SEG][4] dalpha dbeta dgamma dphi.theta
    float* scratch = accK + (size_t)SEG * 4;

    const size_t NP = (size_t)N * P;
    float* ck = a.ckpt + (size_t)bh * a.nseg * NP;       // checkpoints: h before each segment
    float* sb = a.segbuf + (size_t)bh * SEG * NP;        // recomputed states of one segment
    const IO* xg = static_cast<const IO*>(a.x);
    const IO* Bg = static_cast<const IO*>(a.B);
    const IO* Cg = static_cast<const IO*>(a.C);
    const IO* dyg = static_cast<const IO*>(a.dy);
    const bool angle = (a.flags & M3_FLAG_THETA_IS_ANGLE) != 0;

    // stage tokens [t0, t1): X, B of t0-1 .. t1-1 (the carried state for t0 - 1 = -1);
    // with `rev` also dY and C; the coefficients and the rotation of every token
    auto stage = [&](long long t0, long long t1, bool rev) {
        const int nt = (int)(t1 - t0);
        for (int e = tid; e < (nt + 1) * RP; e += NT) {
            const int u = e / RP, k = e - u * RP;
            const long long t = t0 - 1 + u;
            sX[e] = t >= 0 ? to_f(xg[(((size_t)b * T + t) * H + h) * RP + k])
                           : to_f(static_cast<const IO*>(a.x_prev)[(size_t)bh * RP + k]);
        }
        for (int e = tid; e < (nt + 1) * RN; e += NT) {
            const int u = e / RN, k = e - u * RN;
            const long long t = t0 - 1 + u;
            sB[e] = t >= 0 ? to_f(Bg[(((size_t)b * T + t) * G + g) * RN + k])
                           : to_f(static_cast<const IO*>(a.B_prev)[((size_t)b * G + g) * RN + k]);
        }
        if (rev) {
            for (int e = tid; e < nt * RP; e += NT) {
                const int u = e / RP, k = e - u * RP;
                sG[e] = to_f(dyg[(((size_t)b * T + t0 + u) * H + h) * RP + k]);
            }
            for (int e = tid; e < nt * RN; e += NT) {
                const int u = e / RN, k = e - u * RN;
                sC[e] = to_f(Cg[(((size_t)b * T + t0 + u) * G + g) * RN + k]);
            }
        }
        for (int u = tid; u < nt; u += NT) {
            const size_t bt = (size_t)b * T + t0 + u;
            const float dt = a.dt[bt * H + h], Av = a.A[bt * H + h], lv = a.lam[bt * H + h];
            const float al = expf(dt * Av);
            float* k8 = sK + u * 8;
            k8[0] = al;
            k8[1] = (1.f - lv) * dt * al;
            k8[2] = lv * dt;
            k8[3] = dt;
            k8[4] = Av;
            k8[5] = lv;
        }
        for (int e = tid; e < nt * NH; e += NT) {
            const int u = e / NH, k = e - u * NH;
            const size_t bt = (size_t)b * T + t0 + u;
            const float th = a.theta[(bt * G + g) * NH + k];
            float s, c;
            sincosf(angle ? th : a.dt[bt * H + h] * th, &s, &c);
            sCs[e] = c;
            sSn[e] = s;
        }
    };

    float hs[2][CPM];
    // one forward step of this thread's state elements for staged token u
    auto fwd_step = [&](int u) {
        const float* k8 = sK + u * 8;
        const float al = k8[0], be = k8[1], ga = k8[2];
        const float c = sCs[u * NH + i], s = sSn[u * NH + i];
        const float* Xt = sX + (size_t)(u + 1) * RP;
        const float* Xq = sX + (size_t)u * RP;
        const float* Bt = sB + (size_t)(u + 1) * RN;
        const float* Bq = sB + (size_t)u * RN;
#pragma unroll
        for (int q = 0; q < CPM; ++q) {
            const int p = cb + q * CB;
            if (p < P) {
                float ub0 = 0.f, ub1 = 0.f, ug0 = 0.f, ug1 = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    ub0 = fmaf(Bq[r * N + n0], Xq[r * P + p], ub0);
                    ub1 = fmaf(Bq[r * N + n1], Xq[r * P + p], ub1);
                    ug0 = fmaf(Bt[r * N + n0], Xt[r * P + p], ug0);
                    ug1 = fmaf(Bt[r * N + n1], Xt[r * P + p], ug1);
                }
                const float m0 = fmaf(al, hs[0][q], be * ub0), m1 = fmaf(al, hs[1][q], be * ub1);
                hs[0][q] = fmaf(c, m0, fmaf(-s, m1, ga * ug0));
                hs[1][q] = fmaf(s, m0, fmaf(c, m1, ga * ug1));
            }
        }
    };
    auto load_state = [&](const float* src) {
#pragma unroll
        for (int q = 0; q < CPM; ++q) {
            const int p = cb + q * CB;
            if (p < P) {
                hs[0][q] = src[(size_t)n0 * P + p];
                hs[1][q] = src[(size_t)n1 * P + p];
            } else {
                hs[0][q] = hs[1][q] = 0.f;
            }
        }
    };
    auto store_state = [&](float* dst) {
#pragma unroll
        for (int q = 0; q < CPM; ++q) {
            const int p = cb + q * CB;
            if (p < P) {
                dst[(size_t)n0 * P + p] = hs[0][q];
                dst[(size_t)n1 * P + p] = hs[1][q];
            }
        }
    };

    // ---- pass 1: forward from h0, keeping h before every segment
    load_state(a.h0 + (size_t)bh * NP);
    for (int seg = 0; seg < a.nseg; ++seg) {
        const long long t0 = (long long)seg * SEG, t1 = t0 + SEG < T ? t0 + SEG : T;
        store_state(ck + (size_t)seg * NP);
        __syncthreads();            // the previous segment's steps are done with the staging
        stage(t0, t1, false);
        __syncthreads();
        for (int u = 0; u < (int)(t1 - t0); ++u) fwd_step(u);
    }

    // v summed over the state pairs this warp holds, added to *dst (shared) once per warp and
    // column; the lanes of a partial warp add their own values
    auto pair_add = [&](float* dst, float v, bool on) {
        if (wlanes == 32) {
            for (int off = CB; off < 32; off <<= 1) v += __shfl_xor_sync(full, v, off);
            if (lane < CB && on) atomicAdd(dst, v);
        } else if (on) {
            atomicAdd(dst, v);
        }
    };

    // ---- pass 2: segments in reverse; recompute their states, then sweep them backwards
    float lam_[2][CPM];
    if (a.dhT) {
        load_state(a.dhT + (size_t)bh * NP);
#pragma unroll
        for (int q = 0; q < CPM; ++q) { lam_[0][q] = hs[0][q]; lam_[1][q] = hs[1][q]; }
    } else {
#pragma unroll
        for (int q = 0; q < CPM; ++q) lam_[0][q] = lam_[1][q] = 0.f;
    }
    for (int e = tid; e < RP; e += NT) cxp[e] = 0.f;
    float carry[2][R];              // beta_{t+1} dM_{t+1} X_t^T of this pair: dB of token t
#pragma unroll
    for (int r = 0; r < R; ++r) carry[0][r] = carry[1][r] = 0.f;
    float dD_acc = 0.f;
    const float Dh = a.D ? a.D[h] : 0.f;
    for (int seg = a.nseg - 1; seg >= 0; --seg) {
        const long long t0 = (long long)seg * SEG, t1 = t0 + SEG < T ? t0 + SEG : T;
        const int nt = (int)(t1 - t0);
        __syncthreads();
        stage(t0, t1, true);
        for (int e = tid; e < 2 * nt * RP; e += NT) accU[e < nt * RP ? e : SEG * RP + e - nt * RP] = 0.f;
        for (int e = tid; e < 4 * nt; e += NT) accK[e] = 0.f;
        __syncthreads();
        load_state(ck + (size_t)seg * NP);
        for (int u = 0; u < nt; ++u) {
            fwd_step(u);
            if (u + 1 < nt) store_state(sb + (size_t)u * NP);   // h_{t0+u}: h_{t-1} of the next
        }
        // hs = h_{t1-1}
        for (int u = nt - 1; u >= 0; --u) {
            const long long t = t0 + u;
            const size_t bt = (size_t)b * T + t;
            const float* hprev = u > 0 ? sb + (size_t)(u - 1) * NP : ck + (size_t)seg * NP;
            const float* k8 = sK + u * 8;
            const float al = k8[0], be = k8[1], ga = k8[2];
            const float c = sCs[u * NH + i], s = sSn[u * NH + i];
            const float* Xt = sX + (size_t)(u + 1) * RP;
            const float* Xq = sX + (size_t)u * RP;
            const float* Bt = sB + (size_t)(u + 1) * RN;
            const float* Bq = sB + (size_t)u * RN;
            const float* Gt = sG + (size_t)u * RP;
            const float* Ct = sC + (size_t)u * RN;
            float cn[2][R], tn[2][R], sn[2][R];
#pragma unroll
            for (int r = 0; r < R; ++r) cn[0][r] = cn[1][r] = tn[0][r] = tn[1][r] = sn[0][r] = sn[1][r] = 0.f;
            float dphi = 0.f, dal = 0.f;
            float vu[R], vp[R];
            // h_{t-1} of this thread's elements, 4 columns at a time: each group's loads are
            // issued before any of them is used
            float hpv[2][4];
#pragma unroll
            for (int q = 0; q < CPM; ++q) {
                const int p = cb + q * CB;
                if (q % 4 == 0) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int pj = p + j * CB;
                        const bool in = q + j < CPM && pj < P;
                        hpv[0][j] = in ? hprev[(size_t)n0 * P + pj] : 0.f;
                        hpv[1][j] = in ? hprev[(size_t)n1 * P + pj] : 0.f;
                    }
                }
#pragma unroll
                for (int r = 0; r < R; ++r) vu[r] = vp[r] = 0.f;
                if (p < P) {
                    const float hp0 = hpv[0][q % 4], hp1 = hpv[1][q % 4];
                    float l0 = lam_[0][q], l1 = lam_[1][q];
                    float bx0 = 0.f, bx1 = 0.f;
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const float gv = Gt[r * P + p], xv = Xt[r * P + p];
                        l0 = fmaf(Ct[r * N + n0], gv, l0);
                        l1 = fmaf(Ct[r * N + n1], gv, l1);
                        cn[0][r] = fmaf(hs[0][q], gv, cn[0][r]);
                        cn[1][r] = fmaf(hs[1][q], gv, cn[1][r]);
                        bx0 = fmaf(Bt[r * N + n0], xv, bx0);
                        bx1 = fmaf(Bt[r * N + n1], xv, bx1);
                    }
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const float xv = Xt[r * P + p];
                        tn[0][r] = fmaf(l0, xv, tn[0][r]);
                        tn[1][r] = fmaf(l1, xv, tn[1][r]);
                        vu[r] = fmaf(Bt[r * N + n0], l0, Bt[r * N + n1] * l1);
                    }
                    const float u0 = fmaf(-ga, bx0, hs[0][q]), u1 = fmaf(-ga, bx1, hs[1][q]);
                    dphi = fmaf(l1, u0, fmaf(-l0, u1, dphi));
                    const float dm0 = fmaf(c, l0, s * l1), dm1 = fmaf(-s, l0, c * l1);
                    dal = fmaf(dm0, hp0, fmaf(dm1, hp1, dal));
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const float xpv = Xq[r * P + p];
                        sn[0][r] = fmaf(dm0, xpv, sn[0][r]);
                        sn[1][r] = fmaf(dm1, xpv, sn[1][r]);
                        vp[r] = fmaf(Bq[r * N + n0], dm0, Bq[r * N + n1] * dm1);
                    }
                    lam_[0][q] = al * dm0;
                    lam_[1][q] = al * dm1;
                    hs[0][q] = hp0;      // h_{t-1} is the next token's h_t
                    hs[1][q] = hp1;
                }
                // this column's sums over the pairs, for dX of t and of t - 1 (uniform code:
                // every lane of the warp takes part)
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    pair_add(accU + (size_t)u * RP + r * P + p, vu[r], p < P);
                    pair_add(accP + (size_t)u * RP + r * P + p, vp[r], p < P);
                }
            }
            // sums over this pair's column blocks
            for (int off = CB >> 1; off > 0; off >>= 1) {
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    cn[0][r] += __shfl_xor_sync(full, cn[0][r], off);
                    cn[1][r] += __shfl_xor_sync(full, cn[1][r], off);
                    tn[0][r] += __shfl_xor_sync(full, tn[0][r], off);
                    tn[1][r] += __shfl_xor_sync(full, tn[1][r], off);
                    sn[0][r] += __shfl_xor_sync(full, sn[0][r], off);
                    sn[1][r] += __shfl_xor_sync(full, sn[1][r], off);
                }
                dphi += __shfl_xor_sync(full, dphi, off);
                dal += __shfl_xor_sync(full, dal, off);
            }
            // per pair (every lane of a pair holds the pair's sums): the scalar terms
            float dga = 0.f, dbe = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                dga = fmaf(Bt[r * N + n0], tn[0][r], fmaf(Bt[r * N + n1], tn[1][r], dga));
                dbe = fmaf(Bq[r * N + n0], sn[0][r], fmaf(Bq[r * N + n1], sn[1][r], dbe));
            }
            const float th = a.theta[(bt * G + g) * NH + i];
            const float dpt = angle ? 0.f : dphi * th;
            if (cb == 0) {
                // this head's share of the group gradients of token t (and of t - 1's B)
                float* pCt = a.pC + (bt * H + h) * RN;
                float* pBt = a.pB + (bt * H + h) * RN;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    pCt[r * N + n0] = cn[0][r];
                    pCt[r * N + n1] = cn[1][r];
                    pBt[r * N + n0] = fmaf(ga, tn[0][r], carry[0][r]);
                    pBt[r * N + n1] = fmaf(ga, tn[1][r], carry[1][r]);
                    carry[0][r] = be * sn[0][r];
                    carry[1][r] = be * sn[1][r];
                }
                a.pth[(bt * H + h) * NH + i] = angle ? dphi : dphi * k8[3];
            }
            // the scalars summed over the pairs: a full warp folds its pairs, a partial warp's
            // pairs add their own
            {
                float v0 = dal, v1 = dbe, v2 = dga, v3 = dpt;
                if (wlanes == 32) {
                    for (int off = CB; off < 32; off <<= 1) {
                        v0 += __shfl_xor_sync(full, v0, off);
                        v1 += __shfl_xor_sync(full, v1, off);
                        v2 += __shfl_xor_sync(full, v2, off);
                        v3 += __shfl_xor_sync(full, v3, off);
                    }
                }
                if (wlanes == 32 ? lane == 0 : cb == 0) {
                    atomicAdd(accK + u * 4 + 0, v0);
                    atomicAdd(accK + u * 4 + 1, v1);
                    atomicAdd(accK + u * 4 + 2, v2);
                    atomicAdd(accK + u * 4 + 3, v3);
                }
            }
        }
        __syncthreads();
        // the segment's dX: D dY + gamma_t (B^T Lam)_t + beta_{t+1} (Bp^T dM)_{t+1}, the last
        // term from the next segment (cxp) for the segment's last token
        for (int e = tid; e < nt * RP; e += NT) {
            const int u = e / RP, k = e - u * RP;
            const size_t bt = (size_t)b * T + t0 + u;
            const float nxt = u + 1 < nt ? sK[(u + 1) * 8 + 1] * accP[(size_t)(u + 1) * RP + k] : cxp[k];
            const float gv = sG[(size_t)u * RP + k];
            a.dx[(bt * H + h) * RP + k] = fmaf(Dh, gv, fmaf(sK[u * 8 + 2], accU[(size_t)u * RP + k], nxt));
            dD_acc = fmaf(gv, sX[(size_t)(u + 1) * RP + k], dD_acc);
        }
        // the coefficients' gradients of the segment's tokens
        for (int u = tid; u < nt; u += NT) {
            const size_t bt = (size_t)b * T + t0 + u;
            const float* k8 = sK + u * 8;
            const float al = k8[0], dt = k8[3], Av = k8[4], lv = k8[5];
            const float v0 = accK[u * 4], v1 = accK[u * 4 + 1], v2 = accK[u * 4 + 2], v3 = accK[u * 4 + 3];
            a.ddt[bt * H + h] = v0 * al * Av + v1 * (1.f - lv) * (al + dt * al * Av) + v2 * lv + v3;
            a.dA[bt * H + h] = v0 * al * dt + v1 * (1.f - lv) * dt * al * dt;
            a.dlam[bt * H + h] = -v1 * dt * al + v2 * dt;
        }
        __syncthreads();   // every read of cxp above is done
        for (int k = tid; k < RP; k += NT) cxp[k] = sK[1] * accP[k];   // X_{t0-1}'s share
    }
    // starting state: dh0 = Lam, dx_prev = the carried dX of token 0, dB_prev = the carried
    // dB; this head's share of dD
#pragma unroll
    for (int q = 0; q < CPM; ++q) {
        const int p = cb + q * CB;
        if (p < P) {
            a.dh0[(size_t)bh * NP + (size_t)n0 * P + p] = lam_[0][q];
            a.dh0[(size_t)bh * NP + (size_t)n1 * P + p] = lam_[1][q];
        }
    }
    for (int e = tid; e < RP; e += NT) a.dx_prev[(size_t)bh * RP + e] = cxp[e];
    if (cb == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            a.pBprev[(size_t)bh * RN + r * N + n0] = carry[0][r];
            a.pBprev[(size_t)bh * RN + r * N + n1] = carry[1][r];
        }
    }
    if (tid == 0) *scratch = 0.f;
    __syncthreads();
    atomicAdd(scratch, dD_acc);
    __syncthreads();
    if (tid == 0) a.pD[bh] = *scratch;
}

// out[(o G + g) inner + k] = sum over the group's heads j of in[(o H + g hpg + j) inner + k]
__global__ void group_sum_kernel(const float* __restrict__ in, float* __restrict__ out,
                                 long long outer, int G, int hpg, int inner) {
    const long long n = outer * G * inner;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const long long o = e / ((long long)G * inner);
        const int rem = (int)(e - o * G * inner);
        const int g = rem / inner, k = rem - g * inner;
        const float* src = in + ((o * G + g) * (long long)hpg) * inner + k;
        float v = 0.f;
        for (int j = 0; j < hpg; ++j) v += src[(long long)j * inner];
        out[e] = v;
    }
}

// dD[h] = sum over batch rows of the per-(row, head) partials
__global__ void batch_sum_kernel(const float* __restrict__ in, float* __restrict__ out, int batch,
                                 int H) {
    for (int hh = blockIdx.x * blockDim.x + threadIdx.x; hh < H; hh += gridDim.x * blockDim.x) {
        float v = 0.f;
        for (int bb = 0; bb < batch; ++bb) v += in[(size_t)bb * H + hh];
        out[hh] = v;
    }
}


template <typename IO, int R, int CPM>
cudaError_t launch_bwd_c(const BwdArgs& a, cudaStream_t s) {
    const BwdShape sh = bwd_shape(a.N, a.P, R);
    const size_t smem = sizeof(float) * bwd_smem_floats(a.N, a.P, R, a.seg);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(scan_bwd_kernel<IO, R, CPM>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    scan_bwd_kernel<IO, R, CPM><<<(unsigned)(a.batch * a.H), sh.NT, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename IO, int R>
cudaError_t launch_bwd_t(const BwdArgs& a, cudaStream_t s) {
    return bwd_shape(a.N, a.P, R).CP <= 4 ? launch_bwd_c<IO, R, 4>(a, s)
                                          : launch_bwd_c<IO, R, 8>(a, s);
}

template <typename IO>
cudaError_t launch_bwd_io(const BwdArgs& a, int R, cudaStream_t s) {
    switch (R) {
        case 1: return launch_bwd_t<IO, 1>(a, s);
        case 2: return launch_bwd_t<IO, 2>(a, s);
        case 3: return launch_bwd_t<IO, 3>(a, s);
        case 4: return launch_bwd_t<IO, 4>(a, s);
        case 8: return launch_bwd_t<IO, 8>(a, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

cudaError_t launch_group_sum(const float* in, float* out, long long outer, int G, int hpg,
                             int inner, cudaStream_t s) {
    const long long n = outer * G * inner;
    if (n == 0) return cudaSuccess;
    const long long blocks = (n + 255) / 256;
    group_sum_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, s>>>(
        in, out, outer, G, hpg, inner);
    return cudaGetLastError();
}

bool scan_bwd_shape_ok(int N, int P, int R) {
    if (N < 2 || N > 256 || (N & 1) || P < 1 || P > 64) return false;
    if (R != 1 && R != 2 && R != 3 && R != 4 && R != 8) return false;
    const BwdShape sh = bwd_shape(N, P, R);
    return sh.CP <= 8 && sh.NT <= bwd_max_threads(R) && bwd_seg(N, P, R) > 0;
}

int scan_bwd_seg(int N, int P, int R) { return bwd_seg(N, P, R); }

BwdWorkspace scan_bwd_workspace(int batch, int H, int N, int P, int R, long long T) {
    BwdWorkspace w;
    const int seg = bwd_seg(N, P, R);
    w.seg = seg > 0 ? seg : 1;
    w.nseg = (int)((T + w.seg - 1) / w.seg);
    const size_t bH = (size_t)batch * H, NP = (size_t)N * P;
    size_t o = 0;
    w.ckpt = o;   o += bH * w.nseg * NP;
    w.segbuf = o; o += bH * w.seg * NP;
    w.pB = o;     o += (size_t)batch * T * H * R * N;
    w.pC = o;     o += (size_t)batch * T * H * R * N;
    w.pth = o;    o += (size_t)batch * T * H * (N / 2);
    w.pBprev = o; o += bH * R * N;
    w.pD = o;     o += bH;
    w.floats = o;
    return w;
}

cudaError_t launch_scan_bwd(const BwdArgs& a, int R, int io_dtype, cudaStream_t s) {
    cudaError_t e = io_dtype == M3_BF16 ? launch_bwd_io<__nv_bfloat16>(a, R, s)
                                        : launch_bwd_io<float>(a, R, s);
    if (e != cudaSuccess) return e;
    // group sums of the per-head partials (B, C, theta, B_prev) and the batch sum of D
    const int hpg = a.H / a.G, RN = R * a.N;
    const long long bT = (long long)a.batch * a.T;
    if ((e = launch_group_sum(a.pB, a.dB, bT, a.G, hpg, RN, s)) != cudaSuccess) return e;
    if ((e = launch_group_sum(a.pC, a.dC, bT, a.G, hpg, RN, s)) != cudaSuccess) return e;
    if ((e = launch_group_sum(a.pth, a.dtheta, bT, a.G, hpg, a.N / 2, s)) != cudaSuccess) return e;
    if ((e = launch_group_sum(a.pBprev, a.dB_prev, a.batch, a.G, hpg, RN, s)) != cudaSuccess)
        return e;
    if (a.dD) {
        batch_sum_kernel<<<1, 256, 0, s>>>(a.pD, a.dD, a.batch, a.H);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace m3
