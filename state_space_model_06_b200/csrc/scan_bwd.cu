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
// h_t and Lam for state rows 2i, 2i+1 and up to kCP columns in registers.  The states of the
// forward are recomputed: a first pass stores h at every kSeg-th token (checkpoints); then, for
// each segment from the last, its kSeg states are recomputed into a small buffer (kSeg N P
// floats per head, L2-resident) and the segment is swept in reverse.  Sums over columns (dC,
// dB, the angle and the scalar terms) are warp shuffles across the CB lanes of a pair; sums
// over the state pairs (dX and the scalars of dt, A, lam) go through shared memory.  B, C,
// theta and B_prev are shared by the heads of a group, so their gradients are accumulated
// with fp32 atomics (order-dependent rounding only).
#include "m3_internal.h"

namespace m3 {

namespace {

constexpr int kCP = 16;    // most columns per thread
constexpr int kSeg = 16;   // tokens per checkpoint segment

struct BwdShape {
    int CB, CP, NT;        // column blocks, columns per block, threads
};

__host__ __device__ inline BwdShape bwd_shape(int N, int P) {
    BwdShape s;
    s.CB = P <= 16 ? 1 : (P <= 32 ? 2 : 4);
    s.CP = (P + s.CB - 1) / s.CB;
    s.NT = (N / 2) * s.CB;
    return s;
}

// shared memory floats: staging of one token (X, dY, Xp [R][P]; B, C, Bp [R][N]; cos, sin
// [N/2]; 8 scalars), the carried dX of the previous token [R][P], the per-pair partials of the
// pair sums ([N/2][R][P] twice) and of the scalars ([4][N/2])
__host__ __device__ inline size_t bwd_smem_floats(int N, int P, int R) {
    return (size_t)3 * R * P + 3 * R * N + N + 8 + R * P + 2 * (size_t)(N / 2) * R * P + 4 * (N / 2);
}

template <typename IO, int R>
__global__ void __launch_bounds__(512) scan_bwd_kernel(BwdArgs a) {
    extern __shared__ float sm[];
    const int N = a.N, P = a.P, H = a.H, G = a.G;
    const long long T = a.T;
    const BwdShape sh = bwd_shape(N, P);
    const int CB = sh.CB, CP = sh.CP, NT = sh.NT;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - b * H, g = h / (H / G);
    const int tid = threadIdx.x;
    const int i = tid / CB, cb = tid - i * CB;          // state pair, column block
    const int n0 = 2 * i, n1 = 2 * i + 1;
    const int c0 = cb * CP;                              // first column of this thread
    // lanes of this warp that exist (a pair's CB lanes never straddle a warp: CB divides 32)
    const int wlanes = min(32, NT - (tid & ~31));
    const unsigned full = wlanes == 32 ? 0xffffffffu : ((1u << wlanes) - 1u);

    float* sX = sm;                    // [R][P]
    float* sG = sX + R * P;            // [R][P] dY
    float* sXp = sG + R * P;           // [R][P] previous token's X
    float* sB = sXp + R * P;           // [R][N]
    float* sC = sB + R * N;            // [R][N]
    float* sBp = sC + R * N;           // [R][N] previous token's B
    float* scs = sBp + R * N;          // [N/2]
    float* ssn = scs + N / 2;          // [N/2]
    float* ssc = ssn + N / 2;          // alpha beta gamma dt A lam
    float* cxp = ssc + 8;              // [R][P] dX of the previous token (beta part)
    float* pu = cxp + R * P;           // [N/2][R][P] gamma B^T Lam partials
    float* pp = pu + (size_t)(N / 2) * R * P;   // [N/2][R][P] beta Bp^T dM partials
    float* red = pp + (size_t)(N / 2) * R * P;  // [4][N/2] dalpha dbeta dgamma sum dphi theta

    const size_t NP = (size_t)N * P;
    float* ck = a.ckpt + (size_t)bh * a.nseg * NP;       // checkpoints: h before each segment
    float* sb = a.segbuf + (size_t)bh * kSeg * NP;       // recomputed states of one segment
    const IO* xg = static_cast<const IO*>(a.x);
    const IO* Bg = static_cast<const IO*>(a.B);
    const IO* Cg = static_cast<const IO*>(a.C);
    const IO* dyg = static_cast<const IO*>(a.dy);
    const bool angle = (a.flags & M3_FLAG_THETA_IS_ANGLE) != 0;

    // stage token t (t >= 0): X, B, C (C and dY only when `rev`), the previous token's X, B
    // (the carried state at t = 0), the rotation and the coefficients
    auto stage = [&](long long t, bool rev) {
        const size_t bt = (size_t)b * T + t;
        for (int e = tid; e < R * P; e += NT) {
            sX[e] = to_f(xg[(bt * H + h) * R * P + e]);
            if (rev) sG[e] = to_f(dyg[(bt * H + h) * R * P + e]);
            sXp[e] = t > 0 ? to_f(xg[((bt - 1) * H + h) * R * P + e])
                           : to_f(static_cast<const IO*>(a.x_prev)[(size_t)bh * R * P + e]);
        }
        for (int e = tid; e < R * N; e += NT) {
            sB[e] = to_f(Bg[(bt * G + g) * R * N + e]);
            if (rev) sC[e] = to_f(Cg[(bt * G + g) * R * N + e]);
            sBp[e] = t > 0 ? to_f(Bg[((bt - 1) * G + g) * R * N + e])
                           : to_f(static_cast<const IO*>(a.B_prev)[((size_t)b * G + g) * R * N + e]);
        }
        const float dt = a.dt[bt * H + h];
        for (int k = tid; k < N / 2; k += NT) {
            const float th = a.theta[(bt * G + g) * (N / 2) + k];
            float s, c;
            sincosf(angle ? th : dt * th, &s, &c);
            scs[k] = c;
            ssn[k] = s;
        }
        if (tid == 0) {
            const float Av = a.A[bt * H + h], lv = a.lam[bt * H + h];
            const float al = expf(dt * Av);
            ssc[0] = al;
            ssc[1] = (1.f - lv) * dt * al;
            ssc[2] = lv * dt;
            ssc[3] = dt;
            ssc[4] = Av;
            ssc[5] = lv;
        }
    };

    // one forward step of this thread's state elements (staged token)
    float hs[2][kCP];
    auto fwd_step = [&]() {
        const float al = ssc[0], be = ssc[1], ga = ssc[2];
        const float c = scs[i], s = ssn[i];
#pragma unroll
        for (int q = 0; q < kCP; ++q) {
            const int p = c0 + q;
            if (q < CP && p < P) {
                float ub0 = 0.f, ub1 = 0.f, ug0 = 0.f, ug1 = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    ub0 = fmaf(sBp[r * N + n0], sXp[r * P + p], ub0);
                    ub1 = fmaf(sBp[r * N + n1], sXp[r * P + p], ub1);
                    ug0 = fmaf(sB[r * N + n0], sX[r * P + p], ug0);
                    ug1 = fmaf(sB[r * N + n1], sX[r * P + p], ug1);
                }
                const float m0 = fmaf(al, hs[0][q], be * ub0), m1 = fmaf(al, hs[1][q], be * ub1);
                hs[0][q] = fmaf(c, m0, fmaf(-s, m1, ga * ug0));
                hs[1][q] = fmaf(s, m0, fmaf(c, m1, ga * ug1));
            }
        }
    };
    auto load_state = [&](const float* src) {
#pragma unroll
        for (int q = 0; q < kCP; ++q) {
            const int p = c0 + q;
            if (q < CP && p < P) {
                hs[0][q] = src[(size_t)n0 * P + p];
                hs[1][q] = src[(size_t)n1 * P + p];
            } else {
                hs[0][q] = hs[1][q] = 0.f;
            }
        }
    };
    auto store_state = [&](float* dst) {
#pragma unroll
        for (int q = 0; q < kCP; ++q) {
            const int p = c0 + q;
            if (q < CP && p < P) {
                dst[(size_t)n0 * P + p] = hs[0][q];
                dst[(size_t)n1 * P + p] = hs[1][q];
            }
        }
    };

    // ---- pass 1: forward from h0, keeping h before every segment
    load_state(a.h0 + (size_t)bh * NP);
    for (long long t = 0; t < T; ++t) {
        if (t % kSeg == 0) store_state(ck + (size_t)(t / kSeg) * NP);
        __syncthreads();
        stage(t, false);
        __syncthreads();
        fwd_step();
    }

    // ---- pass 2: segments in reverse; recompute their states, then sweep them backwards
    float lam_[2][kCP];
    if (a.dhT) {
        load_state(a.dhT + (size_t)bh * NP);
#pragma unroll
        for (int q = 0; q < kCP; ++q) { lam_[0][q] = hs[0][q]; lam_[1][q] = hs[1][q]; }
    } else {
#pragma unroll
        for (int q = 0; q < kCP; ++q) lam_[0][q] = lam_[1][q] = 0.f;
    }
    for (int e = tid; e < R * P; e += NT) cxp[e] = 0.f;
    float dD_acc = 0.f;
    const float Dh = a.D ? a.D[h] : 0.f;
    for (int seg = a.nseg - 1; seg >= 0; --seg) {
        const long long t0 = (long long)seg * kSeg;
        const long long t1 = t0 + kSeg < T ? t0 + kSeg : T;
        load_state(ck + (size_t)seg * NP);
        for (long long t = t0; t < t1; ++t) {
            __syncthreads();
            stage(t, false);
            __syncthreads();
            fwd_step();
            store_state(sb + (size_t)(t - t0) * NP);
        }
        for (long long t = t1 - 1; t >= t0; --t) {
            // this thread's h_t (registers) and h_{t-1} (read per column below)
            load_state(sb + (size_t)(t - t0) * NP);
            const float* hprev = t > t0 ? sb + (size_t)(t - 1 - t0) * NP : ck + (size_t)seg * NP;
            __syncthreads();   // the previous token's pair sums are done with the staging
            stage(t, true);
            __syncthreads();
            const float al = ssc[0], be = ssc[1], ga = ssc[2];
            const float c = scs[i], s = ssn[i];
            float cn[2][R], tn[2][R], sn[2][R];
#pragma unroll
            for (int r = 0; r < R; ++r) cn[0][r] = cn[1][r] = tn[0][r] = tn[1][r] = sn[0][r] = sn[1][r] = 0.f;
            float dphi = 0.f, dal = 0.f;
#pragma unroll
            for (int q = 0; q < kCP; ++q) {
                const int p = c0 + q;
                if (q < CP && p < P) {
                    float l0 = lam_[0][q], l1 = lam_[1][q];
                    float bx0 = 0.f, bx1 = 0.f;
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const float gv = sG[r * P + p], xv = sX[r * P + p];
                        l0 = fmaf(sC[r * N + n0], gv, l0);
                        l1 = fmaf(sC[r * N + n1], gv, l1);
                        cn[0][r] = fmaf(hs[0][q], gv, cn[0][r]);
                        cn[1][r] = fmaf(hs[1][q], gv, cn[1][r]);
                        bx0 = fmaf(sB[r * N + n0], xv, bx0);
                        bx1 = fmaf(sB[r * N + n1], xv, bx1);
                    }
                    float* pur = pu + (size_t)i * R * P + p;
                    float* ppr = pp + (size_t)i * R * P + p;
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const float xv = sX[r * P + p];
                        tn[0][r] = fmaf(l0, xv, tn[0][r]);
                        tn[1][r] = fmaf(l1, xv, tn[1][r]);
                        pur[r * P] = fmaf(sB[r * N + n0], l0, sB[r * N + n1] * l1);
                    }
                    const float u0 = fmaf(-ga, bx0, hs[0][q]), u1 = fmaf(-ga, bx1, hs[1][q]);
                    dphi = fmaf(l1, u0, fmaf(-l0, u1, dphi));
                    const float dm0 = fmaf(c, l0, s * l1), dm1 = fmaf(-s, l0, c * l1);
                    dal = fmaf(dm0, hprev[(size_t)n0 * P + p], fmaf(dm1, hprev[(size_t)n1 * P + p], dal));
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const float xpv = sXp[r * P + p];
                        sn[0][r] = fmaf(dm0, xpv, sn[0][r]);
                        sn[1][r] = fmaf(dm1, xpv, sn[1][r]);
                        ppr[r * P] = fmaf(sBp[r * N + n0], dm0, sBp[r * N + n1] * dm1);
                    }
                    lam_[0][q] = al * dm0;
                    lam_[1][q] = al * dm1;
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
            const size_t bt = (size_t)b * T + t;
            if (cb == 0) {
                float dga = 0.f, dbe = 0.f;
                float* dCt = a.dC + (bt * G + g) * R * N;
                float* dBt = a.dB + (bt * G + g) * R * N;
                float* dBp = t > 0 ? a.dB + ((bt - 1) * G + g) * R * N : a.dB_prev + ((size_t)b * G + g) * R * N;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    dga = fmaf(sB[r * N + n0], tn[0][r], fmaf(sB[r * N + n1], tn[1][r], dga));
                    dbe = fmaf(sBp[r * N + n0], sn[0][r], fmaf(sBp[r * N + n1], sn[1][r], dbe));
                    atomicAdd(dCt + r * N + n0, cn[0][r]);
                    atomicAdd(dCt + r * N + n1, cn[1][r]);
                    atomicAdd(dBt + r * N + n0, ga * tn[0][r]);
                    atomicAdd(dBt + r * N + n1, ga * tn[1][r]);
                    atomicAdd(dBp + r * N + n0, be * sn[0][r]);
                    atomicAdd(dBp + r * N + n1, be * sn[1][r]);
                }
                const float th = a.theta[(bt * G + g) * (N / 2) + i];
                atomicAdd(a.dtheta + (bt * G + g) * (N / 2) + i, angle ? dphi : dphi * ssc[3]);
                red[i] = dal;
                red[N / 2 + i] = dbe;
                red[N + i] = dga;
                red[3 * (N / 2) + i] = angle ? 0.f : dphi * th;
            }
            __syncthreads();
            // sums over the pairs: dX of this token and the carried dX of the previous one
            float* dXt = a.dx + (bt * H + h) * R * P;
            for (int e = tid; e < R * P; e += NT) {
                float su = 0.f, spv = 0.f;
                for (int k = 0; k < N / 2; ++k) {
                    su += pu[(size_t)k * R * P + e];
                    spv += pp[(size_t)k * R * P + e];
                }
                const float gv = sG[e];
                dXt[e] = fmaf(Dh, gv, fmaf(ga, su, cxp[e]));
                dD_acc = fmaf(gv, sX[e], dD_acc);
                cxp[e] = be * spv;   // X_{t-1}'s share (read and written by this thread only)
            }
            if (tid == 0) {
                float v[4] = {0.f, 0.f, 0.f, 0.f};
                for (int k = 0; k < N / 2; ++k)
#pragma unroll
                    for (int j = 0; j < 4; ++j) v[j] += red[j * (N / 2) + k];
                const float dt = ssc[3], Av = ssc[4], lv = ssc[5];
                const float dalpha = v[0], dbeta = v[1], dgamma = v[2];
                a.ddt[bt * H + h] = dalpha * al * Av + dbeta * (1.f - lv) * (al + dt * al * Av) +
                                    dgamma * lv + v[3];
                a.dA[bt * H + h] = dalpha * al * dt + dbeta * (1.f - lv) * dt * al * dt;
                a.dlam[bt * H + h] = -dbeta * dt * al + dgamma * dt;
            }
        }
    }
    __syncthreads();
    // initial state: dh0 = Lam, dx_prev = the carried dX of token 0, dD over this row's tokens
#pragma unroll
    for (int q = 0; q < kCP; ++q) {
        const int p = c0 + q;
        if (q < CP && p < P) {
            a.dh0[(size_t)bh * NP + (size_t)n0 * P + p] = lam_[0][q];
            a.dh0[(size_t)bh * NP + (size_t)n1 * P + p] = lam_[1][q];
        }
    }
    for (int e = tid; e < R * P; e += NT) a.dx_prev[(size_t)bh * R * P + e] = cxp[e];
    if (a.D && a.dD && tid < R * P) atomicAdd(a.dD + h, dD_acc);
}

template <typename IO, int R>
cudaError_t launch_bwd_t(const BwdArgs& a, cudaStream_t s) {
    const BwdShape sh = bwd_shape(a.N, a.P);
    const size_t smem = sizeof(float) * bwd_smem_floats(a.N, a.P, R);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(scan_bwd_kernel<IO, R>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    scan_bwd_kernel<IO, R><<<(unsigned)(a.batch * a.H), sh.NT, smem, s>>>(a);
    return cudaGetLastError();
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

bool scan_bwd_shape_ok(int N, int P, int R) {
    if (N < 2 || N > 256 || (N & 1) || P < 1 || P > 64) return false;
    if (R != 1 && R != 2 && R != 3 && R != 4 && R != 8) return false;
    const BwdShape sh = bwd_shape(N, P);
    if (sh.NT > 512) return false;
    return sizeof(float) * bwd_smem_floats(N, P, R) <= 227 * 1024;
}

size_t scan_bwd_ws_floats(int batch, int H, int N, int P, long long T) {
    const long long nseg = (T + kSeg - 1) / kSeg;
    return (size_t)batch * H * (size_t)N * P * (size_t)(nseg + kSeg);
}

int scan_bwd_nseg(long long T) { return (int)((T + kSeg - 1) / kSeg); }

int scan_bwd_seg_tokens() { return kSeg; }

cudaError_t launch_scan_bwd(const BwdArgs& a, int R, int io_dtype, cudaStream_t s) {
    if (io_dtype == M3_BF16) return launch_bwd_io<__nv_bfloat16>(a, R, s);
    return launch_bwd_io<float>(a, R, s);
}

}  // namespace m3
