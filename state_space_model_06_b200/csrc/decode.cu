// decode.cu -- fused single-token decode step of the Mamba-3 recurrence.
//
// Mamba-3 paper summary, "Multi-Input, Multi-Output Formulation": at decode time
// the N x P state of every head is read and written once per token and dominates
// memory traffic, so the step is HBM-bound.  This kernel streams each head's fp32
// state exactly once (16-byte vector loads and stores, streaming cache hints) and
// fuses everything the step computes:
//   M   = alpha h + beta * sum_r Bp[:,r] xp[:,r]^T             (Proposition 1, beta term)
//   h'  = R(dt theta) M + gamma * sum_r B[:,r] x[:,r]^T        (Propositions 2 and 4)
//   Y   = h'^T C + D x                                          (MIMO readout, P x R)
// One CTA per (batch, head).  Thread (j, rg) owns float4 column chunk j of the
// state and `ppt` state pairs (rows 2i, 2i+1) with i = rg + k * RG, so every
// rotation is thread-local; the readout's sum over N is finished in shared memory.
// All of a thread's state loads are issued before anything else, so the pairs per thread
// set the bytes in flight per register: 8 for SISO, 4 for MIMO (whose R-fold arithmetic
// per element needs the registers and threads).
#include "m3_internal.h"

namespace m3 {

// Gate input of output element e = r * P + p of head h (bh = batch * H + h): z [b][H][R][P],
// or with the MIMO lightweight expansion z [b][H][P] times the head's weights z_expand[h][r][p].
template <typename IO>
__device__ __forceinline__ float gate_z(const DecodeArgs& a, size_t bh, int h, int R, int P, int e) {
    const IO* z = static_cast<const IO*>(a.z);
    if (a.z_expand) return expand_io<IO>(to_f(z[bh * P + e % P]), a.z_expand[(size_t)h * R * P + e]);
    return to_f(z[bh * R * P + e]);
}

// MAXP: the largest pairs-per-thread count this instantiation handles (a.ppt <= MAXP); it
// sizes the per-thread state registers, so each shape only pays for the pairs it uses.
// BCM: the instantiation with the BC map (BCNorm and BC biases) of m3_decode_step_ex.
// XE: the instantiation with the MIMO lightweight expansion of x or z (the plain ones hold
// none of its code).
template <typename IO, int R, int MAXP, bool BCM, bool XE>
__global__ void __launch_bounds__(512) decode_kernel(DecodeArgs a) {
    extern __shared__ float sm[];
    const int N = a.N, P = a.P, H = a.H, G = a.G;
    const int CPR = P / 4;                 // float4 chunks per state row
    const int RG = (N / 2) / a.ppt;        // row groups
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - b * H, g = h / (H / G);
    const int tid = threadIdx.x;
    const int j = tid % CPR, rg = tid / CPR;

    float* xs = sm;                  // [R][P]
    float* xps = xs + R * P;         // [R][P]
    float* Bs = xps + R * P;         // [R][N]
    float* Bps = Bs + R * N;         // [R][N]
    float* Cs = Bps + R * N;         // [R][N]
    float* cs = Cs + R * N;          // [N/2]
    float* sn = cs + N / 2;          // [N/2]
    float* ypart = sn + N / 2;       // [RG][R][P]
    float* bcs = ypart + RG * R * P; // [3][R] BCNorm scales of B, B_prev, C

    // 1. issue the state loads first: they are the whole cost of the step
    float4* hrow = reinterpret_cast<float4*>(a.h + (size_t)bh * N * P);
    float4 v0[MAXP], v1[MAXP];
#pragma unroll
    for (int k = 0; k < MAXP; ++k) {
        if (k < a.ppt) {
            const int i = rg + k * RG;
            v0[k] = __ldcs(hrow + (size_t)(2 * i) * CPR + j);
            v1[k] = __ldcs(hrow + (size_t)(2 * i + 1) * CPR + j);
        }
    }

    // 2. stage this token's small inputs in shared memory
    // x: [R][P], or (XE) one value per channel expanded by the head's weights [R][P]
    const float* wx = XE && a.x_expand ? a.x_expand + (size_t)h * R * P : nullptr;
    const IO* x = static_cast<const IO*>(a.x) + (size_t)bh * (XE && wx ? 1 : R) * P;
    const IO* xp = static_cast<const IO*>(a.x_prev) + (size_t)bh * R * P;
    const size_t gofs = ((size_t)b * G + g) * R * N;
    const IO* Bg = static_cast<const IO*>(a.B) + gofs;
    const IO* Bpg = static_cast<const IO*>(a.B_prev) + gofs;
    const IO* Cg = static_cast<const IO*>(a.C) + gofs;
    for (int e = tid; e < R * P; e += blockDim.x) {
        if constexpr (XE)
            xs[e] = wx ? expand_io<IO>(to_f(x[e % P]), wx[e]) : to_f(x[e]);
        else
            xs[e] = to_f(x[e]);
        xps[e] = to_f(xp[e]);
    }
    for (int e = tid; e < R * N; e += blockDim.x) {
        Bs[e] = to_f(Bg[e]);
        Bps[e] = to_f(Bpg[e]);
        Cs[e] = to_f(Cg[e]);
    }
    const float dt = a.dt[bh], Av = a.A[bh], lam = a.lam[bh];
    const float* th = a.theta + ((size_t)b * G + g) * (N / 2);
    for (int i = tid; i < N / 2; i += blockDim.x) {
        const float phi = (a.flags & M3_FLAG_THETA_IS_ANGLE) ? th[i] : dt * th[i];
        float s, c;
        sincosf(phi, &s, &c);
        cs[i] = c;
        sn[i] = s;
    }
    __syncthreads();

    // BC map ("Technical Approach", BCNorm and BC biases): each rank column of B, B_prev
    // and C scaled to unit RMS over N (when bc_eps > 0), plus the head's channel bias
    if constexpr (BCM) {
        // one thread per column (3R <= 24 columns of N <= 256): a plain serial sum
        for (int c = tid; c < 3 * R; c += blockDim.x) {      // column c: B r, B_prev r, C r
            float sc = 1.f;
            if (a.bc_eps > 0.f) {
                const float* v = (c < R ? Bs : (c < 2 * R ? Bps : Cs)) + (c % R) * N;
                float ss = 0.f;
                for (int n = 0; n < N; ++n) ss = fmaf(v[n], v[n], ss);
                sc = rsqrtf(ss / (float)N + a.bc_eps);
            }
            bcs[c] = sc;
        }
        __syncthreads();
        const float* Bb = a.B_bias ? a.B_bias + (size_t)h * N : nullptr;
        const float* Cb = a.C_bias ? a.C_bias + (size_t)h * N : nullptr;
        for (int e = tid; e < R * N; e += blockDim.x) {
            const int r = e / N, n = e - r * N;
            Bs[e] = bc_apply(Bs[e], bcs[r], Bb, n);
            Bps[e] = bc_apply(Bps[e], bcs[R + r], Bb, n);
            Cs[e] = bc_apply(Cs[e], bcs[2 * R + r], Cb, n);
        }
        __syncthreads();
    }

    const float alpha = expf(dt * Av);
    const float beta = (1.f - lam) * dt * alpha;
    const float gamma = lam * dt;

    float yp[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) yp[r][q] = 0.f;

#pragma unroll
    for (int k = 0; k < MAXP; ++k) {
        if (k < a.ppt) {
            const int i = rg + k * RG;
            const float c = cs[i], s = sn[i];
            float h0[4] = {v0[k].x, v0[k].y, v0[k].z, v0[k].w};
            float h1[4] = {v1[k].x, v1[k].y, v1[k].z, v1[k].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int p = 4 * j + q;
                float ub0 = 0.f, ub1 = 0.f, ug0 = 0.f, ug1 = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float xpv = xps[r * P + p], xv = xs[r * P + p];
                    ub0 = fmaf(Bps[r * N + 2 * i], xpv, ub0);
                    ub1 = fmaf(Bps[r * N + 2 * i + 1], xpv, ub1);
                    ug0 = fmaf(Bs[r * N + 2 * i], xv, ug0);
                    ug1 = fmaf(Bs[r * N + 2 * i + 1], xv, ug1);
                }
                const float m0 = fmaf(alpha, h0[q], beta * ub0);
                const float m1 = fmaf(alpha, h1[q], beta * ub1);
                const float n0 = fmaf(c, m0, fmaf(-s, m1, gamma * ug0));
                const float n1 = fmaf(s, m0, fmaf(c, m1, gamma * ug1));
                h0[q] = n0;
                h1[q] = n1;
#pragma unroll
                for (int r = 0; r < R; ++r)
                    yp[r][q] = fmaf(n0, Cs[r * N + 2 * i], fmaf(n1, Cs[r * N + 2 * i + 1], yp[r][q]));
            }
            __stcs(hrow + (size_t)(2 * i) * CPR + j, make_float4(h0[0], h0[1], h0[2], h0[3]));
            __stcs(hrow + (size_t)(2 * i + 1) * CPR + j, make_float4(h1[0], h1[1], h1[2], h1[3]));
        }
    }

    // 3. finish the readout's sum over N across row groups
#pragma unroll
    for (int r = 0; r < R; ++r)
        *reinterpret_cast<float4*>(ypart + ((size_t)rg * R + r) * P + 4 * j) =
            make_float4(yp[r][0], yp[r][1], yp[r][2], yp[r][3]);
    __syncthreads();
    const float Dh = a.D ? a.D[h] : 0.f;
    IO* y = static_cast<IO*>(a.y) + (size_t)bh * R * P;
    IO* xpo = static_cast<IO*>(a.x_prev) + (size_t)bh * R * P;
    for (int e = tid; e < R * P; e += blockDim.x) {
        float acc = 0.f;
        for (int k = 0; k < RG; ++k) acc += ypart[(size_t)k * R * P + e];
        float v = acc + Dh * xs[e];
        if constexpr (XE) {
            if (a.z) v = gate_silu(v, gate_z<IO>(a, bh, h, R, P, e));
            y[e] = from_f<IO>(v);
            xpo[e] = from_f<IO>(xs[e]);   // x_prev <- X (this head only; exact in the io dtype)
        } else {
            if (a.z) v = gate_silu(v, to_f(static_cast<const IO*>(a.z)[(size_t)bh * R * P + e]));
            y[e] = from_f<IO>(v);
            xpo[e] = x[e];   // x_prev <- x (this head only; read above before the barrier)
        }
    }
}

template <typename IO, int R, int MAXP, bool BCM, bool XE>
static cudaError_t launch_decode_t(const DecodeArgs& a, int batch, cudaStream_t s) {
    const int RG = (a.N / 2) / a.ppt;
    const int threads = (a.P / 4) * RG;
    const size_t smem =
        sizeof(float) * (size_t)(2 * R * a.P + 3 * R * a.N + a.N + RG * R * a.P + 3 * R);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<IO, R, MAXP, BCM, XE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    decode_kernel<IO, R, MAXP, BCM, XE><<<(unsigned)(batch * a.H), threads, smem, s>>>(a);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------
// MIMO decode with 8 state pairs per thread.  With R rank columns the per-element work is
// R times SISO's, so the update is written as one rank-2R product on packed fp32 pairs:
//   h' = R(phi)(alpha h) + [beta R(phi) Bp | gamma B] [xp | x]^T
// (the rotation is linear and moves onto Bp).  The per-head factors -- U = [beta R Bp |
// gamma B] and C stored duplicated per row, (u, u), so that they feed the FFMA2 operands
// directly, and V = [xp | x] -- are built in shared memory while the state loads are in
// flight.  Thread (j, rg) keeps 8 pairs x 4 columns of the state in registers: twice the
// 16-byte loads in flight per thread of the 4-pair kernel, at about a quarter of its
// instructions per element.

__device__ __forceinline__ float2 lo2(const float4& v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4& v) { return make_float2(v.z, v.w); }

// Row groups merged per warp by shuffles before the shared-memory reduction.
__host__ __device__ inline int mimo_wr(int cpr, int threads) {
    return (threads % 32 == 0 && 32 % cpr == 0) ? 32 / cpr : 1;
}

static size_t mimo_smem_floats(int N, int P, int R, int ppt, bool bcm) {
    const int np2 = N / 2, cpr = P / 4, rg = np2 / ppt;
    const int rgw = rg / mimo_wr(cpr, cpr * rg);
    return (size_t)np2 * 2 * R * 4 + (size_t)np2 * R * 4 + (size_t)np2 * 8 + 2 * R * P +
           (size_t)rgw * R * P + (bcm ? 3 * R * N + 3 * R : 0);
}

template <typename IO, int R, int MAXP, bool BCM, bool XE>
__global__ void __launch_bounds__(512) decode_mimo_kernel(DecodeArgs a) {
    extern __shared__ __align__(16) float sm[];
    constexpr int R2 = 2 * R;
    const int N = a.N, P = a.P, H = a.H, G = a.G, NP2 = a.N / 2, CPR = a.P / 4;
    const int RG = NP2 / a.ppt, nthr = blockDim.x;
    const int bh = blockIdx.x, b = bh / H, h = bh - b * H, g = h / (H / G);
    const int tid = threadIdx.x, j = tid % CPR, rg = tid / CPR;
    const int WR = mimo_wr(CPR, nthr), RGW = RG / WR;

    float4* U4 = reinterpret_cast<float4*>(sm);            // [N/2][2R] (u0, u0, u1, u1)
    float4* C4 = U4 + NP2 * R2;                             // [N/2][R]  (c0, c0, c1, c1)
    float4* rot4 = C4 + NP2 * R;                            // [N/2][2]  (ac, ac, as, as), (-as, -as, 0, 0)
    float* V = reinterpret_cast<float*>(rot4 + NP2 * 2);    // [2R][P]   rows xp_r, then x_r
    float* ypart = V + R2 * P;                              // [RG / WR][R][P]
    float* raw = ypart + RGW * R * P;                       // BC map: [3][R][N] B, B_prev, C
    float* bcs = raw + 3 * R * N;                           // BC map: [3R] column scales

    // 1. the state loads first: they are the whole cost of the step
    float4* hrow = reinterpret_cast<float4*>(a.h + (size_t)bh * N * P);
    float4 v0[MAXP], v1[MAXP];
#pragma unroll
    for (int k = 0; k < MAXP; ++k) {
        if (k < a.ppt) {
            const int i = rg + k * RG;
            v0[k] = __ldcs(hrow + (size_t)(2 * i) * CPR + j);
            v1[k] = __ldcs(hrow + (size_t)(2 * i + 1) * CPR + j);
        }
    }

    // 2. this token's factors, in shared memory
    const float dt = a.dt[bh], Av = a.A[bh], lam = a.lam[bh];
    const float alpha = expf(dt * Av);
    const float beta = (1.f - lam) * dt * alpha;
    const float gamma = lam * dt;
    const float* wx = XE && a.x_expand ? a.x_expand + (size_t)h * R * P : nullptr;
    const IO* x = static_cast<const IO*>(a.x) + (size_t)bh * (XE && wx ? 1 : R) * P;
    const IO* xp = static_cast<const IO*>(a.x_prev) + (size_t)bh * R * P;
    const size_t gofs = ((size_t)b * G + g) * R * N;
    const IO* Bg = static_cast<const IO*>(a.B) + gofs;
    const IO* Bpg = static_cast<const IO*>(a.B_prev) + gofs;
    const IO* Cg = static_cast<const IO*>(a.C) + gofs;
    const float* th = a.theta + ((size_t)b * G + g) * NP2;
    if constexpr (BCM) {
        // BC map ("Technical Approach", BCNorm and BC biases) on B, B_prev and C first
        for (int e = tid; e < R * N; e += nthr) {
            raw[e] = to_f(Bg[e]);
            raw[R * N + e] = to_f(Bpg[e]);
            raw[2 * R * N + e] = to_f(Cg[e]);
        }
        __syncthreads();
        for (int c = tid; c < 3 * R; c += nthr) {          // one thread per column: serial sum
            float sc = 1.f;
            if (a.bc_eps > 0.f) {
                const float* v = raw + (size_t)c * N;       // columns B r, then B_prev r, then C r
                float ss = 0.f;
                for (int n = 0; n < N; ++n) ss = fmaf(v[n], v[n], ss);
                sc = rsqrtf(ss / (float)N + a.bc_eps);
            }
            bcs[c] = sc;
        }
        __syncthreads();
        const float* Bb = a.B_bias ? a.B_bias + (size_t)h * N : nullptr;
        const float* Cb = a.C_bias ? a.C_bias + (size_t)h * N : nullptr;
        for (int e = tid; e < R * N; e += nthr) {
            const int r = e / N, n = e - r * N;
            raw[e] = bc_apply(raw[e], bcs[r], Bb, n);
            raw[R * N + e] = bc_apply(raw[R * N + e], bcs[R + r], Bb, n);
            raw[2 * R * N + e] = bc_apply(raw[2 * R * N + e], bcs[2 * R + r], Cb, n);
        }
        __syncthreads();
    }
    for (int e = tid; e < NP2 * R; e += nthr) {
        const int i = e / R, r = e - i * R;
        const float phi = (a.flags & M3_FLAG_THETA_IS_ANGLE) ? th[i] : dt * th[i];
        float sn, cs;
        sincosf(phi, &sn, &cs);
        if (r == 0) {
            const float ac = alpha * cs, as = alpha * sn;
            rot4[2 * i] = make_float4(ac, ac, as, as);
            rot4[2 * i + 1] = make_float4(-as, -as, 0.f, 0.f);
        }
        const int n0 = r * N + 2 * i;
        float p0, p1, q0, q1, c0, c1;
        if constexpr (BCM) {
            q0 = raw[n0]; q1 = raw[n0 + 1];
            p0 = raw[R * N + n0]; p1 = raw[R * N + n0 + 1];
            c0 = raw[2 * R * N + n0]; c1 = raw[2 * R * N + n0 + 1];
        } else {
            q0 = to_f(Bg[n0]); q1 = to_f(Bg[n0 + 1]);
            p0 = to_f(Bpg[n0]); p1 = to_f(Bpg[n0 + 1]);
            c0 = to_f(Cg[n0]); c1 = to_f(Cg[n0 + 1]);
        }
        const float ub0 = beta * (cs * p0 - sn * p1), ub1 = beta * (sn * p0 + cs * p1);
        const float ug0 = gamma * q0, ug1 = gamma * q1;
        U4[i * R2 + r] = make_float4(ub0, ub0, ub1, ub1);
        U4[i * R2 + R + r] = make_float4(ug0, ug0, ug1, ug1);
        C4[i * R + r] = make_float4(c0, c0, c1, c1);
    }
    for (int e = tid; e < R * P; e += nthr) {
        V[e] = to_f(xp[e]);
        if constexpr (XE)
            V[R * P + e] = wx ? expand_io<IO>(to_f(x[e % P]), wx[e]) : to_f(x[e]);
        else
            V[R * P + e] = to_f(x[e]);
    }
    __syncthreads();

    // 3. rotate + decay, rank-2R update, readout partials -- two columns per instruction
    const float4* V4 = reinterpret_cast<const float4*>(V);
    float2 ya[R], yb[R];     // readout partials of columns 4j, 4j+1 and 4j+2, 4j+3
#pragma unroll
    for (int r = 0; r < R; ++r) ya[r] = yb[r] = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < MAXP; ++k) {
        if (k < a.ppt) {
            const int i = rg + k * RG;
            const float4 rc = rot4[2 * i], rn = rot4[2 * i + 1];
            // row 2i: ac h0 - as h1;  row 2i+1: as h0 + ac h1
            float2 n0a = __ffma2_rn(lo2(rc), lo2(v0[k]), __fmul2_rn(lo2(rn), lo2(v1[k])));
            float2 n0b = __ffma2_rn(lo2(rc), hi2(v0[k]), __fmul2_rn(lo2(rn), hi2(v1[k])));
            float2 n1a = __ffma2_rn(hi2(rc), lo2(v0[k]), __fmul2_rn(lo2(rc), lo2(v1[k])));
            float2 n1b = __ffma2_rn(hi2(rc), hi2(v0[k]), __fmul2_rn(lo2(rc), hi2(v1[k])));
#pragma unroll
            for (int q = 0; q < R2; ++q) {
                const float4 u = U4[i * R2 + q];
                const float4 v = V4[q * CPR + j];
                n0a = __ffma2_rn(lo2(u), lo2(v), n0a);
                n0b = __ffma2_rn(lo2(u), hi2(v), n0b);
                n1a = __ffma2_rn(hi2(u), lo2(v), n1a);
                n1b = __ffma2_rn(hi2(u), hi2(v), n1b);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float4 c = C4[i * R + r];
                ya[r] = __ffma2_rn(n0a, lo2(c), __ffma2_rn(n1a, hi2(c), ya[r]));
                yb[r] = __ffma2_rn(n0b, lo2(c), __ffma2_rn(n1b, hi2(c), yb[r]));
            }
            __stcs(hrow + (size_t)(2 * i) * CPR + j, make_float4(n0a.x, n0a.y, n0b.x, n0b.y));
            __stcs(hrow + (size_t)(2 * i + 1) * CPR + j, make_float4(n1a.x, n1a.y, n1b.x, n1b.y));
        }
    }

    // 4. the readout's sum over N: row groups sharing a warp by shuffles, the rest through
    //    shared memory
    if (WR > 1) {
        for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
            for (int r = 0; r < R; ++r) {
                ya[r].x += __shfl_xor_sync(0xffffffffu, ya[r].x, off);
                ya[r].y += __shfl_xor_sync(0xffffffffu, ya[r].y, off);
                yb[r].x += __shfl_xor_sync(0xffffffffu, yb[r].x, off);
                yb[r].y += __shfl_xor_sync(0xffffffffu, yb[r].y, off);
            }
    }
    if (rg % WR == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r)
            *reinterpret_cast<float4*>(ypart + ((size_t)(rg / WR) * R + r) * P + 4 * j) =
                make_float4(ya[r].x, ya[r].y, yb[r].x, yb[r].y);
    }
    __syncthreads();
    const float Dh = a.D ? a.D[h] : 0.f;
    IO* y = static_cast<IO*>(a.y) + (size_t)bh * R * P;
    IO* xpo = static_cast<IO*>(a.x_prev) + (size_t)bh * R * P;
    for (int e = tid; e < R * P; e += nthr) {
        float acc = 0.f;
        for (int w = 0; w < RGW; ++w) acc += ypart[(size_t)w * R * P + e];
        float v = acc + Dh * V[R * P + e];
        if constexpr (XE) {
            if (a.z) v = gate_silu(v, gate_z<IO>(a, bh, h, R, P, e));
            y[e] = from_f<IO>(v);
            xpo[e] = from_f<IO>(V[R * P + e]);   // x_prev <- X (this head only; exact)
        } else {
            if (a.z) v = gate_silu(v, to_f(static_cast<const IO*>(a.z)[(size_t)bh * R * P + e]));
            y[e] = from_f<IO>(v);
            xpo[e] = x[e];   // x_prev <- x (this head only; read above before the barrier)
        }
    }
}

template <typename IO, int R, bool BCM, bool XE>
static cudaError_t launch_decode_mimo(const DecodeArgs& a, int batch, cudaStream_t s) {
    const int RG = (a.N / 2) / a.ppt;
    const int threads = (a.P / 4) * RG;
    const size_t smem = sizeof(float) * mimo_smem_floats(a.N, a.P, R, a.ppt, BCM);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(decode_mimo_kernel<IO, R, 8, BCM, XE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    decode_mimo_kernel<IO, R, 8, BCM, XE><<<(unsigned)(batch * a.H), threads, smem, s>>>(a);
    return cudaGetLastError();
}

// SISO: the plain kernel with 8 (or 4) pairs per thread.  MIMO: the rank-2R packed kernel
// when the shape takes 8 pairs per thread, else the plain kernel with 4.
template <typename IO, bool BCM, bool XE>
static cudaError_t launch_decode_io(const DecodeArgs& a, int batch, int R, cudaStream_t s) {
    if (a.ppt > 8) return cudaErrorNotSupported;
    if (R != 1 && a.ppt == 8) {
        switch (R) {
            case 2: return launch_decode_mimo<IO, 2, BCM, XE>(a, batch, s);
            case 3: return launch_decode_mimo<IO, 3, BCM, XE>(a, batch, s);
            case 4: return launch_decode_mimo<IO, 4, BCM, XE>(a, batch, s);
            case 8: return launch_decode_mimo<IO, 8, BCM, XE>(a, batch, s);
            default: return cudaErrorNotSupported;
        }
    }
    if (a.ppt > 4 && R != 1) return cudaErrorNotSupported;
    switch (R) {
        case 1: return a.ppt > 4 ? launch_decode_t<IO, 1, 8, BCM, XE>(a, batch, s)
                                 : launch_decode_t<IO, 1, 4, BCM, XE>(a, batch, s);
        case 2: return launch_decode_t<IO, 2, 4, BCM, XE>(a, batch, s);
        case 3: return launch_decode_t<IO, 3, 4, BCM, XE>(a, batch, s);
        case 4: return launch_decode_t<IO, 4, 4, BCM, XE>(a, batch, s);
        case 8: return launch_decode_t<IO, 8, 4, BCM, XE>(a, batch, s);
        default: return cudaErrorNotSupported;
    }
}

template <typename IO, bool BCM>
static cudaError_t launch_decode_x(const DecodeArgs& a, int batch, int R, cudaStream_t s) {
    return (a.x_expand || a.z_expand) ? launch_decode_io<IO, BCM, true>(a, batch, R, s)
                                      : launch_decode_io<IO, BCM, false>(a, batch, R, s);
}

cudaError_t launch_decode(const DecodeArgs& a, int batch, int R, int io_dtype, cudaStream_t s) {
    const bool bc = a.B_bias || a.C_bias || a.bc_eps > 0.f;
    if (io_dtype == M3_BF16)
        return bc ? launch_decode_x<__nv_bfloat16, true>(a, batch, R, s)
                  : launch_decode_x<__nv_bfloat16, false>(a, batch, R, s);
    return bc ? launch_decode_x<float, true>(a, batch, R, s)
              : launch_decode_x<float, false>(a, batch, R, s);
}

// ---------------------------------------------------------------------------------
// previous-token carry: B_prev[b] <- B[b][t], one row of row_bytes per batch entry.
template <typename U>
__global__ void copy_prev_kernel(U* __restrict__ dst, const U* __restrict__ src, long long T,
                                 long long t, int batch, long long row_units) {
    const long long total = (long long)batch * row_units;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long b = e / row_units, k = e - b * row_units;
        dst[e] = src[(b * T + t) * row_units + k];
    }
}

template <typename U>
static cudaError_t launch_copy_prev_t(void* B_prev, const void* B, long long T, long long t,
                                      int batch, size_t row_bytes, cudaStream_t s) {
    const long long row_units = (long long)(row_bytes / sizeof(U));
    const long long total = (long long)batch * row_units;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    long long blocks = (total + threads - 1) / threads;
    if (blocks > 4 * 148) blocks = 4 * 148;
    copy_prev_kernel<U><<<(unsigned)blocks, threads, 0, s>>>(
        static_cast<U*>(B_prev), static_cast<const U*>(B), T, t, batch, row_units);
    return cudaGetLastError();
}

cudaError_t launch_copy_prev(void* B_prev, const void* B, long long T, long long t, int batch,
                             size_t row_bytes, cudaStream_t s) {
    // B and B_prev are 16-byte aligned (checked by the caller); pick the widest unit
    // that divides a row.
    if (row_bytes % 16 == 0) return launch_copy_prev_t<uint4>(B_prev, B, T, t, batch, row_bytes, s);
    if (row_bytes % 4 == 0) return launch_copy_prev_t<uint32_t>(B_prev, B, T, t, batch, row_bytes, s);
    return launch_copy_prev_t<uint16_t>(B_prev, B, T, t, batch, row_bytes, s);
}

}  // namespace m3
