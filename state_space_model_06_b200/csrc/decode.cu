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


// MAXP: the largest pairs-per-thread count this instantiation handles (a.ppt <= MAXP); it
// sizes the per-thread state registers, so each shape only pays for the pairs it uses.
// BCM: the instantiation with the BC map (BCNorm and BC biases) of m3_decode_step_ex.
template <typename IO, int R, int MAXP, bool BCM>
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
    const IO* x = static_cast<const IO*>(a.x) + (size_t)bh * R * P;
    const IO* xp = static_cast<const IO*>(a.x_prev) + (size_t)bh * R * P;
    const size_t gofs = ((size_t)b * G + g) * R * N;
    const IO* Bg = static_cast<const IO*>(a.B) + gofs;
    const IO* Bpg = static_cast<const IO*>(a.B_prev) + gofs;
    const IO* Cg = static_cast<const IO*>(a.C) + gofs;
    for (int e = tid; e < R * P; e += blockDim.x) {
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
        if (a.z) v = gate_silu(v, to_f(static_cast<const IO*>(a.z)[(size_t)bh * R * P + e]));
        y[e] = from_f<IO>(v);
        xpo[e] = x[e];   // x_prev <- x (this head only; read above before the barrier)
    }
}

template <typename IO, int R, int MAXP, bool BCM>
static cudaError_t launch_decode_t(const DecodeArgs& a, int batch, cudaStream_t s) {
    const int RG = (a.N / 2) / a.ppt;
    const int threads = (a.P / 4) * RG;
    const size_t smem =
        sizeof(float) * (size_t)(2 * R * a.P + 3 * R * a.N + a.N + RG * R * a.P + 3 * R);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<IO, R, MAXP, BCM>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    decode_kernel<IO, R, MAXP, BCM><<<(unsigned)(batch * a.H), threads, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename IO, bool BCM>
static cudaError_t launch_decode_io(const DecodeArgs& a, int batch, int R, cudaStream_t s) {
    if (a.ppt > 8 || (a.ppt > 4 && R != 1)) return cudaErrorNotSupported;
    switch (R) {
        case 1: return a.ppt > 4 ? launch_decode_t<IO, 1, 8, BCM>(a, batch, s)
                                 : launch_decode_t<IO, 1, 4, BCM>(a, batch, s);
        case 2: return launch_decode_t<IO, 2, 4, BCM>(a, batch, s);
        case 3: return launch_decode_t<IO, 3, 4, BCM>(a, batch, s);
        case 4: return launch_decode_t<IO, 4, 4, BCM>(a, batch, s);
        case 8: return launch_decode_t<IO, 8, 4, BCM>(a, batch, s);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t launch_decode(const DecodeArgs& a, int batch, int R, int io_dtype, cudaStream_t s) {
    const bool bc = a.B_bias || a.C_bias || a.bc_eps > 0.f;
    if (io_dtype == M3_BF16)
        return bc ? launch_decode_io<__nv_bfloat16, true>(a, batch, R, s)
                  : launch_decode_io<__nv_bfloat16, false>(a, batch, R, s);
    return bc ? launch_decode_io<float, true>(a, batch, R, s)
              : launch_decode_io<float, false>(a, batch, R, s);
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
