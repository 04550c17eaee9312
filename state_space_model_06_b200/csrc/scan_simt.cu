// scan_simt.cu -- sequential fp32 CUDA-core prefill of the Mamba-3 recurrence.
//
// The plain recurrent form (Mamba-3 paper summary, Proposition 1 with the rotation
// of Propositions 2 and 4, MIMO rank-R input/readout), evaluated token by token in
// fp32 in the original frame.  It is the fp32-io path (tight 1e-5 parity: no
// bf16 tensor-core rounding) and the path for shapes the tensor-core kernel does
// not cover.
//
// One CTA per (batch, head).  Column p of the N x P state is independent of the
// other columns (x_t[p] only enters column p), so thread (p, k) owns column p and
// a contiguous block of `ppt` state pairs; the `ns` lanes of one column are
// adjacent, so the readout's sum over N is a warp-shuffle reduction.  Each token's
// small inputs are staged in shared memory; the previous token's stay in the other
// half of a ping-pong buffer for the trapezoid's beta term.
#include "m3_internal.h"

namespace m3 {

template <typename IO, int R, int PPTMAX>
__global__ void __launch_bounds__(1024) scan_simt_kernel(ScanArgs a) {
    extern __shared__ float sm[];
    const int N = a.N, P = a.P, H = a.H, G = a.G;
    const long long T = a.T;
    const int ppt = a.ppt, ns = a.ns;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - b * H, g = h / (H / G);
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int p = tid / ns, k = tid - p * ns;

    const int buf_floats = R * P + 2 * R * N;
    float* buf0 = sm;                      // token t even: x[R][P], B[R][N], C[R][N]
    float* buf1 = sm + buf_floats;         // token t odd
    float* cs = sm + 2 * buf_floats;       // [N/2]
    float* sn = cs + N / 2;                // [N/2]
    float* scal = sn + N / 2;              // alpha, beta, gamma

    // state column p, pairs i = k*ppt + j
    float hs[2 * PPTMAX];
    float* hbase = a.h + (size_t)bh * N * P;
#pragma unroll
    for (int j = 0; j < PPTMAX; ++j) {
        const int i = k * ppt + j;
        if (j < ppt && i < N / 2) {
            hs[2 * j] = hbase[(size_t)(2 * i) * P + p];
            hs[2 * j + 1] = hbase[(size_t)(2 * i + 1) * P + p];
        } else {
            hs[2 * j] = hs[2 * j + 1] = 0.f;
        }
    }

    // BC map (BCNorm scale per column, head bias per channel): the scales of this call's
    // columns start at sB (B), sC (C) and sP (B_prev); null scales mean 1
    const float* Bb = a.B_bias ? a.B_bias + (size_t)h * N : nullptr;
    const float* Cb = a.C_bias ? a.C_bias + (size_t)h * N : nullptr;
    const long long Tp = (T + 3) / 4 * 4;
    const size_t ncol = (size_t)a.batch * G * R * Tp;
    // this (batch, group)'s rows of scales: B [R][Tp], C [R][Tp]; B_prev [R]
    const float* sB = a.bc_scale ? a.bc_scale + ((size_t)b * G + g) * R * Tp : nullptr;
    const float* sC = a.bc_scale ? sB + ncol : nullptr;
    const float* sP = a.bc_scale ? a.bc_scale + 2 * ncol + ((size_t)b * G + g) * R : nullptr;

    // previous token of the first step comes from the carried state (buffer 1)
    {
        const IO* xp = static_cast<const IO*>(a.x_prev) + (size_t)bh * R * P;
        const IO* bp = static_cast<const IO*>(a.B_prev) + ((size_t)b * G + g) * R * N;
        for (int e = tid; e < R * P; e += nthr) buf1[e] = to_f(xp[e]);
        for (int e = tid; e < R * N; e += nthr) {
            const int r = e / N;
            const float sc = sP ? sP[r] : 1.f;
            buf1[R * P + e] = a.bc ? bc_apply(to_f(bp[e]), sc, Bb, e - r * N) : to_f(bp[e]);
        }
    }

    const float Dh = a.D ? a.D[h] : 0.f;
    const int warp_lanes = min(32, nthr - (tid & ~31));
    const unsigned lane_mask = warp_lanes == 32 ? 0xffffffffu : ((1u << warp_lanes) - 1u);

    for (long long t = 0; t < T; ++t) {
        float* cur = (t & 1) ? buf1 : buf0;
        const float* prv = (t & 1) ? buf0 : buf1;
        __syncthreads();   // token t-1 is done with `cur` (it held token t-2) and cs/sn/scal
        const size_t bt = (size_t)b * T + t;
        // x of this token: [R][P], or one value per channel expanded by the head's weights
        const float* wx = a.x_expand ? a.x_expand + (size_t)h * R * P : nullptr;
        const IO* xt = static_cast<const IO*>(a.x) + (bt * H + h) * (wx ? 1 : R) * P;
        const IO* Bt = static_cast<const IO*>(a.B) + (bt * G + g) * R * N;
        const IO* Ct = static_cast<const IO*>(a.C) + (bt * G + g) * R * N;
        const float dt = a.dt[bt * H + h];
        if (wx) {
            for (int e = tid; e < R * P; e += nthr) cur[e] = expand_io<IO>(to_f(xt[e % P]), wx[e]);
        } else {
            for (int e = tid; e < R * P; e += nthr) cur[e] = to_f(xt[e]);
        }
        if (a.bc) {
            for (int e = tid; e < R * N; e += nthr) {
                const int r = e / N, n = e - r * N;
                const size_t si = (size_t)r * Tp + t;
                cur[R * P + e] = bc_apply(to_f(Bt[e]), sB ? sB[si] : 1.f, Bb, n);
                cur[R * P + R * N + e] = bc_apply(to_f(Ct[e]), sC ? sC[si] : 1.f, Cb, n);
            }
        } else {
            for (int e = tid; e < R * N; e += nthr) {
                cur[R * P + e] = to_f(Bt[e]);
                cur[R * P + R * N + e] = to_f(Ct[e]);
            }
        }
        const float* th = a.theta + (bt * G + g) * (N / 2);
        for (int i = tid; i < N / 2; i += nthr) {
            const float phi = (a.flags & M3_FLAG_THETA_IS_ANGLE) ? th[i] : dt * th[i];
            float s, c;
            sincosf(phi, &s, &c);
            cs[i] = c;
            sn[i] = s;
        }
        if (tid == 0) {
            const float Av = a.A[bt * H + h], lam = a.lam[bt * H + h];
            const float alpha = expf(dt * Av);
            scal[0] = alpha;
            scal[1] = (1.f - lam) * dt * alpha;
            scal[2] = lam * dt;
        }
        __syncthreads();

        const float alpha = scal[0], beta = scal[1], gamma = scal[2];
        const float* xc = cur;
        const float* Bc = cur + R * P;
        const float* Cc = cur + R * P + R * N;
        const float* xq = prv;
        const float* Bq = prv + R * P;
        float yp[R];
#pragma unroll
        for (int r = 0; r < R; ++r) yp[r] = 0.f;
#pragma unroll
        for (int j = 0; j < PPTMAX; ++j) {
            const int i = k * ppt + j;
            if (j < ppt && i < N / 2) {
                float ub0 = 0.f, ub1 = 0.f, ug0 = 0.f, ug1 = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    ub0 = fmaf(Bq[r * N + 2 * i], xq[r * P + p], ub0);
                    ub1 = fmaf(Bq[r * N + 2 * i + 1], xq[r * P + p], ub1);
                    ug0 = fmaf(Bc[r * N + 2 * i], xc[r * P + p], ug0);
                    ug1 = fmaf(Bc[r * N + 2 * i + 1], xc[r * P + p], ug1);
                }
                const float m0 = fmaf(alpha, hs[2 * j], beta * ub0);
                const float m1 = fmaf(alpha, hs[2 * j + 1], beta * ub1);
                const float c = cs[i], s = sn[i];
                const float n0 = fmaf(c, m0, fmaf(-s, m1, gamma * ug0));
                const float n1 = fmaf(s, m0, fmaf(c, m1, gamma * ug1));
                hs[2 * j] = n0;
                hs[2 * j + 1] = n1;
#pragma unroll
                for (int r = 0; r < R; ++r)
                    yp[r] = fmaf(n0, Cc[r * N + 2 * i], fmaf(n1, Cc[r * N + 2 * i + 1], yp[r]));
            }
        }
        for (int off = ns >> 1; off > 0; off >>= 1)
#pragma unroll
            for (int r = 0; r < R; ++r) yp[r] += __shfl_xor_sync(lane_mask, yp[r], off);
        if (k == 0) {
            IO* yt = static_cast<IO*>(a.y) + (bt * H + h) * R * P;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float v = yp[r] + Dh * xc[r * P + p];
                if (a.z) {
                    const IO* zt = static_cast<const IO*>(a.z);
                    const float zv = a.z_expand
                        ? expand_io<IO>(to_f(zt[(bt * H + h) * P + p]), a.z_expand[((size_t)h * R + r) * P + p])
                        : to_f(zt[(bt * H + h) * R * P + r * P + p]);
                    v = gate_silu(v, zv);
                }
                yt[r * P + p] = from_f<IO>(v);
            }
        }
    }

#pragma unroll
    for (int j = 0; j < PPTMAX; ++j) {
        const int i = k * ppt + j;
        if (j < ppt && i < N / 2) {
            hbase[(size_t)(2 * i) * P + p] = hs[2 * j];
            hbase[(size_t)(2 * i + 1) * P + p] = hs[2 * j + 1];
        }
    }
    if (k == 0 && T > 0) {
        // x_prev <- X_{T-1}: the expanded value when x comes with expansion weights
        const float* wx = a.x_expand ? a.x_expand + (size_t)h * R * P : nullptr;
        const IO* xl =
            static_cast<const IO*>(a.x) + (((size_t)b * T + (T - 1)) * H + h) * (wx ? 1 : R) * P;
        IO* xpo = static_cast<IO*>(a.x_prev) + (size_t)bh * R * P;
#pragma unroll
        for (int r = 0; r < R; ++r)
            xpo[r * P + p] = wx ? from_f<IO>(to_f(xl[p]) * wx[r * P + p]) : xl[r * P + p];
    }
}

template <typename IO, int R, int PPTMAX>
static cudaError_t launch_simt_t(const ScanArgs& a, cudaStream_t s) {
    const int threads = a.P * a.ns;
    const size_t smem = sizeof(float) * (size_t)(2 * (R * a.P + 2 * R * a.N) + a.N + 4);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(scan_simt_kernel<IO, R, PPTMAX>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    scan_simt_kernel<IO, R, PPTMAX><<<(unsigned)(a.batch * a.H), threads, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename IO, int R>
static cudaError_t launch_simt_r(const ScanArgs& a, cudaStream_t s) {
    if (a.ppt <= 8) return launch_simt_t<IO, R, 8>(a, s);
    if (a.ppt <= 32) return launch_simt_t<IO, R, 32>(a, s);
    return cudaErrorNotSupported;
}

template <typename IO>
static cudaError_t launch_simt_io(const ScanArgs& a, int R, cudaStream_t s) {
    switch (R) {
        case 1: return launch_simt_r<IO, 1>(a, s);
        case 2: return launch_simt_r<IO, 2>(a, s);
        case 3: return launch_simt_r<IO, 3>(a, s);
        case 4: return launch_simt_r<IO, 4>(a, s);
        case 8: return launch_simt_r<IO, 8>(a, s);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t launch_scan_simt(const ScanArgs& a, int R, int io_dtype, cudaStream_t s) {
    if (io_dtype == M3_BF16) return launch_simt_io<__nv_bfloat16>(a, R, s);
    return launch_simt_io<float>(a, R, s);
}

}  // namespace m3
