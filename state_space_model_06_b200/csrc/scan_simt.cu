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
// adjacent, so the readout's sum over N is a warp-shuffle reduction.  Tokens go in
// blocks of up to TB: the whole CTA stages a block's inputs in shared memory at once
// (x, B, C after the BC map, z, the rotation's cos / sin and alpha, beta, gamma per
// token), so the token loop itself reads no global memory and needs no barrier.  Slot 0
// of the block holds the previous token (the carried one, then the last of the block
// before) for the trapezoid's beta term.
#include "m3_internal.h"

namespace m3 {

// Floats of one staged token: x [R][P], B [R][N], C [R][N], z [R][P] (gate only),
// cos / sin [N/2] each, alpha / beta / gamma.
__host__ __device__ inline int simt_token_floats(int N, int P, int R, bool gate) {
    return R * P + 2 * R * N + (gate ? R * P : 0) + N + 4;
}

template <typename IO, int R, int PPTMAX>
__global__ void __launch_bounds__(1024) scan_simt_kernel(ScanArgs a, int TB) {
    extern __shared__ float sm[];
    const int N = a.N, P = a.P, H = a.H, G = a.G;
    const long long T = a.T;
    const int ppt = a.ppt, ns = a.ns;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - b * H, g = h / (H / G);
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int p = tid / ns, k = tid - p * ns;
    const bool gate = a.z != nullptr;
    const int TF = simt_token_floats(N, P, R, gate);
    // token slot layout (slot 0: the previous token; slots 1..TB: the block)
    const int oX = 0, oB = R * P, oC = oB + R * N, oZ = oC + R * N;
    const int oCS = oZ + (gate ? R * P : 0), oSN = oCS + N / 2, oSC = oSN + N / 2;
    auto slot = [&](int s) { return sm + (size_t)s * TF; };

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

    // slot 0 of the first block: the carried previous token
    {
        float* s0 = slot(0);
        const IO* xp = static_cast<const IO*>(a.x_prev) + (size_t)bh * R * P;
        const IO* bp = static_cast<const IO*>(a.B_prev) + ((size_t)b * G + g) * R * N;
        for (int e = tid; e < R * P; e += nthr) s0[oX + e] = to_f(xp[e]);
        for (int e = tid; e < R * N; e += nthr) {
            const int r = e / N;
            const float sc = sP ? sP[r] : 1.f;
            s0[oB + e] = a.bc ? bc_apply(to_f(bp[e]), sc, Bb, e - r * N) : to_f(bp[e]);
        }
    }

    const float Dh = a.D ? a.D[h] : 0.f;
    const int warp_lanes = min(32, nthr - (tid & ~31));
    const unsigned lane_mask = warp_lanes == 32 ? 0xffffffffu : ((1u << warp_lanes) - 1u);
    const float* wx = a.x_expand ? a.x_expand + (size_t)h * R * P : nullptr;
    const float* wz = a.z_expand ? a.z_expand + (size_t)h * R * P : nullptr;

    for (long long t0 = 0; t0 < T; t0 += TB) {
        const int nt = (int)(T - t0 < TB ? T - t0 : TB);
        __syncthreads();   // the previous block's tokens are done
        // ---- stage tokens t0 .. t0 + nt - 1 into slots 1 .. nt
        for (int e = tid; e < nt * R * P; e += nthr) {
            const int tt = e / (R * P), q = e - tt * (R * P);
            const size_t bt = (size_t)b * T + t0 + tt;
            float* d = slot(1 + tt);
            const IO* xt = static_cast<const IO*>(a.x) + (bt * H + h) * (wx ? 1 : R) * P;
            d[oX + q] = wx ? expand_io<IO>(to_f(xt[q % P]), wx[q]) : to_f(xt[q]);
            if (gate) {
                const IO* zt = static_cast<const IO*>(a.z);
                d[oZ + q] = wz ? expand_io<IO>(to_f(zt[(bt * H + h) * P + q % P]), wz[q])
                               : to_f(zt[(bt * H + h) * R * P + q]);
            }
        }
        for (int e = tid; e < nt * R * N; e += nthr) {
            const int tt = e / (R * N), q = e - tt * (R * N);
            const int r = q / N, n = q - r * N;
            const long long t = t0 + tt;
            const size_t bt = (size_t)b * T + t;
            float* d = slot(1 + tt);
            const float bv = to_f(static_cast<const IO*>(a.B)[(bt * G + g) * R * N + q]);
            const float cv = to_f(static_cast<const IO*>(a.C)[(bt * G + g) * R * N + q]);
            if (a.bc) {
                const size_t si = (size_t)r * Tp + t;
                d[oB + q] = bc_apply(bv, sB ? sB[si] : 1.f, Bb, n);
                d[oC + q] = bc_apply(cv, sC ? sC[si] : 1.f, Cb, n);
            } else {
                d[oB + q] = bv;
                d[oC + q] = cv;
            }
        }
        for (int e = tid; e < nt * (N / 2); e += nthr) {
            const int tt = e / (N / 2), i = e - tt * (N / 2);
            const size_t bt = (size_t)b * T + t0 + tt;
            const float dt = a.dt[bt * H + h];
            const float th = a.theta[(bt * G + g) * (N / 2) + i];
            const float phi = (a.flags & M3_FLAG_THETA_IS_ANGLE) ? th : dt * th;
            float sv, cv;
            sincosf(phi, &sv, &cv);
            float* d = slot(1 + tt);
            d[oCS + i] = cv;
            d[oSN + i] = sv;
        }
        for (int tt = tid; tt < nt; tt += nthr) {
            const size_t bt = (size_t)b * T + t0 + tt;
            const float dt = a.dt[bt * H + h];
            const float Av = a.A[bt * H + h], lam = a.lam[bt * H + h];
            const float alpha = expf(dt * Av);
            float* d = slot(1 + tt);
            d[oSC + 0] = alpha;
            d[oSC + 1] = (1.f - lam) * dt * alpha;
            d[oSC + 2] = lam * dt;
        }
        __syncthreads();

        // ---- the block's tokens: no global reads, no barrier
        for (int tt = 0; tt < nt; ++tt) {
            const float* cur = slot(1 + tt);
            const float* prv = slot(tt);
            const size_t bt = (size_t)b * T + t0 + tt;
            const float alpha = cur[oSC], beta = cur[oSC + 1], gamma = cur[oSC + 2];
            const float* xc = cur + oX;
            const float* Bc = cur + oB;
            const float* Cc = cur + oC;
            const float* xq = prv + oX;
            const float* Bq = prv + oB;
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
                    const float c = cur[oCS + i], s = cur[oSN + i];
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
                    if (gate) v = gate_silu(v, cur[oZ + r * P + p]);
                    yt[r * P + p] = from_f<IO>(v);
                }
            }
        }
        // ---- the block's last token becomes slot 0 of the next block
        __syncthreads();
        if (t0 + nt < T) {
            const float* last = slot(nt);
            float* s0 = slot(0);
            for (int e = tid; e < R * P; e += nthr) s0[oX + e] = last[oX + e];
            for (int e = tid; e < R * N; e += nthr) s0[oB + e] = last[oB + e];
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
        const IO* xl =
            static_cast<const IO*>(a.x) + (((size_t)b * T + (T - 1)) * H + h) * (wx ? 1 : R) * P;
        IO* xpo = static_cast<IO*>(a.x_prev) + (size_t)bh * R * P;
#pragma unroll
        for (int r = 0; r < R; ++r)
            xpo[r * P + p] = wx ? from_f<IO>(to_f(xl[p]) * wx[r * P + p]) : xl[r * P + p];
    }
}

// Tokens per staged block: up to 64, within 96 KB of shared memory (TB + 1 token slots).
template <typename IO, int R, int PPTMAX>
static cudaError_t launch_simt_t(const ScanArgs& a, cudaStream_t s) {
    const int threads = a.P * a.ns;
    const int tf = simt_token_floats(a.N, a.P, R, a.z != nullptr);
    int TB = (int)((96 * 1024) / (sizeof(float) * (size_t)tf)) - 1;
    if (TB > 64) TB = 64;
    if (TB < 1) TB = 1;
    const size_t smem = sizeof(float) * (size_t)tf * (TB + 1);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(scan_simt_kernel<IO, R, PPTMAX>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    scan_simt_kernel<IO, R, PPTMAX><<<(unsigned)(a.batch * a.H), threads, smem, s>>>(a, TB);
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
