// bwd_extras.cu -- backward pass of the fused extras (output gate, BC map, MIMO lightweight
// expansion) around the recurrence's backward.
//
// The forward with extras is the plain recurrence on effective inputs ("Technical Approach":
// output gating, BC normalisation and BC biases; "MIMO Parameterization Choices": the
// lightweight expansion):
//     X = x * w_x (per head, rank and channel),  Z = z * w_z,
//     B_h = map(B_g) = B_g s(B_g) + bias_B[h],  C_h likewise,  s(v) = 1 / sqrt(mean v^2 + eps),
//     y = y_pre * SiLU(Z),  y_pre = recurrence(X, B_h, C_h, ...) + D X.
// Its backward: dy_pre = dy Z sig(Z);  dZ = dy y_pre sig(Z) (1 + Z (1 - sig(Z)));  the
// recurrence's backward with one group per head on the effective inputs;  then
//     dx = sum_r dX w_x,  dw_x = sum_{b,t} dX x  (likewise z);
//     dB_g = J_s(sum_{h in g} dB_h),  J_s(du) = s du - (s^3 / N) v <du, v>  (identity without
//     the RMS scale);  dbias_B[h] = sum_{b,t,r} dB_h (+ the carried B_prev's share).
// This file holds the elementwise and reduction kernels of those steps; the host side
// (m3_api.cu) runs them around the forward (for y_pre) and the recurrence's backward.
#include "m3_internal.h"

namespace m3 {

namespace {

unsigned grid_for(long long n, int threads) {
    const long long b = (n + threads - 1) / threads;
    return (unsigned)(b < 148 * 32 ? (b > 0 ? b : 1) : 148 * 32);
}

// X[row][r][p] = io(x[row][p] w[h][r][p]), row = (b, t, h)
template <typename IO>
__global__ void expand_kernel(const IO* __restrict__ x, const float* __restrict__ w,
                              IO* __restrict__ X, long long rows, int H, int R, int P) {
    const long long n = rows * R * P;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int p = (int)(e % P);
        const long long rr = e / P;
        const int r = (int)(rr % R);
        const long long row = rr / R;
        const int h = (int)(row % H);
        X[e] = from_f<IO>(to_f(x[row * P + p]) * w[((size_t)h * R + r) * P + p]);
    }
}

// out[o][h][r][:] = io(v[o][g][r][:] s + bias[h][:]) for every head h of group g; one warp
// per (o, h, r) column
template <typename IO>
__global__ void bcmap_kernel(const IO* __restrict__ v, const float* __restrict__ bias, float eps,
                             IO* __restrict__ out, long long outer, int G, int H, int R, int N) {
    const long long cols = outer * H * R;
    const int lane = threadIdx.x & 31;
    for (long long col = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; col < cols;
         col += ((long long)gridDim.x * blockDim.x) >> 5) {
        const int r = (int)(col % R);
        const long long oh = col / R;
        const int h = (int)(oh % H);
        const long long o = oh / H;
        const int g = h / (H / G);
        const IO* src = v + ((o * G + g) * R + r) * N;
        float s = 1.f;
        if (eps > 0.f) {
            float ss = 0.f;
            for (int n = lane; n < N; n += 32) {
                const float f = to_f(src[n]);
                ss = fmaf(f, f, ss);
            }
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
            s = rsqrtf(ss / (float)N + eps);
        }
        IO* dst = out + col * N;
        for (int n = lane; n < N; n += 32)
            dst[n] = from_f<IO>(fmaf(to_f(src[n]), s, bias ? bias[(size_t)h * N + n] : 0.f));
    }
}

// theta of each head: out[o][h][:] = th[o][g][:]
__global__ void theta_heads_kernel(const float* __restrict__ th, float* __restrict__ out,
                                   long long outer, int G, int H, int NH) {
    const long long n = outer * H * NH;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int j = (int)(e % NH);
        const long long oh = e / NH;
        const int h = (int)(oh % H);
        const long long o = oh / H;
        out[e] = th[(o * G + h / (H / G)) * NH + j];
    }
}

// the gate: per element of y (row = (b, t, h), rank r, channel p)
//   Z = z (or io(z w_z)), sig = 1 / (1 + e^{-Z});  dy_pre = io(dy Z sig);
//   dZ = dy y_pre sig (1 + Z (1 - sig)) -> dz (no expansion) or the scratch dZ
template <typename IO>
__global__ void gate_bwd_kernel(const IO* __restrict__ dy, const IO* __restrict__ ypre,
                                const IO* __restrict__ z, const float* __restrict__ wz,
                                IO* __restrict__ dy_pre, float* __restrict__ dZ, long long rows,
                                int H, int R, int P) {
    const long long n = rows * R * P;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int p = (int)(e % P);
        const long long rr = e / P;
        const int r = (int)(rr % R);
        const long long row = rr / R;
        float Z;
        if (wz) {
            const int h = (int)(row % H);
            Z = to_f(from_f<IO>(to_f(z[row * P + p]) * wz[((size_t)h * R + r) * P + p]));
        } else {
            Z = to_f(z[e]);
        }
        const float sig = 1.f / (1.f + expf(-Z));
        const float g = to_f(dy[e]);
        dy_pre[e] = from_f<IO>(g * Z * sig);
        dZ[e] = g * to_f(ypre[e]) * sig * fmaf(Z, 1.f - sig, 1.f);
    }
}

// dx[row][p] = sum_r dX[row][r][p] w[h][r][p]
__global__ void expand_bwd_kernel(const float* __restrict__ dX, const float* __restrict__ w,
                                  float* __restrict__ dx, long long rows, int H, int R, int P) {
    const long long n = rows * P;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int p = (int)(e % P);
        const long long row = e / P;
        const int h = (int)(row % H);
        float s = 0.f;
        for (int r = 0; r < R; ++r)
            s = fmaf(dX[(row * R + r) * P + p], w[((size_t)h * R + r) * P + p], s);
        dx[e] = s;
    }
}

// dw[h][r][p] += sum over the rows (b, t) of slice blockIdx.y of dX[b,t,h,r,p] x[b,t,h,p]
template <typename IO>
__global__ void expand_wgrad_kernel(const float* __restrict__ dX, const IO* __restrict__ x,
                                    float* __restrict__ dw, long long bt, int H, int R, int P) {
    const int K = H * R * P;
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    const int p = k % P, h = k / (R * P);
    const long long r0 = bt * blockIdx.y / gridDim.y, r1 = bt * (blockIdx.y + 1) / gridDim.y;
    float s = 0.f;
    for (long long row = r0; row < r1; ++row)
        s = fmaf(dX[row * K + k], to_f(x[(row * H + h) * P + p]), s);
    atomicAdd(&dw[k], s);
}

// dbias[h][n] += sum over rows o of slice blockIdx.y and ranks r of dU[o][h][r][n]
__global__ void bias_grad_kernel(const float* __restrict__ dU, float* __restrict__ dbias,
                                 long long outer, int H, int R, int N) {
    const int K = H * N;
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    const int n = k % N, h = k / N;
    const long long r0 = outer * blockIdx.y / gridDim.y, r1 = outer * (blockIdx.y + 1) / gridDim.y;
    float s = 0.f;
    for (long long o = r0; o < r1; ++o)
        for (int r = 0; r < R; ++r) s += dU[((o * H + h) * R + r) * N + n];
    atomicAdd(&dbias[k], s);
}

// dv[o][g][r][:] = J_s(sum over the group's heads of dU[o][h][r][:]), v the raw column;
// one warp per (o, g, r)
template <typename IO>
__global__ void bcmap_bwd_kernel(const float* __restrict__ dU, const IO* __restrict__ v, float eps,
                                 float* __restrict__ dv, long long outer, int G, int H, int R,
                                 int N) {
    const long long cols = outer * G * R;
    const int lane = threadIdx.x & 31;
    const int hpg = H / G;
    for (long long col = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; col < cols;
         col += ((long long)gridDim.x * blockDim.x) >> 5) {
        const int r = (int)(col % R);
        const long long og = col / R;
        const int g = (int)(og % G);
        const long long o = og / G;
        const IO* src = v + col * N;
        float ss = 0.f, dot = 0.f;
        for (int n = lane; n < N; n += 32) {
            float du = 0.f;
            for (int j = 0; j < hpg; ++j) du += dU[((o * H + g * hpg + j) * R + r) * N + n];
            const float f = to_f(src[n]);
            ss = fmaf(f, f, ss);
            dot = fmaf(du, f, dot);
            dv[col * N + n] = du;
        }
        if (eps > 0.f) {
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) {
                ss += __shfl_xor_sync(0xffffffffu, ss, m);
                dot += __shfl_xor_sync(0xffffffffu, dot, m);
            }
            const float s = rsqrtf(ss / (float)N + eps);
            const float k3 = s * s * s / (float)N * dot;
            __syncwarp();
            for (int n = lane; n < N; n += 32)
                dv[col * N + n] = fmaf(s, dv[col * N + n], -k3 * to_f(src[n]));
        }
    }
}

template <typename IO>
cudaError_t ex_fwd_t(const ExBwdPlan& pl, cudaStream_t s) {
    const long long bt = (long long)pl.batch * pl.T;
    const int H = pl.H, G = pl.G, R = pl.R, P = pl.P, N = pl.N;
    if (pl.X) {
        const long long n = bt * H * R * P;
        expand_kernel<IO><<<grid_for(n, 256), 256, 0, s>>>(static_cast<const IO*>(pl.x), pl.x_expand,
                                                          static_cast<IO*>(pl.X), bt * H, H, R, P);
    }
    if (pl.Bh) {
        const long long cols = bt * H * R;
        bcmap_kernel<IO><<<grid_for(cols * 32, 256), 256, 0, s>>>(
            static_cast<const IO*>(pl.B), pl.B_bias, pl.eps, static_cast<IO*>(pl.Bh), bt, G, H, R, N);
        bcmap_kernel<IO><<<grid_for(cols * 32, 256), 256, 0, s>>>(
            static_cast<const IO*>(pl.C), pl.C_bias, pl.eps, static_cast<IO*>(pl.Ch), bt, G, H, R, N);
        const long long pcols = (long long)pl.batch * H * R;
        bcmap_kernel<IO><<<grid_for(pcols * 32, 256), 256, 0, s>>>(
            static_cast<const IO*>(pl.B_prev), pl.B_bias, pl.eps, static_cast<IO*>(pl.Bph),
            pl.batch, G, H, R, N);
        const long long n = bt * H * (N / 2);
        theta_heads_kernel<<<grid_for(n, 256), 256, 0, s>>>(pl.theta, pl.thh, bt, G, H, N / 2);
    }
    return cudaGetLastError();
}

template <typename IO>
cudaError_t ex_gate_t(const ExBwdPlan& pl, cudaStream_t s) {
    const long long rows = (long long)pl.batch * pl.T * pl.H;
    const long long n = rows * pl.R * pl.P;
    gate_bwd_kernel<IO><<<grid_for(n, 256), 256, 0, s>>>(
        static_cast<const IO*>(pl.dy), static_cast<const IO*>(pl.ypre), static_cast<const IO*>(pl.z),
        pl.z_expand, static_cast<IO*>(pl.dy_pre), pl.dZ, rows, pl.H, pl.R, pl.P);
    return cudaGetLastError();
}

template <typename IO>
cudaError_t ex_post_t(const ExBwdPlan& pl, cudaStream_t s) {
    const long long bt = (long long)pl.batch * pl.T;
    const int H = pl.H, G = pl.G, R = pl.R, P = pl.P, N = pl.N;
    const int slices = 64;
    if (pl.X) {
        expand_bwd_kernel<<<grid_for(bt * H * P, 256), 256, 0, s>>>(pl.dX, pl.x_expand, pl.dx, bt * H, H, R, P);
        if (pl.dx_expand) {
            const int K = H * R * P;
            expand_wgrad_kernel<IO><<<dim3((K + 255) / 256, slices), 256, 0, s>>>(
                pl.dX, static_cast<const IO*>(pl.x), pl.dx_expand, bt, H, R, P);
        }
    }
    if (pl.z && pl.z_expand) {
        expand_bwd_kernel<<<grid_for(bt * H * P, 256), 256, 0, s>>>(pl.dZ, pl.z_expand, pl.dz, bt * H, H, R, P);
        if (pl.dz_expand) {
            const int K = H * R * P;
            expand_wgrad_kernel<IO><<<dim3((K + 255) / 256, slices), 256, 0, s>>>(
                pl.dZ, static_cast<const IO*>(pl.z), pl.dz_expand, bt, H, R, P);
        }
    }
    if (pl.Bh) {
        const int K = H * N;
        if (pl.dB_bias) {
            bias_grad_kernel<<<dim3((K + 255) / 256, slices), 256, 0, s>>>(pl.dBh, pl.dB_bias, bt, H, R, N);
            bias_grad_kernel<<<dim3((K + 255) / 256, 1), 256, 0, s>>>(pl.dBph, pl.dB_bias, pl.batch, H, R, N);
        }
        if (pl.dC_bias)
            bias_grad_kernel<<<dim3((K + 255) / 256, slices), 256, 0, s>>>(pl.dCh, pl.dC_bias, bt, H, R, N);
        const long long cols = bt * G * R;
        bcmap_bwd_kernel<IO><<<grid_for(cols * 32, 256), 256, 0, s>>>(
            pl.dBh, static_cast<const IO*>(pl.B), pl.eps, pl.dB, bt, G, H, R, N);
        bcmap_bwd_kernel<IO><<<grid_for(cols * 32, 256), 256, 0, s>>>(
            pl.dCh, static_cast<const IO*>(pl.C), pl.eps, pl.dC, bt, G, H, R, N);
        const long long pcols = (long long)pl.batch * G * R;
        bcmap_bwd_kernel<IO><<<grid_for(pcols * 32, 256), 256, 0, s>>>(
            pl.dBph, static_cast<const IO*>(pl.B_prev), pl.eps, pl.dB_prev, pl.batch, G, H, R, N);
        cudaError_t e = launch_group_sum(pl.dthh, pl.dtheta, bt, G, H / G, N / 2, s);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

__global__ void status_or_kernel(uint32_t* dst, const uint32_t* src) {
    if (threadIdx.x == 0 && *src) atomicOr(dst, *src);
}

}  // namespace

cudaError_t launch_status_or(uint32_t* dst, const uint32_t* src, cudaStream_t s) {
    status_or_kernel<<<1, 32, 0, s>>>(dst, src);
    return cudaGetLastError();
}

cudaError_t launch_ex_bwd_inputs(const ExBwdPlan& pl, int io_dtype, cudaStream_t s) {
    return io_dtype == M3_BF16 ? ex_fwd_t<__nv_bfloat16>(pl, s) : ex_fwd_t<float>(pl, s);
}
cudaError_t launch_ex_bwd_gate(const ExBwdPlan& pl, int io_dtype, cudaStream_t s) {
    return io_dtype == M3_BF16 ? ex_gate_t<__nv_bfloat16>(pl, s) : ex_gate_t<float>(pl, s);
}
cudaError_t launch_ex_bwd_post(const ExBwdPlan& pl, int io_dtype, cudaStream_t s) {
    return io_dtype == M3_BF16 ? ex_post_t<__nv_bfloat16>(pl, s) : ex_post_t<float>(pl, s);
}

}  // namespace m3
