// bcnorm.cu -- BCNorm scales of a prefill call ("Technical Approach", BC normalisation:
// each token's B and C are scaled to unit RMS after their projection).
//
// The recurrence kernels apply the BC map v * s + bias while they unpack B and C; the
// per-column scale s = 1 / sqrt(mean_n v^2 + eps) is a reduction over the N state
// channels, which the rotation warps of the tensor-core kernel hold spread over lanes and
// warps.  This prologue computes every scale of the call once (one warp per column; B and
// C are read once more, about 3 % of the call's bytes at the 1.5B-scale shapes) into the
// workspace, where the kernels read them as one float per token and rank column.
//
// Layout (floats): B scales [b][G][R][Tp], then C scales [b][G][R][Tp], then B_prev scales
// [b][G][R]; Tp = T rounded up to a multiple of 4, so that every row of tokens starts on
// 16 bytes and the tensor-core kernel can fetch a sub-chunk's scales with one TMA copy.
#include "m3_internal.h"

namespace m3 {

namespace {

template <typename IO>
__global__ void __launch_bounds__(256) bc_scale_kernel(const IO* __restrict__ B,
                                                       const IO* __restrict__ C,
                                                       const IO* __restrict__ B_prev,
                                                       long long cols, long long prev_cols, int N,
                                                       long long T, long long Tp, int GR,
                                                       float eps, float* __restrict__ out) {
    const long long total = 2 * cols + prev_cols;
    const int lane = threadIdx.x & 31;
    for (long long col = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; col < total;
         col += ((long long)gridDim.x * blockDim.x) >> 5) {
        const IO* v = col < cols ? B + col * N
                                 : (col < 2 * cols ? C + (col - cols) * N : B_prev + (col - 2 * cols) * N);
        float ss = 0.f;
        for (int n = lane; n < N; n += 32) {
            const float f = to_f(v[n]);
            ss = fmaf(f, f, ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) {
            long long o;
            if (col < 2 * cols) {
                // input column c = (b T + t) GR + gr  ->  output ((b GR + gr) Tp + t)
                const long long c = col < cols ? col : col - cols;
                const long long gr = c % GR, bt = c / GR, t = bt % T, b = bt / T;
                o = (col < cols ? 0 : cols / T * Tp) + (b * GR + gr) * Tp + t;
            } else {
                o = 2 * (cols / T) * Tp + (col - 2 * cols);
            }
            out[o] = rsqrtf(ss / (float)N + eps);
        }
    }
}

template <typename IO>
cudaError_t launch_t(const ScanArgs& a, int R, float eps, float* out, cudaStream_t s) {
    const long long cols = (long long)a.batch * a.T * a.G * R;
    const long long prev_cols = (long long)a.batch * a.G * R;
    const long long warps = 2 * cols + prev_cols;
    long long blocks = (warps + 7) / 8;
    if (blocks > 148 * 16) blocks = 148 * 16;
    bc_scale_kernel<IO><<<(unsigned)blocks, 256, 0, s>>>(
        static_cast<const IO*>(a.B), static_cast<const IO*>(a.C),
        static_cast<const IO*>(a.B_prev), cols, prev_cols, a.N, (long long)a.T,
        (long long)bc_tpad(a.T), a.G * R, eps, out);
    return cudaGetLastError();
}

}  // namespace

size_t bc_scale_floats(int batch, long long T, int G, int R) {
    return (size_t)(2 * (long long)batch * G * R * bc_tpad(T) + (long long)batch * G * R);
}

cudaError_t launch_bc_scales(const ScanArgs& a, int R, int io_dtype, float eps, float* out,
                             cudaStream_t s) {
    if (io_dtype == M3_BF16) return launch_t<__nv_bfloat16>(a, R, eps, out, s);
    return launch_t<float>(a, R, eps, out, s);
}

}  // namespace m3
