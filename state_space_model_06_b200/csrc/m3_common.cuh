// m3_common.cuh -- small device helpers shared by the CUDA kernels of the library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "m3.h"

namespace m3 {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Output gate ("Technical Approach", output gating): the readout v (skip included) times
// SiLU(z) = z / (1 + e^-z).  A large negative z gives e^-z = inf and a gate of -0.
__device__ __forceinline__ float gate_silu(float v, float z) { return v * (z / (1.f + expf(-z))); }

// One element of the BC map ("Technical Approach", BCNorm and BC biases): v * s + bias,
// with s the column's BCNorm scale (1 when off) and bias the head's channel bias (0 when off).
__device__ __forceinline__ float bc_apply(float v, float s, const float* bias, int n) {
    return fmaf(v, s, bias ? bias[n] : 0.f);
}

// MIMO lightweight expansion ("Multi-Input, Multi-Output (MIMO) Formulation", MIMO
// Parameterization Choices): one stored value v of a head channel p times the head's
// data-independent weight w[r][p] gives rank column r's value, rounded to the io dtype.
template <typename IO>
__device__ __forceinline__ float expand_io(float v, float w) { return to_f(from_f<IO>(v * w)); }

// Argument block of one decode step (device pointers, validated on the host).
struct DecodeArgs {
    const void* x;       // [b][H][R][P] io
    const void* B;       // [b][G][R][N] io
    const void* C;       // [b][G][R][N] io
    const float* dt;     // [b][H]
    const float* A;      // [b][H]
    const float* lam;    // [b][H]
    const float* theta;  // [b][G][N/2]
    const float* D;      // [H] or null
    float* h;            // [b][H][N][P]
    void* x_prev;        // [b][H][R][P] io
    const void* B_prev;  // [b][G][R][N] io (read only here; updated by a follow-up copy)
    void* y;             // [b][H][R][P] io
    const void* z;       // [b][H][R][P] io: output gate, or null for none
    const float* B_bias; // [H][N]: BC bias of B, or null
    const float* C_bias; // [H][N]: BC bias of C, or null
    float bc_eps;        // > 0: RMS-normalise B, B_prev and C columns over N (BCNorm)
    const float* x_expand;  // [H][R][P]: x is [b][H][P], X[r][p] = x[p] w[h][r][p]; or null
    const float* z_expand;  // [H][R][P]: z is [b][H][P], likewise; or null
    int H, G, P, N;
    int ppt;             // state pairs per thread
    uint32_t flags;
};

// Argument block of one prefill call.
struct ScanArgs {
    const void* x;       // [b][T][H][R][P] io
    const void* B;       // [b][T][G][R][N] io
    const void* C;       // [b][T][G][R][N] io
    const float* dt;     // [b][T][H]
    const float* A;      // [b][T][H]
    const float* lam;    // [b][T][H]
    const float* theta;  // [b][T][G][N/2]
    const float* D;      // [H] or null
    float* h;            // [b][H][N][P]   in: h0, out: h_T
    void* x_prev;        // [b][H][R][P]   in/out
    const void* B_prev;  // [b][G][R][N]   read only here; updated by a follow-up copy
    void* y;             // [b][T][H][R][P] io
    const void* z;       // [b][T][H][R][P] io: output gate, or null for none
    const float* B_bias; // [H][N]: BC bias of B, or null
    const float* C_bias; // [H][N]: BC bias of C, or null
    // BCNorm scales 1 / sqrt(mean_n v^2 + eps) (workspace; null when off), one per column:
    // B [b][G][R][Tp], then C [b][G][R][Tp], then B_prev [b][G][R] (Tp: T rounded up to 4)
    const float* bc_scale;
    bool bc;             // any BC map (bias or normalisation) is applied
    const float* x_expand;  // [H][R][P]: x is [b][T][H][P], X[r][p] = x[p] w[h][r][p]; or null
    const float* z_expand;  // [H][R][P]: z is [b][T][H][P], likewise; or null
    uint32_t* status;    // workspace status word (may be null)
    void* ws;            // workspace after the status block and the BCNorm scales
    size_t ws_bytes;     // bytes at ws (the tensor-core kernel's segment records)
    long long T;
    int batch, H, G, P, N;
    int chunk;
    int ppt, ns;         // SIMT kernel: pairs per lane, lanes per column
    uint32_t flags;
};

// Argument block of one backward call (gradients of m3_scan_fwd without extras).
struct BwdArgs {
    const void* x;       // [b][T][H][R][P] io
    const void* B;       // [b][T][G][R][N] io
    const void* C;       // [b][T][G][R][N] io
    const float* dt;     // [b][T][H]
    const float* A;      // [b][T][H]
    const float* lam;    // [b][T][H]
    const float* theta;  // [b][T][G][N/2]
    const float* D;      // [H] or null
    const float* h0;     // [b][H][N][P]   state the forward call started from
    const void* x_prev;  // [b][H][R][P] io
    const void* B_prev;  // [b][G][R][N] io
    const void* dy;      // [b][T][H][R][P] io: dL/dy
    const float* dhT;    // [b][H][N][P]: dL/dh_T, or null
    float* dx;           // [b][T][H][R][P]
    float* dB;           // [b][T][G][R][N]  (summed over the group's heads)
    float* dC;           // [b][T][G][R][N]  (likewise)
    float* ddt;          // [b][T][H]
    float* dA;           // [b][T][H]
    float* dlam;         // [b][T][H]
    float* dtheta;       // [b][T][G][N/2]   (likewise)
    float* dD;           // [H] (summed over batch and tokens) or null
    float* dh0;          // [b][H][N][P]
    float* dx_prev;      // [b][H][R][P]
    float* dB_prev;      // [b][G][R][N]     (likewise)
    // workspace
    float* ckpt;         // [b][H][nseg][N][P] states before each segment
    float* segbuf;       // [b][H][seg][N][P] recomputed states of one segment
    float* pB;           // [b][T][H][R][N] per-head shares of dB
    float* pC;           // [b][T][H][R][N] per-head shares of dC
    float* pth;          // [b][T][H][N/2]  per-head shares of dtheta
    float* pBprev;       // [b][H][R][N]    per-head shares of dB_prev
    float* pD;           // [b][H]          per-(row, head) shares of dD
    int seg, nseg;       // tokens per segment, segments
    long long T;
    int batch, H, G, P, N;
    uint32_t flags;
};

}  // namespace m3
