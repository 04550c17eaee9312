// m3_internal.h -- launchers between the C ABI (m3_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>

#include "m3_common.cuh"

namespace m3 {

// Bits of the workspace status word: a bounded device-side wait that gave up ORs in the
// timeout code; the debug range scan ORs in the range bit.
constexpr uint32_t M3_STATUS_TIMEOUT_BIT = (uint32_t)M3_ERR_TIMEOUT;
constexpr uint32_t M3_STATUS_RANGE_BIT = 1u << 8;

// The inputs the debug range scan of M3_FLAG_DEBUG_CHECKS reads (null: not checked) and
// their element counts.
struct RangeCheckArgs {
    const void *x, *B, *C, *z, *x_prev, *B_prev;   // io dtype: finite
    const float *dt, *A, *lam;                     // dt > 0, A <= 0, lam in [0, 1]
    const float *theta, *D, *h;                    // finite
    size_t n_x, n_BC, n_z, n_xp, n_bp, n_coef, n_theta, n_D, n_h;
    uint32_t* status;
};
cudaError_t launch_range_checks(const RangeCheckArgs& a, int io_dtype, cudaStream_t s);

// Every host-side check m3_scan_fwd_ex makes before it launches anything, except the
// workspace checks; sets *need to the workspace bytes the call needs.
m3_status scan_validate(const m3_dims* d, int32_t seqlen, int32_t chunk, const void* x,
                        const void* B, const void* C, const float* dt, const float* A,
                        const float* lam, const float* theta, const float* D,
                        const m3_extras* ex, const m3_state* state, const void* y,
                        uint32_t flags, size_t* need);

// decode step: one CTA per (batch, head); template on io type and rank
cudaError_t launch_decode(const DecodeArgs& a, int batch, int R, int io_dtype, cudaStream_t s);

// Decode step as a persistent streaming kernel (MIMO N = P = 64, rank 2 or 4, every fused
// part; SISO N = 128, P = 64 as half-heads, plain or gated): each warp streams heads or
// half-heads through a bulk-copied shared-memory slot
bool decode_stream_ok(const DecodeArgs& a, int R);
cudaError_t launch_decode_stream(const DecodeArgs& a, int batch, int R, int io_dtype,
                                 cudaStream_t s);

// sequential fp32 CUDA-core prefill: one CTA per (batch, head)
cudaError_t launch_scan_simt(const ScanArgs& a, int R, int io_dtype, cudaStream_t s);

// tcgen05 chunked prefill (bf16 io).  Returns cudaErrorNotSupported for shapes
// the kernel does not cover (the caller then reports M3_ERR_UNSUPPORTED or
// falls back to the SIMT kernel).
int scan_tc_chunk(int N, int P, int R, int chunk, int H);   // tile chunk, 0 = none
size_t scan_tc_workspace_bytes(int batch, int H, int N, int P, int R, long long T, int chunk);
// sequence segments per (batch, head) the tensor-core prefill uses for nch chunks over BH
// (batch * head) streams, given the workspace for their records
int scan_tc_segments(int BH, long long nch);
cudaError_t launch_scan_tc(const ScanArgs& a, int R, cudaStream_t s);

// BCNorm scales of every B, C and B_prev column of a prefill call into a.bc_scale
// (floats: B [b][G][R][Tp], C [b][G][R][Tp], then B_prev [b][G][R]; Tp = bc_tpad(T)).
__host__ __device__ inline long long bc_tpad(long long T) { return (T + 3) / 4 * 4; }
size_t bc_scale_floats(int batch, long long T, int G, int R);
cudaError_t launch_bc_scales(const ScanArgs& a, int R, int io_dtype, float eps, float* out,
                             cudaStream_t s);

// backward pass (sequential fp32, one CTA per (batch, head)): the shapes it covers and its
// workspace plan (float offsets of the checkpoints, the segment buffer and the per-head
// partial sums), then the kernels (the pass itself and the group / batch sums)
struct BwdWorkspace {
    int seg, nseg;
    size_t ckpt, segbuf, pB, pC, pth, pBprev, pD, floats;
};
bool scan_bwd_shape_ok(int N, int P, int R);
BwdWorkspace scan_bwd_workspace(int batch, int H, int N, int P, int R, long long T);
cudaError_t launch_scan_bwd(const BwdArgs& a, int R, int io_dtype, cudaStream_t s);

// chunked backward on the tensor cores (SISO, bf16 io, P 64, N 64 / 128): the shapes it
// covers, its workspace bytes (after the status block) and the launch (four kernels; dB, dC,
// dtheta, dB_prev and dD are accumulated with atomics and must be zero on entry)
bool scan_bwd_tc_ok(int io_dtype, int N, int P, int R);
size_t scan_bwd_tc_workspace_bytes(int batch, int H, int N, int R, long long T);
cudaError_t launch_scan_bwd_tc(const BwdArgs& a, int R, void* ws, uint32_t* status,
                               unsigned long long limit_ns, cudaStream_t s);

// sum of per-head partials over the heads of each group (fixed order):
// out[(o G + g) inner + k] = sum_j in[(o H + g hpg + j) inner + k]
cudaError_t launch_group_sum(const float* in, float* out, long long outer, int G, int hpg,
                             int inner, cudaStream_t s);

// backward of the fused extras: the pointers of one call (null where a part is off)
struct ExBwdPlan {
    int batch, H, G, R, P, N;
    long long T;
    float eps;
    // the call's inputs
    const void* x;
    const void* B;
    const void* C;
    const void* B_prev;
    const float* theta;
    const void* z;
    const float* B_bias;
    const float* C_bias;
    const float* x_expand;
    const float* z_expand;
    const void* dy;
    // effective inputs (workspace): expanded x, per-head mapped B / C / B_prev and theta,
    // the ungated output, the gate's dL/dy_pre and dL/dZ
    void* X;
    void* Bh;
    void* Ch;
    void* Bph;
    float* thh;
    void* ypre;
    void* dy_pre;
    float* dZ;
    // the recurrence's gradients of the effective inputs (workspace)
    float* dX;
    float* dBh;
    float* dCh;
    float* dBph;
    float* dthh;
    // outputs
    float* dx;
    float* dB;
    float* dC;
    float* dB_prev;
    float* dtheta;
    float* dz;
    float* dB_bias;
    float* dC_bias;
    float* dx_expand;
    float* dz_expand;
};
cudaError_t launch_ex_bwd_inputs(const ExBwdPlan& pl, int io_dtype, cudaStream_t s);
cudaError_t launch_ex_bwd_gate(const ExBwdPlan& pl, int io_dtype, cudaStream_t s);
cudaError_t launch_ex_bwd_post(const ExBwdPlan& pl, int io_dtype, cudaStream_t s);
// *dst |= *src (device status words)
cudaError_t launch_status_or(uint32_t* dst, const uint32_t* src, cudaStream_t s);

// B_prev <- B[:, t] for every (batch, group): the previous-token input of the
// next call, written after every head of the group has read the old value.
cudaError_t launch_copy_prev(void* B_prev, const void* B, long long T, long long t, int batch,
                             size_t row_bytes, cudaStream_t s);

}  // namespace m3
