// m3_api.cu -- the C ABI (include/m3.h): host-side validation and dispatch.
//
// Every argument is checked here before anything is launched; the kernels assume
// validated input.  Nothing in this file allocates device memory or synchronises,
// except m3_query_status.
#include <cstring>

#include "m3_internal.h"

using namespace m3;

namespace {

constexpr size_t kStatusBytes = 256;   // status block at the head of the workspace

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t io_bytes(int io_dtype) { return io_dtype == M3_BF16 ? 2 : 4; }

m3_status check_dims(const m3_dims* d) {
    if (!d) return M3_ERR_NULL;
    if (d->io_dtype != M3_F32 && d->io_dtype != M3_BF16) return M3_ERR_DTYPE;
    if (d->batch < 1 || d->nheads < 1 || d->ngroups < 1 || d->headdim < 1 || d->dstate < 2 ||
        d->rank < 1)
        return M3_ERR_SHAPE;
    if (d->nheads % d->ngroups) return M3_ERR_SHAPE;
    if (d->dstate % 2) return M3_ERR_SHAPE;
    if (d->dstate > 1024 || d->headdim > 1024 || d->rank > 8) return M3_ERR_UNSUPPORTED;
    return M3_OK;
}

m3_status check_state(const m3_state* st) {
    if (!st || !st->h || !st->x_prev || !st->B_prev) return M3_ERR_NULL;
    if (!aligned(st->h, 16) || !aligned(st->x_prev, 16) || !aligned(st->B_prev, 16))
        return M3_ERR_ALIGN;
    return M3_OK;
}

bool rank_has_kernel(int R) { return R == 1 || R == 2 || R == 3 || R == 4 || R == 8; }

// SIMT prefill thread shape: ns lanes per state column (a power of two <= 32),
// ppt pairs per lane; P * ns threads.  At most 8 pairs per lane, and more lanes (down to
// one pair each) while the CTA has fewer than 256 threads: one CTA per (batch, head) runs
// its tokens one after the other, so a small CTA would leave the token chain to a few
// threads (measured on B200 for b1 H2 P16 N16 T256: 16 threads, 460 us per call).
bool simt_shape(int N, int P, int* ppt, int* ns) {
    const int pairs = N / 2;
    int n = 1;
    while ((pairs + n - 1) / n > 8 && n < 32) n *= 2;
    while (P * n < 256 && 2 * n <= pairs && n < 32) n *= 2;
    int p = (pairs + n - 1) / n;
    while (P * n > 1024 && n > 1) {
        n /= 2;
        p = (pairs + n - 1) / n;
    }
    if (p > 32 || P * n > 1024) return false;
    *ppt = p;
    *ns = n;
    return true;
}

// Decode thread shape: P/4 column chunks x (N/2)/ppt row groups.  More state pairs per
// thread keep more 16-byte loads in flight per register: SISO (R = 1) takes 8 pairs per
// thread when that leaves at least 128 threads (measured on B200, batch 256, N 128: 169 us
// per token against 204 us with 4 pairs); MIMO, with R times the arithmetic per element,
// stays at 4.
bool decode_shape(int N, int P, int R, int* ppt) {
    if (P % 4 || P > 256 || N > 256) return false;
    const int pairs = N / 2, cpr = P / 4;
    // MIMO: 8 pairs per thread in the rank-2R packed kernel, with whole warps of at least 64
    // threads (batch 256, N 64, R 4: see the decode notes)
    if (R != 1 && pairs % 8 == 0) {
        const int threads = cpr * (pairs / 8);
        if (threads >= 64 && threads <= 512 && threads % 32 == 0) {
            *ppt = 8;
            return true;
        }
    }
    for (int c : {8, 4, 2, 1}) {
        if (pairs % c || (c == 8 && R != 1)) continue;
        const int threads = cpr * (pairs / c);
        if (threads <= 512 && (threads >= 128 || c == 1)) {
            *ppt = c;
            return true;
        }
    }
    return false;
}

m3_status launch_status(cudaError_t e) {
    if (e == cudaSuccess) return M3_OK;
    if (e == cudaErrorNotSupported) return M3_ERR_UNSUPPORTED;
    return M3_ERR_LAUNCH;
}

}  // namespace

extern "C" {

const char* m3_status_string(m3_status s) {
    switch (s) {
        case M3_OK: return "ok";
        case M3_ERR_NULL: return "a required pointer is NULL";
        case M3_ERR_SHAPE: return "dimensions, seqlen or chunk out of range";
        case M3_ERR_DTYPE: return "unknown io dtype";
        case M3_ERR_ALIGN: return "pointer not aligned as documented";
        case M3_ERR_UNSUPPORTED: return "shape not supported by any kernel of this build";
        case M3_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case M3_ERR_LAUNCH: return "kernel launch failed";
        case M3_ERR_TIMEOUT: return "a bounded device-side wait timed out";
        case M3_ERR_CUDA: return "CUDA runtime call failed";
        case M3_ERR_RANGE: return "an input value is outside its documented range (debug checks)";
    }
    return "unknown status";
}

m3_status m3_state_bytes(const m3_dims* d, size_t* h_bytes, size_t* x_prev_bytes,
                         size_t* B_prev_bytes) {
    m3_status st = check_dims(d);
    if (st != M3_OK) return st;
    const size_t e = io_bytes(d->io_dtype);
    if (h_bytes) *h_bytes = sizeof(float) * (size_t)d->batch * d->nheads * d->dstate * d->headdim;
    if (x_prev_bytes) *x_prev_bytes = e * (size_t)d->batch * d->nheads * d->rank * d->headdim;
    if (B_prev_bytes) *B_prev_bytes = e * (size_t)d->batch * d->ngroups * d->rank * d->dstate;
    return M3_OK;
}

m3_status m3_state_init(const m3_dims* d, m3_state* state, const float* h0, void* stream) {
    m3_status st = check_dims(d);
    if (st != M3_OK) return st;
    if ((st = check_state(state)) != M3_OK) return st;
    size_t hb, xb, bb;
    m3_state_bytes(d, &hb, &xb, &bb);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = h0 ? cudaMemcpyAsync(state->h, h0, hb, cudaMemcpyDeviceToDevice, s)
                       : cudaMemsetAsync(state->h, 0, hb, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(state->x_prev, 0, xb, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(state->B_prev, 0, bb, s);
    return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

}  // extern "C"

namespace {

bool bc_norm_on(const m3_extras* ex) { return ex && ex->bc_norm_eps > 0.f; }
bool bc_any(const m3_extras* ex) { return ex && (ex->B_bias || ex->C_bias || ex->bc_norm_eps > 0.f); }

// Bytes of the BCNorm scale buffer after the status block (256-byte aligned).  The
// workspace is laid out as [status block][BCNorm scales][tensor-core segment records].
size_t bc_bytes(const m3_dims* d, int32_t seqlen, const m3_extras* ex) {
    if (!bc_norm_on(ex)) return 0;
    const size_t n = sizeof(float) * bc_scale_floats(d->batch, seqlen, d->ngroups, d->rank);
    return (n + 255) / 256 * 256;
}

}  // namespace

extern "C" {

m3_status m3_scan_workspace_bytes_ex(const m3_dims* d, int32_t seqlen, int32_t chunk,
                                     const m3_extras* ex, size_t* bytes) {
    m3_status st = m3_scan_workspace_bytes(d, seqlen, chunk, bytes);
    if (st != M3_OK) return st;
    *bytes += bc_bytes(d, seqlen, ex);
    return M3_OK;
}

m3_status m3_scan_workspace_bytes(const m3_dims* d, int32_t seqlen, int32_t chunk, size_t* bytes) {
    m3_status st = check_dims(d);
    if (st != M3_OK) return st;
    if (!bytes) return M3_ERR_NULL;
    if (seqlen < 0) return M3_ERR_SHAPE;
    if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return M3_ERR_SHAPE;
    size_t extra = 0;
    const int qt = scan_tc_chunk(d->dstate, d->headdim, d->rank, chunk, d->nheads);
    if (d->io_dtype == M3_BF16 && qt)
        extra = scan_tc_workspace_bytes(d->batch, d->nheads, d->dstate, d->headdim, d->rank,
                                        seqlen, qt);
    *bytes = kStatusBytes + ((extra + 255) / 256) * 256;
    return M3_OK;
}

}  // extern "C"

namespace m3 {

m3_status scan_validate(const m3_dims* d, int32_t seqlen, int32_t chunk, const void* x,
                        const void* B, const void* C, const float* dt, const float* A,
                        const float* lam, const float* theta, const float* D,
                        const m3_extras* ex, const m3_state* state, const void* y,
                        uint32_t flags, size_t* need) {
    const void* z = ex ? ex->z : nullptr;
    m3_status st = check_dims(d);
    if (st != M3_OK) return st;
    if (seqlen < 0) return M3_ERR_SHAPE;
    if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return M3_ERR_SHAPE;
    if ((st = check_state(state)) != M3_OK) return st;
    // the minimum: the status block and the BCNorm scales; the segment records that
    // m3_scan_workspace_bytes adds are optional (without them the call runs unsegmented)
    *need = kStatusBytes + bc_bytes(d, seqlen, ex);
    if (seqlen == 0) return M3_OK;   // no tokens: nothing is read, written or launched
    if (!x || !B || !C || !dt || !A || !lam || !theta || !y) return M3_ERR_NULL;
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16) ||
        !aligned(dt, 4) || !aligned(A, 4) || !aligned(lam, 4) || !aligned(theta, 4) ||
        (D && !aligned(D, 4)) || (z && !aligned(z, 16)) ||
        (ex && ex->B_bias && !aligned(ex->B_bias, 4)) || (ex && ex->C_bias && !aligned(ex->C_bias, 4)) ||
        (ex && ex->x_expand && !aligned(ex->x_expand, 16)) ||
        (ex && ex->z_expand && !aligned(ex->z_expand, 16)))
        return M3_ERR_ALIGN;
    if (ex && !(ex->bc_norm_eps >= 0.f)) return M3_ERR_SHAPE;   // negative or NaN epsilon
    if (ex && ex->z_expand && !z) return M3_ERR_NULL;           // an expanded gate needs z
    const int N = d->dstate, P = d->headdim, R = d->rank;
    const int qt = scan_tc_chunk(N, P, R, chunk, d->nheads);
    const bool use_tc = !(flags & M3_FLAG_FORCE_SIMT) && d->io_dtype == M3_BF16 && qt &&
                        aligned(dt, 16) && aligned(A, 16) && aligned(lam, 16) &&
                        aligned(theta, 16);
    int ppt = 0, ns = 0;
    if (!use_tc && (!rank_has_kernel(R) || !simt_shape(N, P, &ppt, &ns)))
        return M3_ERR_UNSUPPORTED;
    return M3_OK;
}

}  // namespace m3

namespace {

// Prefill with the optional fused parts of `ex` (null: none); every check happens before
// any launch.
m3_status scan_impl(const m3_dims* d, int32_t seqlen, int32_t chunk, const void* x,
                    const void* B, const void* C, const float* dt, const float* A,
                    const float* lam, const float* theta, const float* D, const m3_extras* ex,
                    m3_state* state, void* y, void* workspace, size_t workspace_bytes,
                    uint32_t flags, void* stream) {
    const void* z = ex ? ex->z : nullptr;
    size_t need = 0;
    m3_status st = scan_validate(d, seqlen, chunk, x, B, C, dt, A, lam, theta, D, ex, state, y,
                                 flags, &need);
    if (st != M3_OK || seqlen == 0) return st;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return M3_ERR_WORKSPACE;
    const size_t base = kStatusBytes;   // the BCNorm scales follow the status block

    const int N = d->dstate, P = d->headdim, R = d->rank;
    // the tensor-core kernel reads dt / A / lam / theta with TMA (16-byte aligned rows)
    const int qt = scan_tc_chunk(N, P, R, chunk, d->nheads);
    const bool use_tc = !(flags & M3_FLAG_FORCE_SIMT) && d->io_dtype == M3_BF16 && qt &&
                        aligned(dt, 16) && aligned(A, 16) && aligned(lam, 16) &&
                        aligned(theta, 16);
    int ppt = 0, ns = 0;
    if (!use_tc) simt_shape(N, P, &ppt, &ns);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    ScanArgs a;
    std::memset(&a, 0, sizeof(a));
    a.x = x; a.B = B; a.C = C; a.dt = dt; a.A = A; a.lam = lam; a.theta = theta; a.D = D;
    a.h = state->h; a.x_prev = state->x_prev; a.B_prev = state->B_prev; a.y = y; a.z = z;
    a.B_bias = ex ? ex->B_bias : nullptr;
    a.C_bias = ex ? ex->C_bias : nullptr;
    a.bc = bc_any(ex);
    a.x_expand = ex ? ex->x_expand : nullptr;
    a.z_expand = ex ? ex->z_expand : nullptr;
    a.bc_scale = bc_norm_on(ex) ? reinterpret_cast<const float*>(static_cast<char*>(workspace) + base)
                                : nullptr;
    a.status = static_cast<uint32_t*>(workspace);
    a.ws = static_cast<char*>(workspace) + need;
    a.ws_bytes = workspace_bytes - need;
    a.T = seqlen; a.batch = d->batch; a.H = d->nheads; a.G = d->ngroups; a.P = P; a.N = N;
    a.chunk = use_tc ? qt : chunk; a.ppt = ppt; a.ns = ns; a.flags = flags;

    if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s) != cudaSuccess) return M3_ERR_CUDA;
    cudaError_t e = cudaSuccess;
    if (flags & M3_FLAG_DEBUG_CHECKS) {
        const size_t b = d->batch, T = seqlen, H = d->nheads, G = d->ngroups;
        const size_t xw = (ex && ex->x_expand) ? 1 : R, zw = (ex && ex->z_expand) ? 1 : R;
        RangeCheckArgs rc;
        std::memset(&rc, 0, sizeof(rc));
        rc.x = x; rc.n_x = b * T * H * xw * P;
        rc.B = B; rc.C = C; rc.n_BC = b * T * G * R * N;
        rc.z = z; rc.n_z = z ? b * T * H * zw * P : 0;
        rc.x_prev = state->x_prev; rc.n_xp = b * H * R * P;
        rc.B_prev = state->B_prev; rc.n_bp = b * G * R * N;
        rc.dt = dt; rc.A = A; rc.lam = lam; rc.n_coef = b * T * H;
        rc.theta = theta; rc.n_theta = b * T * G * (N / 2);
        rc.D = D; rc.n_D = D ? H : 0;
        rc.h = state->h; rc.n_h = b * H * N * P;
        rc.status = a.status;
        e = launch_range_checks(rc, d->io_dtype, s);
        if (e != cudaSuccess) return launch_status(e);
    }
    if (a.bc_scale)
        e = launch_bc_scales(a, R, d->io_dtype, ex->bc_norm_eps,
                             reinterpret_cast<float*>(static_cast<char*>(workspace) + base), s);
    if (e != cudaSuccess) return launch_status(e);
    e = use_tc ? launch_scan_tc(a, R, s) : launch_scan_simt(a, R, d->io_dtype, s);
    if (e != cudaSuccess) return launch_status(e);
    const size_t row = io_bytes(d->io_dtype) * (size_t)d->ngroups * R * N;
    e = launch_copy_prev(state->B_prev, B, seqlen, seqlen - 1, d->batch, row, s);
    return launch_status(e);
}

// Decode step with an optional output gate z (null: none).
m3_status decode_impl(const m3_dims* d, const void* x, const void* B, const void* C,
                      const float* dt, const float* A, const float* lam, const float* theta,
                      const float* D, const m3_extras* ex, m3_state* state, void* y,
                      uint32_t flags, void* stream) {
    const void* z = ex ? ex->z : nullptr;
    m3_status st = check_dims(d);
    if (st != M3_OK) return st;
    if (!x || !B || !C || !dt || !A || !lam || !theta || !y) return M3_ERR_NULL;
    if ((st = check_state(state)) != M3_OK) return st;
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16) ||
        !aligned(dt, 4) || !aligned(A, 4) || !aligned(lam, 4) || !aligned(theta, 4) ||
        (D && !aligned(D, 4)) || (z && !aligned(z, 16)) ||
        (ex && ex->B_bias && !aligned(ex->B_bias, 4)) || (ex && ex->C_bias && !aligned(ex->C_bias, 4)) ||
        (ex && ex->x_expand && !aligned(ex->x_expand, 16)) ||
        (ex && ex->z_expand && !aligned(ex->z_expand, 16)))
        return M3_ERR_ALIGN;
    if (ex && !(ex->bc_norm_eps >= 0.f)) return M3_ERR_SHAPE;
    if (ex && ex->z_expand && !z) return M3_ERR_NULL;
    if (flags & M3_FLAG_DEBUG_CHECKS) return M3_ERR_UNSUPPORTED;   // no status word to report into
    int ppt = 0;
    if (!rank_has_kernel(d->rank) || !decode_shape(d->dstate, d->headdim, d->rank, &ppt))
        return M3_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.x = x; a.B = B; a.C = C; a.dt = dt; a.A = A; a.lam = lam; a.theta = theta; a.D = D;
    a.h = state->h; a.x_prev = state->x_prev; a.B_prev = state->B_prev; a.y = y; a.z = z;
    a.B_bias = ex ? ex->B_bias : nullptr;
    a.C_bias = ex ? ex->C_bias : nullptr;
    a.bc_eps = ex ? ex->bc_norm_eps : 0.f;
    a.x_expand = ex ? ex->x_expand : nullptr;
    a.z_expand = ex ? ex->z_expand : nullptr;
    a.H = d->nheads; a.G = d->ngroups; a.P = d->headdim; a.N = d->dstate;
    a.ppt = ppt; a.flags = flags;
    cudaError_t e = decode_stream_ok(a, d->rank)
                        ? launch_decode_stream(a, d->batch, d->rank, d->io_dtype, s)
                        : launch_decode(a, d->batch, d->rank, d->io_dtype, s);
    if (e != cudaSuccess) return launch_status(e);
    const size_t row = io_bytes(d->io_dtype) * (size_t)d->ngroups * d->rank * d->dstate;
    e = launch_copy_prev(state->B_prev, B, 1, 0, d->batch, row, s);
    return launch_status(e);
}

}  // namespace

extern "C" {

m3_status m3_scan_fwd(const m3_dims* d, int32_t seqlen, int32_t chunk, const void* x,
                      const void* B, const void* C, const float* dt, const float* A,
                      const float* lam, const float* theta, const float* D, m3_state* state,
                      void* y, void* workspace, size_t workspace_bytes, uint32_t flags,
                      void* stream) {
    return scan_impl(d, seqlen, chunk, x, B, C, dt, A, lam, theta, D, nullptr, state, y,
                     workspace, workspace_bytes, flags, stream);
}

m3_status m3_scan_fwd_ex(const m3_dims* d, int32_t seqlen, int32_t chunk, const void* x,
                         const void* B, const void* C, const float* dt, const float* A,
                         const float* lam, const float* theta, const float* D,
                         const m3_extras* ex, m3_state* state, void* y, void* workspace,
                         size_t workspace_bytes, uint32_t flags, void* stream) {
    return scan_impl(d, seqlen, chunk, x, B, C, dt, A, lam, theta, D, ex, state, y, workspace,
                     workspace_bytes, flags, stream);
}

m3_status m3_scan_fwd_gated(const m3_dims* d, int32_t seqlen, int32_t chunk, const void* x,
                            const void* B, const void* C, const float* dt, const float* A,
                            const float* lam, const float* theta, const float* D,
                            const void* z, m3_state* state, void* y, void* workspace,
                            size_t workspace_bytes, uint32_t flags, void* stream) {
    if (!z && seqlen != 0) return M3_ERR_NULL;
    m3_extras ex;
    std::memset(&ex, 0, sizeof(ex));
    ex.z = z;
    return scan_impl(d, seqlen, chunk, x, B, C, dt, A, lam, theta, D, &ex, state, y, workspace,
                     workspace_bytes, flags, stream);
}

m3_status m3_decode_step(const m3_dims* d, const void* x, const void* B, const void* C,
                         const float* dt, const float* A, const float* lam,
                         const float* theta, const float* D, m3_state* state, void* y,
                         uint32_t flags, void* stream) {
    return decode_impl(d, x, B, C, dt, A, lam, theta, D, nullptr, state, y, flags, stream);
}

m3_status m3_decode_step_ex(const m3_dims* d, const void* x, const void* B, const void* C,
                            const float* dt, const float* A, const float* lam,
                            const float* theta, const float* D, const m3_extras* ex,
                            m3_state* state, void* y, uint32_t flags, void* stream) {
    return decode_impl(d, x, B, C, dt, A, lam, theta, D, ex, state, y, flags, stream);
}

m3_status m3_decode_step_gated(const m3_dims* d, const void* x, const void* B, const void* C,
                               const float* dt, const float* A, const float* lam,
                               const float* theta, const float* D, const void* z,
                               m3_state* state, void* y, uint32_t flags, void* stream) {
    if (!z) return M3_ERR_NULL;
    m3_extras ex;
    std::memset(&ex, 0, sizeof(ex));
    ex.z = z;
    return decode_impl(d, x, B, C, dt, A, lam, theta, D, &ex, state, y, flags, stream);
}

m3_status m3_scan_bwd_workspace_bytes(const m3_dims* d, int32_t seqlen, size_t* bytes) {
    m3_status st = check_dims(d);
    if (st != M3_OK) return st;
    if (!bytes) return M3_ERR_NULL;
    if (seqlen < 0) return M3_ERR_SHAPE;
    const size_t fl = scan_bwd_workspace(d->batch, d->nheads, d->dstate, d->headdim, d->rank,
                                         seqlen).floats;
    size_t need = ((fl * sizeof(float) + 255) / 256) * 256;
    if (scan_bwd_tc_ok(d->io_dtype, d->dstate, d->headdim, d->rank)) {
        const size_t tc = scan_bwd_tc_workspace_bytes(d->batch, d->nheads, d->dstate, d->rank, seqlen);
        if (tc > need) need = tc;
    }
    *bytes = kStatusBytes + need;
    return M3_OK;
}

m3_status m3_scan_bwd(const m3_dims* d, int32_t seqlen, const void* x, const void* B,
                      const void* C, const float* dt, const float* A, const float* lam,
                      const float* theta, const float* D, const m3_state* state0,
                      const void* dy, const float* dhT, const m3_grads* gr, void* workspace,
                      size_t workspace_bytes, uint32_t flags, void* stream) {
    m3_status st = check_dims(d);
    if (st != M3_OK) return st;
    if (seqlen < 0) return M3_ERR_SHAPE;
    if ((st = check_state(state0)) != M3_OK) return st;
    if (!gr) return M3_ERR_NULL;
    if (seqlen == 0) return M3_OK;
    if (!x || !B || !C || !dt || !A || !lam || !theta || !dy) return M3_ERR_NULL;
    if (!gr->dx || !gr->dB || !gr->dC || !gr->ddt || !gr->dA || !gr->dlam || !gr->dtheta ||
        !gr->dh0 || !gr->dx_prev || !gr->dB_prev)
        return M3_ERR_NULL;
    const void* f4[] = {dt, A, lam, theta, D, dhT, gr->dx, gr->dB, gr->dC, gr->ddt, gr->dA,
                        gr->dlam, gr->dtheta, gr->dD, gr->dh0, gr->dx_prev, gr->dB_prev};
    for (const void* q : f4)
        if (q && !aligned(q, 4)) return M3_ERR_ALIGN;
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(dy, 16))
        return M3_ERR_ALIGN;
    const int N = d->dstate, P = d->headdim, R = d->rank;
    if (!scan_bwd_shape_ok(N, P, R)) return M3_ERR_UNSUPPORTED;
    size_t need = 0;
    m3_scan_bwd_workspace_bytes(d, seqlen, &need);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return M3_ERR_WORKSPACE;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.x = x; a.B = B; a.C = C; a.dt = dt; a.A = A; a.lam = lam; a.theta = theta; a.D = D;
    a.h0 = state0->h; a.x_prev = state0->x_prev; a.B_prev = state0->B_prev;
    a.dy = dy; a.dhT = dhT;
    a.dx = gr->dx; a.dB = gr->dB; a.dC = gr->dC; a.ddt = gr->ddt; a.dA = gr->dA;
    a.dlam = gr->dlam; a.dtheta = gr->dtheta; a.dD = D ? gr->dD : nullptr; a.dh0 = gr->dh0;
    a.dx_prev = gr->dx_prev; a.dB_prev = gr->dB_prev;
    const BwdWorkspace wp = scan_bwd_workspace(d->batch, d->nheads, N, P, R, seqlen);
    float* ws = reinterpret_cast<float*>(static_cast<char*>(workspace) + kStatusBytes);
    a.seg = wp.seg; a.nseg = wp.nseg;
    a.ckpt = ws + wp.ckpt; a.segbuf = ws + wp.segbuf; a.pB = ws + wp.pB; a.pC = ws + wp.pC;
    a.pth = ws + wp.pth; a.pBprev = ws + wp.pBprev; a.pD = ws + wp.pD;
    a.T = seqlen; a.batch = d->batch; a.H = d->nheads; a.G = d->ngroups; a.P = P; a.N = N;
    a.flags = flags;
    if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s) != cudaSuccess) return M3_ERR_CUDA;
    if (flags & M3_FLAG_DEBUG_CHECKS) {
        const size_t b = d->batch, T = seqlen, H = d->nheads, G = d->ngroups;
        RangeCheckArgs rc;
        std::memset(&rc, 0, sizeof(rc));
        rc.x = x; rc.n_x = b * T * H * R * P;
        rc.B = B; rc.C = C; rc.n_BC = b * T * G * R * N;
        rc.z = dy; rc.n_z = b * T * H * R * P;   // dL/dy: finite
        rc.x_prev = state0->x_prev; rc.n_xp = b * H * R * P;
        rc.B_prev = state0->B_prev; rc.n_bp = b * G * R * N;
        rc.dt = dt; rc.A = A; rc.lam = lam; rc.n_coef = b * T * H;
        rc.theta = theta; rc.n_theta = b * T * G * (N / 2);
        rc.D = D; rc.n_D = D ? H : 0;
        rc.h = state0->h; rc.n_h = b * H * N * P;
        rc.status = static_cast<uint32_t*>(workspace);
        cudaError_t e = launch_range_checks(rc, d->io_dtype, s);
        if (e != cudaSuccess) return launch_status(e);
    }
    const bool tc = !(flags & M3_FLAG_FORCE_SIMT) && scan_bwd_tc_ok(d->io_dtype, N, P, R) &&
                    aligned(gr->dx, 16) && aligned(gr->dB, 16) && aligned(gr->dC, 16);
    if (tc) {
        // the group-shared gradients and dD are accumulated with atomics
        const size_t b = d->batch, T = seqlen, G = d->ngroups, Rs = R;
        if (cudaMemsetAsync(gr->dB, 0, b * T * G * Rs * N * sizeof(float), s) != cudaSuccess ||
            cudaMemsetAsync(gr->dC, 0, b * T * G * Rs * N * sizeof(float), s) != cudaSuccess ||
            cudaMemsetAsync(gr->dtheta, 0, b * T * G * (N / 2) * sizeof(float), s) != cudaSuccess ||
            cudaMemsetAsync(gr->dB_prev, 0, b * G * Rs * N * sizeof(float), s) != cudaSuccess ||
            (D && gr->dD && cudaMemsetAsync(gr->dD, 0, d->nheads * sizeof(float), s) != cudaSuccess))
            return M3_ERR_CUDA;
        return launch_status(launch_scan_bwd_tc(a, R, static_cast<char*>(workspace) + kStatusBytes,
                                                static_cast<uint32_t*>(workspace),
                                                (flags & M3_FLAG_TEST_STALL) ? 50000000ull
                                                                             : 2000000000ull,
                                                s));
    }
    return launch_status(launch_scan_bwd(a, R, d->io_dtype, s));
}

}  // extern "C"

namespace {

// the fused extras of a backward call: which parts are on and where their buffers sit in
// the workspace (byte offsets; the recurrence backward's own workspace comes first, so that
// its status word is the call's)
struct ExLayout {
    m3_dims de;   // effective dims: one group per head when the BC map is on
    bool xe, bc, gate;
    size_t inner, fwd, fwd_bytes, hS, xpS, bpS, ypre, dypre, dZ, X, dX, Bh, Ch, Bph, thh;
    size_t dBh, dCh, dBph, dthh, bytes;
};

bool ex_any(const m3_extras* ex) {
    return ex && (ex->z || ex->B_bias || ex->C_bias || ex->bc_norm_eps > 0.f || ex->x_expand ||
                  ex->z_expand);
}

ExLayout ex_layout(const m3_dims* d, int32_t T, const m3_extras* ex) {
    ExLayout L;
    std::memset(&L, 0, sizeof(L));
    L.xe = ex->x_expand != nullptr;
    L.bc = ex->B_bias || ex->C_bias || ex->bc_norm_eps > 0.f;
    L.gate = ex->z != nullptr;
    L.de = *d;
    if (L.bc) L.de.ngroups = d->nheads;
    const size_t io = d->io_dtype == M3_BF16 ? 2 : 4;
    const size_t b = d->batch, H = d->nheads, R = d->rank, P = d->headdim, N = d->dstate;
    const size_t bt = b * (size_t)T, Ge = L.de.ngroups;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += (bytes + 255) / 256 * 256;
        return at;
    };
    size_t inner = 0;
    m3_scan_bwd_workspace_bytes(&L.de, T, &inner);
    L.inner = take(inner);
    if (L.gate) {
        m3_scan_workspace_bytes(&L.de, T, 64, &L.fwd_bytes);
        L.fwd = take(L.fwd_bytes);
        L.hS = take(b * H * N * P * 4);
        L.xpS = take(b * H * R * P * io);
        L.bpS = take(b * Ge * R * N * io);
        L.ypre = take(bt * H * R * P * io);
        L.dypre = take(bt * H * R * P * io);
        if (ex->z_expand) L.dZ = take(bt * H * R * P * 4);
    }
    if (L.xe) {
        L.X = take(bt * H * R * P * io);
        L.dX = take(bt * H * R * P * 4);
    }
    if (L.bc) {
        L.Bh = take(bt * H * R * N * io);
        L.Ch = take(bt * H * R * N * io);
        L.Bph = take(b * H * R * N * io);
        L.thh = take(bt * H * (N / 2) * 4);
        L.dBh = take(bt * H * R * N * 4);
        L.dCh = take(bt * H * R * N * 4);
        L.dBph = take(b * H * R * N * 4);
        L.dthh = take(bt * H * (N / 2) * 4);
    }
    L.bytes = o;
    return L;
}

}  // namespace

extern "C" {

m3_status m3_scan_bwd_workspace_bytes_ex(const m3_dims* d, int32_t seqlen, const m3_extras* ex,
                                         size_t* bytes) {
    if (ex && !(ex->bc_norm_eps >= 0.f)) return M3_ERR_SHAPE;   // negative or NaN epsilon
    if (!ex_any(ex)) return m3_scan_bwd_workspace_bytes(d, seqlen, bytes);
    m3_status st = check_dims(d);
    if (st != M3_OK) return st;
    if (!bytes) return M3_ERR_NULL;
    if (seqlen < 0 || !(ex->bc_norm_eps >= 0.f)) return M3_ERR_SHAPE;
    *bytes = ex_layout(d, seqlen, ex).bytes;
    return M3_OK;
}

m3_status m3_scan_bwd_ex(const m3_dims* d, int32_t seqlen, const void* x, const void* B,
                         const void* C, const float* dt, const float* A, const float* lam,
                         const float* theta, const float* D, const m3_state* state0,
                         const m3_extras* ex, const void* dy, const float* dhT,
                         const m3_grads* gr, const m3_extra_grads* xg, void* workspace,
                         size_t workspace_bytes, uint32_t flags, void* stream) {
    if (ex && !(ex->bc_norm_eps >= 0.f)) return M3_ERR_SHAPE;   // negative or NaN epsilon
    if (!ex_any(ex))
        return m3_scan_bwd(d, seqlen, x, B, C, dt, A, lam, theta, D, state0, dy, dhT, gr,
                           workspace, workspace_bytes, flags, stream);
    m3_status st = check_dims(d);
    if (st != M3_OK) return st;
    if (seqlen < 0 || !(ex->bc_norm_eps >= 0.f)) return M3_ERR_SHAPE;
    if ((st = check_state(state0)) != M3_OK) return st;
    if (!gr || !xg) return M3_ERR_NULL;
    if (ex->z_expand && !ex->z) return M3_ERR_NULL;
    if ((ex->z && !xg->dz) || (ex->B_bias && !xg->dB_bias) || (ex->C_bias && !xg->dC_bias) ||
        (ex->x_expand && !xg->dx_expand) || (ex->z_expand && !xg->dz_expand))
        return M3_ERR_NULL;
    if ((ex->z && !aligned(ex->z, 16)) || (ex->x_expand && !aligned(ex->x_expand, 16)) ||
        (ex->z_expand && !aligned(ex->z_expand, 16)) || (ex->B_bias && !aligned(ex->B_bias, 4)) ||
        (ex->C_bias && !aligned(ex->C_bias, 4)) || (xg->dz && !aligned(xg->dz, 4)) ||
        (xg->dB_bias && !aligned(xg->dB_bias, 4)) || (xg->dC_bias && !aligned(xg->dC_bias, 4)) ||
        (xg->dx_expand && !aligned(xg->dx_expand, 4)) || (xg->dz_expand && !aligned(xg->dz_expand, 4)))
        return M3_ERR_ALIGN;
    if (seqlen == 0) return M3_OK;
    if (!x || !B || !C || !dt || !A || !lam || !theta || !dy) return M3_ERR_NULL;
    if (!gr->dx || !gr->dB || !gr->dC || !gr->ddt || !gr->dA || !gr->dlam || !gr->dtheta ||
        !gr->dh0 || !gr->dx_prev || !gr->dB_prev)
        return M3_ERR_NULL;
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(dy, 16))
        return M3_ERR_ALIGN;
    if (!scan_bwd_shape_ok(d->dstate, d->headdim, d->rank)) return M3_ERR_UNSUPPORTED;
    const ExLayout L = ex_layout(d, seqlen, ex);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < L.bytes) return M3_ERR_WORKSPACE;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* base = static_cast<char*>(workspace);
    const size_t io = d->io_dtype == M3_BF16 ? 2 : 4;
    const size_t b = d->batch, H = d->nheads, R = d->rank, P = d->headdim, N = d->dstate;
    ExBwdPlan pl;
    std::memset(&pl, 0, sizeof(pl));
    pl.batch = d->batch; pl.H = d->nheads; pl.G = d->ngroups; pl.R = R; pl.P = P; pl.N = N;
    pl.T = seqlen; pl.eps = ex->bc_norm_eps;
    pl.x = x; pl.B = B; pl.C = C; pl.B_prev = state0->B_prev; pl.theta = theta; pl.z = ex->z;
    pl.B_bias = ex->B_bias; pl.C_bias = ex->C_bias; pl.x_expand = ex->x_expand;
    pl.z_expand = ex->z_expand; pl.dy = dy;
    pl.dx = gr->dx; pl.dB = gr->dB; pl.dC = gr->dC; pl.dB_prev = gr->dB_prev;
    pl.dtheta = gr->dtheta; pl.dz = xg->dz; pl.dB_bias = xg->dB_bias; pl.dC_bias = xg->dC_bias;
    pl.dx_expand = xg->dx_expand; pl.dz_expand = xg->dz_expand;
    if (L.xe) {
        pl.X = base + L.X;
        pl.dX = reinterpret_cast<float*>(base + L.dX);
    }
    if (L.bc) {
        pl.Bh = base + L.Bh; pl.Ch = base + L.Ch; pl.Bph = base + L.Bph;
        pl.thh = reinterpret_cast<float*>(base + L.thh);
        pl.dBh = reinterpret_cast<float*>(base + L.dBh);
        pl.dCh = reinterpret_cast<float*>(base + L.dCh);
        pl.dBph = reinterpret_cast<float*>(base + L.dBph);
        pl.dthh = reinterpret_cast<float*>(base + L.dthh);
    }
    if (L.gate) {
        pl.ypre = base + L.ypre;
        pl.dy_pre = base + L.dypre;
        pl.dZ = ex->z_expand ? reinterpret_cast<float*>(base + L.dZ) : xg->dz;
    }
    // the parameter gradients are sums accumulated with atomics
    float* zero[] = {xg->dx_expand, xg->dz_expand, xg->dB_bias, xg->dC_bias};
    const size_t zn[] = {H * R * P, H * R * P, H * N, H * N};
    for (int i = 0; i < 4; ++i)
        if (zero[i] && cudaMemsetAsync(zero[i], 0, zn[i] * sizeof(float), s) != cudaSuccess)
            return M3_ERR_CUDA;
    cudaError_t e = launch_ex_bwd_inputs(pl, d->io_dtype, s);
    if (e != cudaSuccess) return launch_status(e);
    const void* Xe = L.xe ? pl.X : x;
    const void* Be = L.bc ? pl.Bh : B;
    const void* Ce = L.bc ? pl.Ch : C;
    const float* the = L.bc ? pl.thh : theta;
    const void* Bpe = L.bc ? pl.Bph : state0->B_prev;
    const uint32_t fwd_flags = flags & (M3_FLAG_THETA_IS_ANGLE | M3_FLAG_FORCE_SIMT);
    if (L.gate) {
        // the ungated output y_pre: the forward from a copy of the starting state
        m3_state ss;
        ss.h = reinterpret_cast<float*>(base + L.hS);
        ss.x_prev = base + L.xpS;
        ss.B_prev = base + L.bpS;
        if (cudaMemcpyAsync(ss.h, state0->h, b * H * N * P * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(ss.x_prev, state0->x_prev, b * H * R * P * io, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(ss.B_prev, Bpe, b * L.de.ngroups * R * N * io, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return M3_ERR_CUDA;
        st = m3_scan_fwd(&L.de, seqlen, 64, Xe, Be, Ce, dt, A, lam, the, D, &ss, pl.ypre,
                         base + L.fwd, L.fwd_bytes, fwd_flags, stream);
        if (st != M3_OK) return st;
        if ((e = launch_ex_bwd_gate(pl, d->io_dtype, s)) != cudaSuccess) return launch_status(e);
    }
    m3_state s0;
    s0.h = state0->h;
    s0.x_prev = state0->x_prev;
    s0.B_prev = const_cast<void*>(Bpe);
    m3_grads ig = *gr;
    if (L.xe) ig.dx = pl.dX;
    if (L.bc) {
        ig.dB = pl.dBh;
        ig.dC = pl.dCh;
        ig.dtheta = pl.dthh;
        ig.dB_prev = pl.dBph;
    }
    size_t inner = 0;
    m3_scan_bwd_workspace_bytes(&L.de, seqlen, &inner);
    st = m3_scan_bwd(&L.de, seqlen, Xe, Be, Ce, dt, A, lam, the, D, &s0, L.gate ? pl.dy_pre : dy,
                     dhT, &ig, base + L.inner, inner, flags, stream);
    if (st != M3_OK) return st;
    if (L.gate &&
        (e = launch_status_or(static_cast<uint32_t*>(workspace),
                              reinterpret_cast<const uint32_t*>(base + L.fwd), s)) != cudaSuccess)
        return launch_status(e);
    return launch_status(launch_ex_bwd_post(pl, d->io_dtype, s));
}

m3_status m3_query_status(const void* workspace, void* stream) {
    if (!workspace) return M3_ERR_NULL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return M3_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return M3_ERR_CUDA;
    if (word == 0) return M3_OK;
    if (word & M3_STATUS_TIMEOUT_BIT) return M3_ERR_TIMEOUT;
    if (word & M3_STATUS_RANGE_BIT) return M3_ERR_RANGE;
    return M3_ERR_TIMEOUT;
}

}  // extern "C"
