// checks.cu -- the non-trapping device scan of M3_FLAG_DEBUG_CHECKS.
//
// The recurrence's coefficients are only meaningful inside their ranges ("Technical
// Approach", Proposition 1): the step dt > 0 (after softplus), A <= 0 so that
// alpha = exp(dt A) <= 1, and the trapezoid weight lam in [0, 1] (after sigmoid).  These
// ranges are the caller's contract.  With the debug flag, one extra kernel reads every
// input of the call once and, where a value is out of range or not finite, ORs
// M3_STATUS_RANGE_BIT into the workspace status word (m3_query_status reports
// M3_ERR_RANGE).  It never traps and never changes an input: the call itself still runs.
#include "m3_internal.h"

namespace m3 {

namespace {

template <typename T>
__device__ __forceinline__ bool finite_io(T v) {
    return isfinite(to_f(v));
}

// grid-stride pass over n values of one array; true where every value passed `ok`
template <typename T, typename F>
__device__ __forceinline__ bool all_of(const T* p, size_t n, F ok) {
    bool good = true;
    if (!p) return true;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        good &= ok(p[i]);
    return good;
}

template <typename IO>
__global__ void range_check_kernel(RangeCheckArgs a) {
    bool good = true;
    auto fin = [](IO v) { return finite_io(v); };
    auto finf = [](float v) { return isfinite(v) != 0; };
    good &= all_of(static_cast<const IO*>(a.x), a.n_x, fin);
    good &= all_of(static_cast<const IO*>(a.B), a.n_BC, fin);
    good &= all_of(static_cast<const IO*>(a.C), a.n_BC, fin);
    good &= all_of(static_cast<const IO*>(a.z), a.n_z, fin);
    good &= all_of(static_cast<const IO*>(a.x_prev), a.n_xp, fin);
    good &= all_of(static_cast<const IO*>(a.B_prev), a.n_bp, fin);
    good &= all_of(a.dt, a.n_coef, [](float v) { return isfinite(v) && v > 0.f; });
    good &= all_of(a.A, a.n_coef, [](float v) { return isfinite(v) && v <= 0.f; });
    good &= all_of(a.lam, a.n_coef, [](float v) { return v >= 0.f && v <= 1.f; });
    good &= all_of(a.theta, a.n_theta, finf);
    good &= all_of(a.D, a.n_D, finf);
    good &= all_of(a.h, a.n_h, finf);
    if (__any_sync(0xffffffffu, !good) && (threadIdx.x & 31) == 0)
        atomicOr(a.status, M3_STATUS_RANGE_BIT);
}

}  // namespace

cudaError_t launch_range_checks(const RangeCheckArgs& a, int io_dtype, cudaStream_t s) {
    if (!a.status) return cudaErrorInvalidValue;
    const int threads = 256, blocks = 2 * 148;
    if (io_dtype == M3_BF16)
        range_check_kernel<__nv_bfloat16><<<blocks, threads, 0, s>>>(a);
    else
        range_check_kernel<float><<<blocks, threads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace m3
