// scan_noalloc.cu -- prefill entry point for callers that cannot allocate device memory.
//
// m3_scan_fwd needs a small caller-owned workspace.  Some callers have no way to get one:
// a plugin running inside a host framework whose caching allocator owns all of the
// device memory, or a latency-critical serving loop that must not call cudaMalloc
// (it can synchronise the device and fragment a pre-reserved pool).  For them this
// file keeps one fixed scratch buffer in a file-scope __device__ array -- every GPU
// that loads the library holds it until the process exits -- and runs the regular
// prefill entry point with that buffer as its workspace.
#include "m3_internal.h"

namespace {

// Stated maximum of the scratch this entry point can lend to a prefill call.
constexpr size_t kNoAllocScratchBytes = 64 * 1024;

__device__ __align__(256) unsigned char g_m3_noalloc_scratch[kNoAllocScratchBytes];

// In host code the array's name only stands in for the device symbol: the address a
// kernel may use is looked up with the stream's device current.  The stream must belong
// to the current device (a stream of another device would be handed this device's array).
// The lookup is repeated on every call rather than cached, so that an address never
// outlives a device reset; only the first lookup on a device loads the array there.
m3_status scratch_address(void* stream, void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return M3_ERR_CUDA;
    if (stream) {
        int sdev = -1;
        if (cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &sdev) != cudaSuccess)
            return M3_ERR_CUDA;
        if (sdev != dev) return M3_ERR_UNSUPPORTED;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_m3_noalloc_scratch) != cudaSuccess || !p) return M3_ERR_CUDA;
    *out = p;
    return M3_OK;
}

}  // namespace

extern "C" m3_status m3_scan_fwd_noalloc(const m3_dims* dims, int32_t seqlen, int32_t chunk,
                                         const void* x, const void* B, const void* C,
                                         const float* dt, const float* A, const float* lam,
                                         const float* theta, const float* D, m3_state* state,
                                         void* y, uint32_t flags, void* stream) {
    // every host-side check first: a bad argument is reported before any CUDA call
    size_t need = 0;
    m3_status st = m3::scan_validate(dims, seqlen, chunk, x, B, C, dt, A, lam, theta, D,
                                     nullptr, state, y, flags, &need);
    if (st != M3_OK) return st;
    if (need > kNoAllocScratchBytes) return M3_ERR_WORKSPACE;
    // the status word lives in the shared array and is never read back
    if (flags & M3_FLAG_DEBUG_CHECKS) return M3_ERR_UNSUPPORTED;
    if (seqlen == 0) return M3_OK;
    void* ws = nullptr;
    if ((st = scratch_address(stream, &ws)) != M3_OK) return st;
    return m3_scan_fwd(dims, seqlen, chunk, x, B, C, dt, A, lam, theta, D, state, y, ws,
                       kNoAllocScratchBytes, flags, stream);
}
