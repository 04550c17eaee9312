// scan_noalloc.cu -- prefill entry point for callers that cannot allocate device memory.
//
// m3_scan_fwd needs a small caller-owned workspace.  Some callers have no way to get one:
// a plugin running inside a host framework whose caching allocator owns all of the
// device memory, or a latency-critical serving loop that must not call cudaMalloc
// (it can synchronise the device and fragment a pre-reserved pool).  For them this
// file keeps one fixed scratch buffer in a file-scope __device__ array -- every GPU
// that loads the library holds it until the process exits -- and runs the regular
// prefill entry point with that buffer as its workspace.
#include <mutex>

#include "m3_internal.h"

namespace {

// Stated maximum of the scratch this entry point can lend to a prefill call.
constexpr size_t kNoAllocScratchBytes = 64 * 1024;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_m3_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];   // device address of the array, per device ordinal

// In host code the array's name only stands in for the device symbol; the address a
// kernel may use is looked up once per device, with that device current.
m3_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return M3_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return M3_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_m3_noalloc_scratch) != cudaSuccess || !p)
            return M3_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return M3_OK;
}

}  // namespace

extern "C" m3_status m3_scan_fwd_noalloc(const m3_dims* dims, int32_t seqlen, int32_t chunk,
                                         const void* x, const void* B, const void* C,
                                         const float* dt, const float* A, const float* lam,
                                         const float* theta, const float* D, m3_state* state,
                                         void* y, uint32_t flags, void* stream) {
    size_t need = 0;
    m3_status st = m3_scan_workspace_bytes(dims, seqlen, chunk, &need);
    if (st != M3_OK) return st;
    if (need > kNoAllocScratchBytes) return M3_ERR_WORKSPACE;
    void* ws = nullptr;
    if ((st = scratch_address(&ws)) != M3_OK) return st;
    return m3_scan_fwd(dims, seqlen, chunk, x, B, C, dt, A, lam, theta, D, state, y, ws,
                       kNoAllocScratchBytes, flags, stream);
}
